"""Host logic of bench.py that needs no GPU: the DRAM-traffic lookup that feeds
roofline.traffic only while the kernel sources match the ncu capture."""
import bench


def test_traffic_reported_only_for_unchanged_sources(tmp_path, monkeypatch):
    digest = bench.sources_digest("gemm_qkv")
    f = tmp_path / "traffic.txt"
    f.write_text("# comment\n"
                 f"class=gemm_qkv workload=w sources={digest} dram_bytes_per_launch=123456 launches=24\n"
                 "class=attention workload=w sources=0000000000000000 dram_bytes_per_launch=99 launches=24\n")
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    value, note = bench.load_traffic("gemm_qkv", "w")
    assert value == 123456.0 and "ncu" in note
    value, note = bench.load_traffic("attention", "w")
    assert value is None and "changed" in note
    value, note = bench.load_traffic("gemm_ffn_up_gelu", "w")
    assert value is None
    value, note = bench.load_traffic("gemm_qkv", "other_workload")
    assert value is None


def test_missing_traffic_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "absent.txt"))
    assert bench.load_traffic("gemm_qkv", "w")[0] is None


def test_gemm_classes_share_a_digest_and_attention_differs():
    assert bench.sources_digest("gemm_qkv") == bench.sources_digest("gemm_out_proj_ln")
    assert bench.sources_digest("gemm_qkv") != bench.sources_digest("attention")
