"""Host logic of bench.py that needs no GPU: the DRAM-traffic lookup that feeds
roofline.traffic only while the kernel sources match the ncu capture."""
import bench


def test_traffic_reported_only_for_unchanged_sources(tmp_path, monkeypatch):
    digest = bench.sources_digest("gemm_qkv")
    f = tmp_path / "traffic.txt"
    f.write_text("# comment\n"
                 f"class=gemm_qkv workload=w sources={digest} dram_bytes_per_launch=123456 launches=24\n"
                 "class=attention workload=w sources=0000000000000000 dram_bytes_per_launch=99 launches=24\n")
    monkeypatch.setattr(bench, "TRAFFIC_GLOB", str(f))
    value, note = bench.load_traffic("gemm_qkv", "w")
    assert value == 123456.0 and "ncu" in note
    value, note = bench.load_traffic("attention", "w")
    assert value is None and "changed" in note
    value, note = bench.load_traffic("gemm_ffn_up_gelu", "w")
    assert value is None
    value, note = bench.load_traffic("gemm_qkv", "other_workload")
    assert value is None


def test_missing_traffic_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "TRAFFIC_GLOB", str(tmp_path / "absent_*.txt"))
    assert bench.load_traffic("gemm_qkv", "w")[0] is None


def test_gemm_classes_share_a_digest_and_attention_differs():
    assert bench.sources_digest("gemm_qkv") == bench.sources_digest("gemm_out_proj_ln")
    assert bench.sources_digest("gemm_qkv") != bench.sources_digest("attention")
    # the quantizer and the small-batch kernel have their own source sets
    assert bench.source_set("quant_e4m3") == "quant" and bench.source_set("small_batch_forward") == "small"
    assert bench.sources_digest("quant_e4m3") != bench.sources_digest("small_batch_forward")
    assert bench.source_set("attention", 512) == "attention_long"
    # the fused embedding + input projection kernel is keyed by its own file
    assert bench.source_set("embed_proj") == "embed_proj"
    assert bench.sources_digest("embed_proj") not in (bench.sources_digest("gemm_qkv"), bench.sources_digest("attention"))


def test_embedding_kernel_counts_the_input_projection_flops():
    arch = {"hidden": 768, "emb": 128, "ffn": 2048, "out_dim": 512, "n_exec": 12}
    f = bench.flops_per_class([10, 20], arch, 30)
    assert f["embed_proj"] == f["gemm_in_proj"] == 2.0 * 30 * 128 * 768


def test_long_attention_has_its_own_digest_and_lines(tmp_path, monkeypatch):
    """Batches with a sequence longer than 128 run the long-sequence attention
    kernel: its traffic line is keyed by that kernel's sources."""
    short, long_ = bench.sources_digest("attention", 128), bench.sources_digest("attention", 512)
    assert short != long_
    assert bench.sources_digest("gemm_qkv", 512) == bench.sources_digest("gemm_qkv", 128)
    (tmp_path / "dram_traffic_a.txt").write_text(f"class=attention workload=s sources={short} dram_bytes_per_launch=5\n")
    (tmp_path / "dram_traffic_b.txt").write_text(f"class=attention workload=l sources={long_} dram_bytes_per_launch=7\n")
    monkeypatch.setattr(bench, "TRAFFIC_GLOB", str(tmp_path / "dram_traffic_*.txt"))
    assert bench.load_traffic("attention", "s", 128)[0] == 5.0
    assert bench.load_traffic("attention", "l", 512)[0] == 7.0
    assert bench.load_traffic("attention", "l", 128)[0] is None


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` times the oracle on the host cores (no GPU) and
    prints one JSON line with the native arm's metric, unit and workload label."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"],
                         cwd=root, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["higher_is_better"] is True and line["value"] > 0
    assert line["config"]["workload"] == "b256_T128_packed"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
