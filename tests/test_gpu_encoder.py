"""Whole-encoder parity on the GPU, through the C ABI, against the fp64 oracle.

Every workload of the suite runs at its full size on the GPU, packed and
padded, and every valid row of every sequence is compared with the oracle
(which computes each sequence alone, unpadded; its results are shared by the
packed and padded runs of a workload).  Padding rows must be exactly zero.
Error paths must leave the output byte-identical to its sentinel fill.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import synth
import transformer_encoder_albert_b200 as tea
from parity_util import check_bf16, check_fp32, oracle_rows, record_parity

pytestmark = pytest.mark.gpu
A = synth.ARCH

# oracle outputs of whole workloads (bf16 weights, default architecture), by name
_ORACLE = {}


def _oracle_all(weights, wl, ids, mask, L):
    if wl.name not in _ORACLE:
        _ORACLE[wl.name] = oracle_rows(weights, ids, mask, L, list(range(len(L))))
    return _ORACLE[wl.name]


@pytest.fixture(scope="module")
def w_bf16():
    return synth.make_weights(seed=1234, bf16=True)


@pytest.fixture(scope="module")
def w_fp32():
    return synth.make_weights(seed=1234, bf16=False)


def _t(a, dtype=None):
    return torch.as_tensor(a).to("cuda") if dtype is None else torch.as_tensor(a).to("cuda", dtype)


def _run(weights, wl, dtype="bf16", pack=True, n_exec=None, out_dim=None, max_tokens=None):
    ids, mask, L = synth.make_batch(wl)
    enc = tea.Encoder(weights, A, dtype=dtype, max_tokens=max_tokens or wl.B * wl.T, pack=pack,
                      n_exec=n_exec, out_dim=wl.out_dim if out_dim is None else out_dim)
    out = enc.forward(_t(ids), _t(mask))
    st = enc.status()
    enc.close()
    assert st == 0, tea.STATUS_NAMES[st]
    return ids, mask, L, out.float().cpu().numpy()


def _compare(weights, wl, got, ids, mask, L, seqs, fp32=False, n_exec=None, out_dim=None, ref=None, label=None):
    od = wl.out_dim if out_dim is None else out_dim
    if ref is None:
        ref = oracle_rows(weights, ids, mask, L, seqs, n_exec=n_exec, out_dim=od)
    worst_err, worst_cos = 0.0, 1.0
    for b in seqs:
        n = int(L[b])
        if fp32:
            worst_err = max(worst_err, check_fp32(got[b, :n], ref[b], f"{wl.name} seq {b}"))
        else:
            # out_dim == 0 returns hidden states: a checkpoint, not the encoder output
            e, c = check_bf16(got[b, :n], ref[b], f"{wl.name} seq {b} (L={n})", checkpoint=(od == 0))
            worst_err, worst_cos = max(worst_err, e), min(worst_cos, c)
    for b in range(len(L)):
        assert np.all(got[b, int(L[b]):] == 0.0), f"padding rows of seq {b} not zero"
    record_parity(label or wl.name, len(seqs), int(sum(int(L[b]) for b in seqs)), worst_err,
                  None if fp32 else worst_cos, "rel" if fp32 else "abs")


def test_tiny_fp32_T36(w_fp32):
    wl = synth.WORKLOADS["tiny_fp32_T36"]
    ids, mask, L, got = _run(w_fp32, wl, dtype="fp32")
    _compare(w_fp32, wl, got, ids, mask, L, [0], fp32=True)


@pytest.mark.parametrize("name", ["b8_T128", "b64_T128_normal", "b32_T512_long", "b256_T128", "b1_T64_latency"])
@pytest.mark.parametrize("pack", [True, False])
def test_workload_every_sequence(w_bf16, name, pack):
    """A whole bf16 workload, packed by length or on all B*T padded rows: every
    valid row of every sequence against the oracle."""
    wl = synth.WORKLOADS[name]
    ids, mask, L, got = _run(w_bf16, wl, pack=pack)
    ref = _oracle_all(w_bf16, wl, ids, mask, L)
    _compare(w_bf16, wl, got, ids, mask, L, list(range(wl.B)), ref=ref,
             label=f"{name} {'packed' if pack else 'padded'}")


@pytest.mark.parametrize("lengths,T", [((1, 2, 3, 127, 128, 129), 129), ((1, 2, 3, 64, 127, 128), 128),
                                       ((1,), 1), ((2, 1), 2)])
@pytest.mark.parametrize("pack", [True, False])
def test_edge_lengths_in_one_batch(w_bf16, lengths, T, pack):
    """Sequences of 1, 2 and 3 tokens beside ones at and around a 128-row tile
    (and the 128-token attention boundary) in one batch; single-token batches."""
    B = len(lengths)
    rng = np.random.default_rng(sum(lengths) + T)
    L = np.array(lengths, np.int64)
    ids = np.zeros((B, T), np.int64)
    mask = np.zeros((B, T), np.uint8)
    for b, n in enumerate(lengths):
        if n > 2:
            ids[b, 1:n - 1] = rng.integers(1, A["vocab"], size=n - 2)
        mask[b, :n] = 1
    enc = tea.Encoder(w_bf16, A, max_tokens=B * T, pack=pack)
    got = enc.forward(_t(ids), _t(mask)).float().cpu().numpy()
    assert enc.status() == 0
    enc.close()
    wl = synth.Workload(f"edge_T{T}", B, T, "full")
    _compare(w_bf16, wl, got, ids, mask, L, list(range(B)),
             label=f"lengths {list(lengths)} T={T} {'packed' if pack else 'padded'}")


@pytest.mark.parametrize("n_exec", [0, 1, 2])
def test_stage_checkpoints_hidden_states(w_bf16, n_exec):
    """Connected checkpoints: the [T, 768] states after the embedding + input
    projection (n_exec=0) and after one and two shared-layer executions."""
    wl = synth.Workload("stages", 4, 96, "uniform", lo=5, hi=96, seed=77)
    ids, mask, L, got = _run(w_bf16, wl, n_exec=n_exec, out_dim=0)
    _compare(w_bf16, wl, got, ids, mask, L, list(range(wl.B)), n_exec=n_exec, out_dim=0)


def test_random_layer_norm_affine_catches_swaps():
    w = synth.make_weights(seed=99, bf16=True, ln_affine="random")
    wl = synth.Workload("affine", 3, 64, "uniform", lo=10, hi=64, seed=78)
    ids, mask, L, got = _run(w, wl, n_exec=3)
    _compare(w, wl, got, ids, mask, L, list(range(wl.B)), n_exec=3)


@pytest.mark.parametrize("n_groups,n_exec", [(2, 12), (3, 12), (12, 12), (2, 5)])
def test_grouped_sharing_matches_oracle(n_groups, n_exec):
    """n_groups weight sets over n_exec executions (consecutive blocks per set):
    every sequence of a ragged batch against the grouped oracle."""
    w = synth.make_weights(seed=41 + n_groups, bf16=True, ln_affine="random", n_groups=n_groups)
    wl = synth.Workload("grouped", 6, 96, "uniform", lo=5, hi=96, seed=80 + n_groups)
    ids, mask, L = synth.make_batch(wl)
    enc = tea.Encoder(w, A, max_tokens=wl.B * wl.T, n_exec=n_exec, n_groups=n_groups)
    got = enc.forward(_t(ids), _t(mask)).float().cpu().numpy()
    assert enc.status() == 0
    enc.close()
    for b in range(wl.B):
        n = int(L[b])
        ref = oracle.encode_grouped(w, A, ids[b, :n], mask[b, :n], n_groups, n_exec=n_exec)
        check_bf16(got[b, :n], ref, f"grouped G={n_groups} seq {b} (L={n})")
        assert np.all(got[b, n:] == 0.0)


def test_grouped_sharing_fp32(w_fp32):
    w = synth.make_weights(seed=47, bf16=False, ln_affine="random", n_groups=3)
    wl = synth.Workload("grouped32", 2, 30, "uniform", lo=4, hi=30, seed=90, dtype="fp32")
    ids, mask, L = synth.make_batch(wl)
    enc = tea.Encoder(w, A, dtype="fp32", max_tokens=wl.B * wl.T, n_exec=6, n_groups=3)
    got = enc.forward(_t(ids), _t(mask)).float().cpu().numpy()
    assert enc.status() == 0
    enc.close()
    for b in range(wl.B):
        n = int(L[b])
        ref = oracle.encode_grouped(w, A, ids[b, :n], mask[b, :n], 3, n_exec=6)
        check_fp32(got[b, :n], ref, f"grouped fp32 seq {b}")


def test_grouped_sharing_rejects_more_groups_than_executions():
    w = synth.make_weights(seed=48, bf16=True, n_groups=4)
    with pytest.raises(tea.AlbertError):
        tea.Encoder(w, A, max_tokens=64, n_exec=3, n_groups=4)


@pytest.mark.parametrize("dtype,out_dim", [("bf16", 512), ("bf16", 0), ("fp32", 512)])
def test_transposed_output_layout(w_bf16, w_fp32, dtype, out_dim):
    """out_layout 1 returns [B, D, T]: the token-major output transposed per
    sequence (same arithmetic, so bit-equal), zeros at padding positions."""
    w = w_bf16 if dtype == "bf16" else w_fp32
    wl = synth.WORKLOADS["b8_T128"] if dtype == "bf16" else synth.Workload("t32", 3, 40, "uniform", lo=3, hi=40, seed=91)
    ids, mask, L = synth.make_batch(wl)
    n_exec = None if dtype == "bf16" else 2
    a = tea.Encoder(w, A, dtype=dtype, max_tokens=wl.B * wl.T, n_exec=n_exec, out_dim=out_dim)
    b = tea.Encoder(w, A, dtype=dtype, max_tokens=wl.B * wl.T, n_exec=n_exec, out_dim=out_dim, out_layout=1)
    tok = a.forward(_t(ids), _t(mask)).cpu()
    tr = b.forward(_t(ids), _t(mask)).cpu()
    assert a.status() == 0 and b.status() == 0
    D = out_dim or 768
    assert tuple(tr.shape) == (wl.B, D, wl.T)
    assert torch.equal(tr, tok.transpose(1, 2))
    # against the oracle on two sequences
    ref = oracle_rows(w, ids, mask, L, [0, 1], n_exec=n_exec, out_dim=out_dim)
    for s in (0, 1):
        n = int(L[s])
        got = tr[s, :, :n].float().numpy().T
        if dtype == "fp32":
            check_fp32(got, ref[s], f"transposed seq {s}")
        else:
            check_bf16(got, ref[s], f"transposed seq {s}", checkpoint=(out_dim == 0))
    # the host path fills the same [B, D, T] buffer
    if dtype == "bf16" and out_dim == 512:
        out_h = torch.empty(wl.B, D, wl.T, dtype=torch.bfloat16).pin_memory()
        assert b.forward_host(torch.as_tensor(ids).pin_memory(), torch.as_tensor(mask).pin_memory(), out_h) == 0
        assert torch.equal(out_h, tr)
    # packed rows have no per-sequence [D, T] form
    cu = torch.tensor(np.concatenate([[0], np.cumsum(L)]).astype(np.int32), device="cuda")
    packed = _t(np.concatenate([ids[s, :L[s]] for s in range(wl.B)]))
    with pytest.raises(tea.AlbertError):
        b.forward_varlen(packed, cu, int(L.max()))
    a.close()
    b.close()


def test_fp32_small_padded_batch(w_fp32):
    wl = synth.Workload("fp32b", 3, 40, "uniform", lo=2, hi=40, seed=79, dtype="fp32", out_dim=512)
    ids, mask, L, got = _run(w_fp32, wl, dtype="fp32", n_exec=3)
    _compare(w_fp32, wl, got, ids, mask, L, list(range(wl.B)), fp32=True, n_exec=3)


def test_varlen_equals_padded_api(w_bf16):
    wl = synth.WORKLOADS["b64_T128_normal"]
    ids, mask, L = synth.make_batch(wl)
    enc = tea.Encoder(w_bf16, A, max_tokens=wl.B * wl.T)
    padded = enc.forward(_t(ids), _t(mask)).float().cpu().numpy()
    packed_ids = np.concatenate([ids[b, :L[b]] for b in range(wl.B)])
    cu = np.concatenate([[0], np.cumsum(L)]).astype(np.int32)
    out = enc.forward_varlen(_t(packed_ids), _t(cu), int(L.max())).float().cpu().numpy()
    assert enc.status() == 0
    enc.close()
    for b in range(wl.B):
        np.testing.assert_array_equal(out[cu[b]:cu[b + 1]], padded[b, :L[b]])


def test_repeat_calls_are_deterministic_and_stateless(w_bf16):
    """A second request with another shape does not change the first one's result."""
    wl1, wl2 = synth.WORKLOADS["b8_T128"], synth.WORKLOADS["b1_T64_latency"]
    enc = tea.Encoder(w_bf16, A, max_tokens=4096)
    i1, m1, _ = synth.make_batch(wl1)
    i2, m2, _ = synth.make_batch(wl2)
    a = enc.forward(_t(i1), _t(m1)).clone()
    enc.forward(_t(i2), _t(m2))
    b = enc.forward(_t(i1), _t(m1))
    assert enc.status() == 0
    assert torch.equal(a, b)
    enc.close()


def test_expired_wait_reports_timeout_and_leaves_output_untouched(w_bf16):
    """The failure path of the kernels' bounded waits, without faulting the GPU:
    a GEMM whose producer withholds its operand loads can never see its first
    tile, so its wait runs out after the handle's short limit.  The forward
    reports ALBERT_ERR_TIMEOUT, no later kernel writes `out`, the call returns
    well before the default 2 s limit could have expired, and the next forward
    on the same handle and context is correct again."""
    wl = synth.WORKLOADS["b8_T128"]
    ids, mask, L = synth.make_batch(wl)
    enc = tea.Encoder(w_bf16, A, max_tokens=wl.B * wl.T)
    good = enc.forward(_t(ids), _t(mask)).clone()
    assert enc.status() == 0
    enc.set_wait_limit(200_000)  # 200 us
    for cls in ("embed_proj", "gemm_qkv", "gemm_ffn_down_ln", "gemm_final_proj"):
        enc.test_stall([cls])
        out = _sentinel(ids.shape)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        tea.albert_forward(enc.h, _t(ids), _t(mask), out)
        st = enc.status()
        elapsed = time.perf_counter() - t0
        assert st == 8, f"{cls}: status {tea.STATUS_NAMES.get(st, st)}"  # ALBERT_ERR_TIMEOUT
        assert elapsed < 1.0, f"{cls}: {elapsed:.2f} s, the short limit did not apply"
        assert torch.all(out == 3.25), f"{cls}: output written"
    enc.test_stall([])
    enc.set_wait_limit(0)
    assert torch.equal(enc.forward(_t(ids), _t(mask)), good)
    assert enc.status() == 0
    enc.close()


def test_forward_host_buffers_match_device_path(w_bf16):
    wl = synth.WORKLOADS["b8_T128"]
    ids, mask, L = synth.make_batch(wl)
    enc = tea.Encoder(w_bf16, A, max_tokens=wl.B * wl.T)
    dev = enc.forward(_t(ids), _t(mask)).cpu()
    ids_h = torch.as_tensor(ids).pin_memory()
    mask_h = torch.as_tensor(mask).pin_memory()
    out_h = torch.empty(wl.B, wl.T, 512, dtype=torch.bfloat16).pin_memory()
    assert enc.forward_host(ids_h, mask_h, out_h) == 0
    assert torch.equal(dev, out_h)
    enc.close()


def test_forward_host_async_pipeline_matches_device_path(w_bf16):
    """Five batches of different lengths through the pipelined host path (two in
    flight, output copies overlapping the next forward) equal the device path."""
    wl = synth.WORKLOADS["b8_T128"]
    enc = tea.Encoder(w_bf16, A, max_tokens=wl.B * wl.T)
    batches, outs, refs = [], [], []
    for k in range(5):
        ids, mask, L = synth.make_batch(wl, seed=100 + k)
        refs.append(enc.forward(_t(ids), _t(mask)).cpu())
        batches.append((torch.as_tensor(ids).pin_memory(), torch.as_tensor(mask).pin_memory()))
        outs.append(torch.full((wl.B, wl.T, 512), 7.0, dtype=torch.bfloat16).pin_memory())
    for k in range(5):
        assert enc.forward_host_async(batches[k][0], batches[k][1], outs[k]) == 0
    assert enc.forward_host_wait() == 0
    for k in range(5):
        assert torch.equal(refs[k], outs[k]), f"batch {k}"
    enc.close()


def test_forward_host_async_reports_a_bad_batch_when_reaped(w_bf16):
    wl = synth.WORKLOADS["b8_T128"]
    enc = tea.Encoder(w_bf16, A, max_tokens=wl.B * wl.T)
    ids, mask, L = synth.make_batch(wl)
    ref = enc.forward(_t(ids), _t(mask)).cpu()
    bad = ids.copy()
    bad[2, int(L[2]) // 2] = 178
    # host buffers stay referenced until forward_host_wait (the copies are asynchronous)
    ids_h = [torch.as_tensor(a).pin_memory() for a in (ids, bad, ids, ids)]
    mask_h = torch.as_tensor(mask).pin_memory()
    outs = [torch.zeros(wl.B, wl.T, 512, dtype=torch.bfloat16).pin_memory() for _ in range(4)]
    rcs = [enc.forward_host_async(ids_h[k], mask_h, outs[k]) for k in range(4)]
    # call k returns the status of batch k - 2: the bad batch 1 surfaces at call 3
    assert rcs == [0, 0, 0, 4]
    assert enc.forward_host_wait() == 0
    for k in (0, 2, 3):
        assert torch.equal(ref, outs[k]), f"batch {k}"
    enc.close()


def test_forward_varlen_host_async_matches_device_path(w_bf16):
    """Packed batches through the pipelined host path (only valid rows cross the
    bus), interleaved with padded ones on the same staging slots, equal the device
    path's rows; host-side shape checks reject a bad cu_seqlens before any work."""
    wl = synth.WORKLOADS["b8_T128"]
    enc = tea.Encoder(w_bf16, A, max_tokens=wl.B * wl.T)
    keep, refs, outs = [], [], []
    for k in range(4):
        ids, mask, L = synth.make_batch(wl, seed=200 + k)
        ref = enc.forward(_t(ids), _t(mask)).cpu()
        if k % 2:  # a padded batch between packed ones
            ids_h, mask_h = torch.as_tensor(ids).pin_memory(), torch.as_tensor(mask).pin_memory()
            out_h = torch.zeros(wl.B, wl.T, 512, dtype=torch.bfloat16).pin_memory()
            assert enc.forward_host_async(ids_h, mask_h, out_h) == 0
            keep.append((ids_h, mask_h))
            refs.append(ref)
        else:
            packed = np.concatenate([ids[b, :L[b]] for b in range(wl.B)])
            cu = np.concatenate([[0], np.cumsum(L)]).astype(np.int32)
            ids_h, cu_h = torch.as_tensor(packed).pin_memory(), torch.as_tensor(cu).pin_memory()
            out_h = torch.full((int(cu[-1]), 512), 7.0, dtype=torch.bfloat16).pin_memory()
            assert enc.forward_varlen_host_async(ids_h, cu_h, int(L.max()), out_h) == 0
            keep.append((ids_h, cu_h))
            refs.append(torch.cat([ref[b, :L[b]] for b in range(wl.B)]))
        outs.append(out_h)
    assert enc.forward_host_wait() == 0
    for k in range(4):
        assert torch.equal(refs[k], outs[k]), f"batch {k}"
    bad_cu = torch.tensor([1, 5], dtype=torch.int32)
    assert enc.forward_varlen_host_async(torch.zeros(5, dtype=torch.int64), bad_cu, 5,
                                         torch.zeros(5, 512, dtype=torch.bfloat16)) == 3  # ALBERT_ERR_SHAPE
    big_cu = torch.tensor([0, wl.B * wl.T + 1], dtype=torch.int32)
    assert enc.forward_varlen_host_async(torch.zeros(1, dtype=torch.int64), big_cu, 128,
                                         torch.zeros(1, 512, dtype=torch.bfloat16)) == 3
    enc.close()


# ------------------------------------------------------------ error paths ----

def _sentinel(shape):
    return torch.full((*shape, 512), 3.25, device="cuda", dtype=torch.bfloat16)


def test_invalid_id_leaves_output_untouched(w_bf16):
    wl = synth.WORKLOADS["b8_T128"]
    ids, mask, L = synth.make_batch(wl)
    enc = tea.Encoder(w_bf16, A, max_tokens=wl.B * wl.T)
    good = enc.forward(_t(ids), _t(mask)).clone()
    for bad in (178, -1, 10**12):
        ids_bad = ids.copy()
        ids_bad[3, int(L[3]) // 2] = bad
        out = _sentinel(ids.shape)
        tea.albert_forward(enc.h, _t(ids_bad), _t(mask), out)
        assert enc.status() == 4  # ALBERT_ERR_ID
        assert torch.all(out == 3.25)
    # an invalid id in a padding slot is ignored
    ids_pad = ids.copy()
    ids_pad[0, -1] = 999 if L[0] < wl.T else 0
    out = enc.forward(_t(ids_pad), _t(mask))
    assert enc.status() == 0
    if L[0] < wl.T:
        assert torch.equal(out[0], good[0])
    # and the next valid call reproduces the earlier result
    assert torch.equal(enc.forward(_t(ids), _t(mask)), good)
    enc.close()


def test_invalid_id_small_batch_path(w_bf16):
    """The same rejection on the small-batch path (standalone embedding kernel in
    front of the persistent forward) as on the fused embedding + projection kernel
    above."""
    wl = synth.WORKLOADS["b1_T64_latency"]
    ids, mask, L = synth.make_batch(wl)
    enc = tea.Encoder(w_bf16, A, max_tokens=wl.B * wl.T)
    enc.set_small_batch_kernel(True)
    good = enc.forward(_t(ids), _t(mask)).clone()
    ids_bad = ids.copy()
    ids_bad[0, int(L[0]) // 2] = 178
    out = _sentinel(ids.shape)
    tea.albert_forward(enc.h, _t(ids_bad), _t(mask), out)
    assert enc.status() == 4  # ALBERT_ERR_ID
    assert torch.all(out == 3.25)
    assert torch.equal(enc.forward(_t(ids), _t(mask)), good)
    enc.close()


def test_bad_masks_are_rejected(w_bf16):
    wl = synth.WORKLOADS["b8_T128"]
    ids, mask, L = synth.make_batch(wl)
    enc = tea.Encoder(w_bf16, A, max_tokens=wl.B * wl.T)
    holes = mask.copy()
    holes[2, 1] = 0  # not a prefix
    empty = mask.copy()
    empty[5, :] = 0  # empty sequence
    late = mask.copy()
    late[1, -1] = 1 if L[1] < wl.T - 1 else late[1, -1]
    cases = [holes, empty] + ([late] if L[1] < wl.T - 1 else [])
    for m in cases:
        out = _sentinel(ids.shape)
        tea.albert_forward(enc.h, _t(ids), _t(m), out)
        assert enc.status() == 5  # ALBERT_ERR_MASK
        assert torch.all(out == 3.25)
    enc.close()


def test_host_shape_errors(w_bf16):
    enc = tea.Encoder(w_bf16, A, max_tokens=1000)
    ids = torch.zeros(2, 513, dtype=torch.int64, device="cuda")
    mask = torch.ones(2, 513, dtype=torch.uint8, device="cuda")
    out = _sentinel((2, 513))
    with pytest.raises(tea.AlbertError) as e:
        tea.albert_forward(enc.h, ids, mask, out)
    assert e.value.code == 3
    ids = torch.zeros(8, 128, dtype=torch.int64, device="cuda")  # 1024 > 1000 rows
    with pytest.raises(tea.AlbertError) as e:
        tea.albert_forward(enc.h, ids, torch.ones_like(ids, dtype=torch.uint8), _sentinel((8, 128)))
    assert e.value.code == 3
    enc.close()


def test_varlen_rejections(w_bf16):
    enc = tea.Encoder(w_bf16, A, max_tokens=300)
    ids = torch.zeros(400, dtype=torch.int64, device="cuda")
    out = torch.full((400, 512), 3.25, device="cuda", dtype=torch.bfloat16)
    for cu, code in (([0, 10, 10, 20], 6), ([1, 10, 20], 6), ([0, 128, 256, 384], 3), ([0, 100, 250], 6)):
        tea.albert_forward_varlen(enc.h, ids, _t(np.array(cu, np.int32)), 128, out)
        assert enc.status() == code, cu
        assert torch.all(out == 3.25)
    enc.close()
