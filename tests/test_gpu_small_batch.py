"""The small-batch path: at most 128 token rows run as ONE persistent kernel
after the embedding (the layer's steps as phases separated by grid barriers).
Parity against the fp64 oracle on
every valid row, agreement with the per-layer kernels, the varlen entry, error
and timeout paths, determinism and the launch count."""
import time

import numpy as np
import pytest
import torch

import synth
import transformer_encoder_albert_b200 as tea
from parity_util import check_bf16, oracle_rows, record_parity

pytestmark = pytest.mark.gpu
A = synth.ARCH


@pytest.fixture(scope="module")
def w_bf16():
    return synth.make_weights(seed=1234, bf16=True)


def _t(a):
    return torch.as_tensor(a).to("cuda")


def _batch(lengths, T, seed):
    rng = np.random.default_rng(seed)
    B = len(lengths)
    ids = np.zeros((B, T), np.int64)
    mask = np.zeros((B, T), np.uint8)
    for b, n in enumerate(lengths):
        if n > 2:
            ids[b, 1:n - 1] = rng.integers(1, A["vocab"], size=n - 2)
        mask[b, :n] = 1
    return ids, mask, np.array(lengths, np.int64)


def _forward(w, ids, mask, small=True, **kw):
    enc = tea.Encoder(w, A, max_tokens=ids.size, **kw)
    enc.set_small_batch_kernel(small)
    out = enc.forward(_t(ids), _t(mask)).float().cpu().numpy()
    st = enc.status()
    launches = enc.last_forward_launches()
    enc.close()
    assert st == 0, tea.STATUS_NAMES.get(st, st)
    return out, launches


def _check_all(w, ids, mask, L, got, label, n_exec=None, out_dim=None):
    ref = oracle_rows(w, ids, mask, L, list(range(len(L))), n_exec=n_exec, out_dim=out_dim)
    worst_e, worst_c = 0.0, 1.0
    for b in range(len(L)):
        n = int(L[b])
        e, c = check_bf16(got[b, :n], ref[b], f"{label} seq {b} (L={n})", checkpoint=(out_dim == 0))
        worst_e, worst_c = max(worst_e, e), min(worst_c, c)
        assert np.all(got[b, n:] == 0.0), f"{label}: padding rows of seq {b} not zero"
    record_parity(label, len(L), int(L.sum()), worst_e, worst_c, "abs")


@pytest.mark.parametrize("lengths,T", [((64,), 64), ((128,), 128), ((1, 2, 31, 32), 32), ((64, 17), 64),
                                       ((1,), 1), ((3, 1, 2), 40)])
def test_small_batch_kernel_matches_oracle(w_bf16, lengths, T):
    ids, mask, L = _batch(lengths, T, seed=sum(lengths) + 7 * T)
    got, launches = _forward(w_bf16, ids, mask, small=True)
    assert launches == 4  # prep, embedding, the persistent forward, padding rows
    _check_all(w_bf16, ids, mask, L, got, f"small-batch kernel lengths {list(lengths)} T={T}")


def test_small_batch_kernel_agrees_with_per_layer_kernels(w_bf16):
    wl = synth.WORKLOADS["b1_T64_latency"]
    ids, mask, L = synth.make_batch(wl)
    small, n_small = _forward(w_bf16, ids, mask, small=True)
    layers, n_layers = _forward(w_bf16, ids, mask, small=False)
    assert n_small == 4 and n_layers == 64
    # two bf16 pipelines with different rounding points: within the output bar of each other
    assert float(np.max(np.abs(small - layers))) <= 3e-2


@pytest.mark.parametrize("n_exec", [1, 2, 3])
def test_small_batch_hidden_state_checkpoints(n_exec):
    """out_dim 0 returns LN2 of the last execution: the [T, 768] checkpoints,
    with random LayerNorm gamma/beta so that a swap of the two shows."""
    w = synth.make_weights(seed=99, bf16=True, ln_affine="random")
    ids, mask, L = _batch((40, 9, 1), 40, seed=3 + n_exec)
    got, _ = _forward(w, ids, mask, small=True, n_exec=n_exec, out_dim=0)
    _check_all(w, ids, mask, L, got, f"small-batch kernel checkpoint n_exec={n_exec}", n_exec=n_exec, out_dim=0)


def test_small_batch_varlen_entry(w_bf16):
    lengths = (40, 1, 25)
    ids, mask, L = _batch(lengths, 40, seed=11)
    enc = tea.Encoder(w_bf16, A, max_tokens=ids.size)
    enc.set_small_batch_kernel(True)
    padded = enc.forward(_t(ids), _t(mask)).float().cpu().numpy()
    packed_ids = np.concatenate([ids[b, :L[b]] for b in range(len(L))])
    cu = np.concatenate([[0], np.cumsum(L)]).astype(np.int32)
    out = enc.forward_varlen(_t(packed_ids), _t(cu), int(L.max())).float().cpu().numpy()
    assert enc.last_forward_launches() == 3  # prep, embedding, the persistent forward
    assert enc.status() == 0
    enc.close()
    for b in range(len(L)):
        np.testing.assert_array_equal(out[cu[b]:cu[b + 1]], padded[b, :L[b]])


def test_small_batch_is_deterministic_and_reusable(w_bf16):
    ids, mask, L = _batch((50, 13), 64, seed=21)
    ids2, mask2, _ = _batch((64,), 64, seed=22)
    enc = tea.Encoder(w_bf16, A, max_tokens=128)
    enc.set_small_batch_kernel(True)
    a = enc.forward(_t(ids), _t(mask)).clone()
    enc.forward(_t(ids2), _t(mask2))
    b = enc.forward(_t(ids), _t(mask))
    assert enc.status() == 0
    assert torch.equal(a, b)
    enc.close()


def test_small_batch_bad_id_leaves_output_untouched(w_bf16):
    ids, mask, L = _batch((30, 20), 32, seed=5)
    ids[1, 3] = 500
    enc = tea.Encoder(w_bf16, A, max_tokens=64)
    enc.set_small_batch_kernel(True)
    out = torch.full((2, 32, 512), 3.25, device="cuda", dtype=torch.bfloat16)
    tea.albert_forward(enc.h, _t(ids), _t(mask), out)
    assert enc.status() == 4  # ALBERT_ERR_ID
    assert torch.all(out == 3.25)
    enc.close()


def test_small_batch_expired_wait_reports_timeout(w_bf16):
    """Withheld loads inside the persistent kernel: its first operand wait runs
    out after the short limit, every CTA leaves at the next grid barrier, the
    forward reports ALBERT_ERR_TIMEOUT with `out` untouched, and the handle
    works again afterwards."""
    ids, mask, L = _batch((64,), 64, seed=9)
    enc = tea.Encoder(w_bf16, A, max_tokens=64)
    enc.set_small_batch_kernel(True)
    good = enc.forward(_t(ids), _t(mask)).clone()
    enc.set_wait_limit(200_000)
    enc.test_stall(["small_batch_forward"])
    out = torch.full((1, 64, 512), 3.25, device="cuda", dtype=torch.bfloat16)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    tea.albert_forward(enc.h, _t(ids), _t(mask), out)
    st = enc.status()
    assert st == 8, tea.STATUS_NAMES.get(st, st)
    assert time.perf_counter() - t0 < 1.0
    assert torch.all(out == 3.25)
    enc.test_stall([])
    enc.set_wait_limit(0)
    assert torch.equal(enc.forward(_t(ids), _t(mask)), good)
    assert enc.status() == 0
    enc.close()


def test_small_batch_forward_in_a_cuda_graph(w_bf16):
    """The persistent forward (a cooperative launch after a counter reset) captured
    in a CUDA graph: replays give the stream-launch result."""
    wl = synth.WORKLOADS["b1_T64_latency"]
    ids, mask, L = synth.make_batch(wl)
    ids_d, mask_d = _t(ids), _t(mask)
    enc = tea.Encoder(w_bf16, A, max_tokens=wl.B * wl.T)
    enc.set_small_batch_kernel(True)
    ref = enc.forward(ids_d, mask_d).clone()
    out = torch.empty_like(ref)
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        enc.forward(ids_d, mask_d, out)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    assert enc.status() == 0
    del g
    enc.close()
