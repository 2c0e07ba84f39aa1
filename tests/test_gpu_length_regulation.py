"""Length regulation on the GPU (albert_length_regulate) against the fp64 oracle.

Durations, frame starts and frame offsets are integers: bit-exact.  Frames are
copies of bf16 feature rows: bit-exact.  Covers the pages' worked example,
ragged batches, several speeds, the bench-size batch (sampled frames), and the
capacity / sequence-offset errors.
"""
import numpy as np
import pytest
import torch

import synth
import transformer_encoder_albert_b200 as tea
from oracle import length_regulation as lr

pytestmark = pytest.mark.gpu


def _run(z, feats, cu, speed=1.0, max_frames=None):
    zt = torch.tensor(z, dtype=torch.float32, device="cuda")
    ft = torch.tensor(feats, dtype=torch.float32, device="cuda").to(torch.bfloat16)
    ct = torch.tensor(np.asarray(cu), dtype=torch.int32, device="cuda")
    return tea.length_regulate(zt, ft, ct, speed=speed, max_frames=max_frames)


def _check(z, feats, cu, speed):
    st, d, start, cuf, frames = _run(z, feats, cu, speed)
    assert st == 0
    rd, rstart, rcuf, _ = lr.length_regulate(z, speed, feats, cu)
    assert np.array_equal(d.cpu().numpy(), rd)
    assert np.array_equal(start.cpu().numpy(), rstart)
    assert np.array_equal(cuf.cpu().numpy(), rcuf)
    A = int(rcuf[-1])
    got = frames[:A].float().cpu().numpy()
    assert np.array_equal(got, np.repeat(feats.astype(np.float32), rd, axis=0))
    return rd


def test_worked_example_from_the_pages():
    z = np.full((3, 4), -40.0, np.float32)
    z[0, :2] = z[1, :1] = z[2, :3] = 40.0
    feats = np.repeat(np.arange(3, dtype=np.float32)[:, None], 512, axis=1)
    st, d, start, cuf, frames = _run(z, feats, [0, 3])
    assert st == 0
    assert d.tolist() == [2, 1, 3] and cuf.tolist() == [0, 6]
    assert frames[:6, 0].float().tolist() == [0, 0, 1, 2, 2, 2]


@pytest.mark.parametrize("speed", [1.0, 0.7, 2.0])
def test_ragged_batch_matches_oracle(speed):
    rng = np.random.default_rng(11)
    lens = rng.integers(1, 130, size=37)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    n = int(cu[-1])
    z = synth.make_duration_logits(n, seed=3)
    feats = synth.make_features(n, 512, seed=4)
    d = _check(z, feats, cu, speed)
    assert d.min() >= 1


def test_width_768_and_single_token():
    z = synth.make_duration_logits(1, channels=7, seed=5)
    feats = synth.make_features(1, 768, seed=6)
    _check(z, feats, [0, 1], 1.0)


def test_bench_size_batch_sampled():
    """The b256_T128 batch (18,797 tokens, 50 channels): durations and offsets exact
    everywhere, frames compared on sampled tokens."""
    wl = synth.WORKLOADS["b256_T128"]
    _, _, L = synth.make_batch(wl)
    cu = np.concatenate([[0], np.cumsum(L)]).astype(np.int32)
    n = int(cu[-1])
    z = synth.make_duration_logits(n)
    feats = synth.make_features(n, 512)
    st, d, start, cuf, frames = _run(z, feats, cu)
    assert st == 0
    rd = lr.durations(z, 1.0)
    rstart, rcuf = lr.frame_offsets(rd, cu)
    assert np.array_equal(d.cpu().numpy(), rd)
    assert np.array_equal(start.cpu().numpy(), rstart) and np.array_equal(cuf.cpu().numpy(), rcuf)
    rng = np.random.default_rng(0)
    fr = frames.float()
    for t in rng.choice(n, 64, replace=False).tolist() + [0, n - 1]:
        rows = fr[int(rstart[t]):int(rstart[t]) + int(rd[t])].cpu().numpy()
        assert np.array_equal(rows, np.repeat(feats[t:t + 1], int(rd[t]), axis=0))


def test_capacity_error_leaves_frames_untouched():
    z = synth.make_duration_logits(20, seed=9)
    feats = synth.make_features(20, 512, seed=10)
    A = int(lr.durations(z, 1.0).sum())
    zt = torch.tensor(z, device="cuda")
    ft = torch.tensor(feats, device="cuda").to(torch.bfloat16)
    ct = torch.tensor([0, 20], dtype=torch.int32, device="cuda")
    st, _, _, _, _ = tea.length_regulate(zt, ft, ct, max_frames=A)
    assert st == 0
    # one frame short: ALBERT_ERR_SHAPE, nothing written
    frames = torch.full((A - 1, 512), 5.0, dtype=torch.bfloat16, device="cuda")
    dur = torch.empty(20, dtype=torch.int32, device="cuda")
    start = torch.empty(20, dtype=torch.int32, device="cuda")
    cuf = torch.empty(2, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    scratch = torch.empty(int(tea.lib().albert_length_regulate_scratch_bytes(20)), dtype=torch.uint8, device="cuda")
    P = tea._ptr
    rc = tea.lib().albert_length_regulate(P(zt), 50, 1.0, P(ft), 512, P(ct), 1, 20, P(dur), P(start), P(cuf),
                                          P(frames), A - 1, P(scratch), P(status), tea._stream_ptr())
    torch.cuda.synchronize()
    assert rc == 0 and int(status.item()) == 3
    assert torch.all(frames == 5.0)


def test_bad_offsets_and_host_rejections():
    z = synth.make_duration_logits(10, seed=12)
    feats = synth.make_features(10, 512, seed=13)
    st, *_ = _run(z, feats, [0, 6, 4, 10])  # not monotone
    assert st == 6  # ALBERT_ERR_SEQLENS
    st, *_ = _run(z, feats, [0, 6, 9])  # does not end at n_tok
    assert st == 6
    st, *_ = _run(z, feats, [0, 10], speed=0.0)
    assert st == 2  # ALBERT_ERR_CONFIG: speed must be positive
