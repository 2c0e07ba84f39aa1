"""Single-kernel parity on the GPU, through the library's C ABI.

Each kernel runs alone on seeded inputs, over sizes that span several tiles
plus a ragged tail, and is compared with the oracle's stage functions (fp64)
on the same bf16-representable inputs.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import transformer_encoder_albert_b200 as tea

pytestmark = pytest.mark.gpu


def _bf16_t(a):
    return torch.tensor(synth.bf16_round(np.asarray(a, np.float32)), dtype=torch.float32).to("cuda").to(torch.bfloat16)


def _np(t):
    return t.float().cpu().numpy().astype(np.float64)


def _close(got, ref, rel=8e-3, what=""):
    """bf16 output: error bounded by output rounding (2^-8 relative) plus an
    accumulation term proportional to the row scale."""
    scale = np.max(np.abs(ref))
    err = np.abs(got - ref)
    bound = rel * np.abs(ref) + 2e-3 * scale
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} elements off, worst {err.max():.3e} (scale {scale:.3e})"


VARIANTS = ["single", "pair", "narrow"]


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("M,N,K", [(1, 256, 64), (300, 768, 128), (129, 2304, 768), (700, 2048, 768), (257, 512, 768)])
def test_gemm_bias(M, N, K, variant):
    r = np.random.default_rng(M + N + K)
    A, W, b = r.normal(0, 1, (M, K)), r.normal(0, 0.05, (N, K)), r.normal(0, 0.1, N)
    At, Wt = _bf16_t(A), _bf16_t(W)
    Y = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
    assert tea.test_gemm(At, Wt, torch.tensor(b, dtype=torch.float32, device="cuda"), Y, 0, variant=variant) == 0
    ref = oracle.linear(_np(At), _np(Wt), np.float32(b).astype(np.float64))
    _close(_np(Y), ref, what="bias")


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("M", [5, 200, 640])
def test_gemm_gelu(M, variant):
    r = np.random.default_rng(M)
    N, K = 2048, 768
    A, W, b = r.normal(0, 1, (M, K)), r.normal(0, 0.05, (N, K)), r.normal(0, 0.1, N)
    At, Wt = _bf16_t(A), _bf16_t(W)
    Y = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
    assert tea.test_gemm(At, Wt, torch.tensor(b, dtype=torch.float32, device="cuda"), Y, 1, variant=variant) == 0
    ref = oracle.gelu(oracle.linear(_np(At), _np(Wt), np.float32(b).astype(np.float64)))
    _close(_np(Y), ref, what="gelu")


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("M,K", [(3, 768), (130, 768), (513, 2048), (1000, 768)])
def test_gemm_residual_layer_norm(M, K, variant):
    r = np.random.default_rng(M * 7 + K)
    N = 768
    A, W, b = r.normal(0, 1, (M, K)), r.normal(0, 0.05, (N, K)), r.normal(0, 0.1, N)
    R = r.normal(0.3, 1.0, (M, N))
    g, beta = 1 + r.normal(0, 0.1, N), r.normal(0, 0.1, N)
    At, Wt, Rt = _bf16_t(A), _bf16_t(W), _bf16_t(R)
    Y = torch.empty(M, N, device="cuda", dtype=torch.bfloat16)
    f = lambda a: torch.tensor(a, dtype=torch.float32, device="cuda")
    assert tea.test_gemm(At, Wt, f(b), Y, 2, R=Rt, ln_g=f(g), ln_b=f(beta), eps=1e-12, variant=variant) == 0
    z = oracle.linear(_np(At), _np(Wt), np.float32(b).astype(np.float64)) + _np(Rt)
    ref = oracle.layer_norm(z, np.float32(g).astype(np.float64), np.float32(beta).astype(np.float64), 1e-12)
    _close(_np(Y), ref, what="ln")


@pytest.mark.parametrize("variant", VARIANTS)
def test_gemm_scatter_rows(variant):
    r = np.random.default_rng(9)
    M, N, K = 333, 512, 768
    A, W, b = r.normal(0, 1, (M, K)), r.normal(0, 0.05, (N, K)), r.normal(0, 0.1, N)
    At, Wt = _bf16_t(A), _bf16_t(W)
    dst = r.permutation(M + 50)[:M].astype(np.int32)
    dst[::7] = -1
    Y = torch.full((M + 50, N), 7.0, device="cuda", dtype=torch.bfloat16)
    assert tea.test_gemm(At, Wt, torch.tensor(b, dtype=torch.float32, device="cuda"), Y, 3,
                         row_dst=torch.tensor(dst, device="cuda"), variant=variant) == 0
    ref = oracle.linear(_np(At), _np(Wt), np.float32(b).astype(np.float64))
    got = _np(Y)
    keep = dst >= 0
    _close(got[dst[keep]], ref[keep], what="scatter")
    untouched = np.setdiff1d(np.arange(M + 50), dst[keep])
    assert np.all(got[untouched] == 7.0)


def _attention_case(lengths, fp32=False, seed=0, legacy=False, scale=1.0, qkv=None):
    r = np.random.default_rng(seed)
    n = int(sum(lengths))
    if qkv is None:
        qkv = r.normal(0, scale, (n, 3 * 768))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    if fp32:
        q_dev = torch.tensor(qkv, dtype=torch.float32, device="cuda")
        ctx = torch.empty(n, 768, device="cuda", dtype=torch.float32)
    else:
        q_dev = _bf16_t(qkv)
        ctx = torch.empty(n, 768, device="cuda", dtype=torch.bfloat16)
    assert tea.test_attention(q_dev, torch.tensor(cu, device="cuda"), max(lengths), ctx, fp32=fp32,
                              legacy=legacy) == 0
    q64 = _np(q_dev)
    got = _np(ctx)
    for s, L in enumerate(lengths):
        rows = slice(cu[s], cu[s + 1])
        x = q64[rows]
        ref = oracle.attention(x[:, :768], x[:, 768:1536], x[:, 1536:], np.ones(L, np.uint8), 12)
        if fp32:
            assert np.max(np.abs(got[rows] - ref)) <= 1e-5 * max(1.0, np.max(np.abs(ref)))
        else:
            _close(got[rows], ref, rel=2e-2, what=f"attention L={L}")


def test_attention_bf16_ragged_lengths():
    _attention_case([1, 2, 7, 16, 63, 64, 65, 100, 127, 128, 129, 200])


def test_attention_tcgen05_short_sequences():
    """max_len <= 128 runs the tcgen05 kernel: every length 1..128 class."""
    _attention_case([1, 2, 3, 15, 16, 17, 31, 32, 33, 63, 64, 65, 96, 127, 128, 40, 5], seed=7)


def test_attention_tcgen05_paired_sequences():
    """Sequences of at most 64 tokens share an item two by two (64-row halves):
    halves of 1, 31, 32, 33, 63 and 64 rows, a pair's second half shorter and
    longer than 32, longer sequences in between, an odd count (one unpaired), and
    peaked scores, so that a key leaking from one half into the other would show."""
    r = np.random.default_rng(21)
    lengths = [1, 64, 100, 64, 33, 31, 128, 32, 63, 65, 2, 40, 127, 17, 3, 50, 64]
    lengths += [int(x) for x in r.integers(1, 129, 40)]
    _attention_case(lengths, seed=22, scale=2.0)


def test_attention_tcgen05_item_table_overflow():
    """More items per CTA than its shared-memory table holds (512): 13,000 sequences
    of 1..4 tokens pair into 6,500 groups, 78,000 (group, head) items over at most
    148 CTAs, so items past the table are read from the group array in global
    memory.  Every row must be finite; a spread sample of sequences (including
    the last ones, which only the overflow path reaches) is checked against the
    oracle."""
    r = np.random.default_rng(31)
    lengths = [int(x) for x in r.integers(1, 5, 13000)]
    n = int(sum(lengths))
    qkv = r.normal(0, 1, (n, 3 * 768))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    q_dev = _bf16_t(qkv)
    ctx = torch.empty(n, 768, device="cuda", dtype=torch.bfloat16)
    assert tea.test_attention(q_dev, torch.tensor(cu, device="cuda"), max(lengths), ctx) == 0
    got = _np(ctx)
    assert np.all(np.isfinite(got))
    q64 = _np(q_dev)
    for s in list(range(0, 13000, 97)) + list(range(12950, 13000)):
        rows = slice(cu[s], cu[s + 1])
        x = q64[rows]
        ref = oracle.attention(x[:, :768], x[:, 768:1536], x[:, 1536:], np.ones(lengths[s], np.uint8), 12)
        _close(got[rows], ref, rel=2e-2, what=f"attention seq {s} L={lengths[s]}")


@pytest.mark.parametrize("case", ["uniform", "all_short", "boundary"])
def test_attention_groups_match_definition(case):
    """The device's grouping (warp ballots) equals the plain definition."""
    from test_attention_groups_cpu import pair_groups, packed
    r = np.random.default_rng({"uniform": 1, "all_short": 2, "boundary": 3}[case])
    if case == "uniform":
        L = r.integers(16, 129, 256)
    elif case == "all_short":
        L = r.integers(1, 65, 301)
    else:
        L = r.choice([1, 63, 64, 65, 127, 128], 97)
    starts, lens = packed(L)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32), device="cuda")
    got = tea.test_attention_groups(cu, int(max(lens)))
    assert got == [tuple(map(int, g)) for g in pair_groups(starts, lens)]


def test_attention_mma_sync_kernel_short_sequences():
    _attention_case([1, 16, 33, 64, 100, 128], seed=8, legacy=True)


def test_attention_bf16_long_sequences():
    """129 <= max_len <= 512 runs the tcgen05 kernel with one item per
    (sequence, 128-query block, head)."""
    _attention_case([256, 300, 511, 512], seed=1)


def test_attention_tcgen05_long_kernel_every_block_count():
    """Lengths around every key-block boundary (1 to 4 blocks of 128, ragged last
    block and last query block) and short sequences sharing the launch."""
    _attention_case([129, 1, 130, 255, 256, 257, 64, 383, 384, 385, 2, 447, 448, 449, 511, 512, 128, 200], seed=11)


def test_attention_tcgen05_long_kernel_peaked_softmax():
    """Scores with a spread of ~16 (QKV ~ N(0, 4)): most probabilities underflow
    far below the row maximum, exercising the exponentials' clamp."""
    _attention_case([500, 129, 384, 257], seed=13, scale=4.0)


def _last_key_dominates(lengths, seed):
    """Q/K/V rows in which, for every head, each query is u + noise and the
    sequence's last key is 3u (u = +-1 per dimension): its score exceeds every
    other by about 2^29 in the exponential, so every row raises its running
    maximum on its last key block."""
    r = np.random.default_rng(seed)
    n = int(sum(lengths))
    qkv = r.normal(0, 1, (n, 3 * 768))
    u = r.choice([-1.0, 1.0], 768)
    qkv[:, :768] = u + r.normal(0, 0.25, (n, 768))
    for end in np.cumsum(lengths):
        qkv[end - 1, 768:1536] = 3.0 * u
    return qkv


def test_attention_tcgen05_long_kernel_rescale_on_last_block():
    """Every row rescales O on its last key block.  With one item per slot that
    block is the slot's last, whose rescale waits for the commit that stands in
    for the next S; with several items per slot it waits for the next item's
    first S."""
    few = [200, 320, 449, 512]              # 156 items over 296 slots
    _attention_case(few, qkv=_last_key_dominates(few, 31))
    many = [512] * 30 + [300] * 10 + [129]  # 1,812 items, about six per slot
    _attention_case(many, qkv=_last_key_dominates(many, 32))


def test_attention_tcgen05_long_kernel_item_table_overflow():
    """More items per CTA than the long kernel's shared-memory table holds (512):
    3,300 sequences of 129..200 tokens give 79,200 (sequence, query block, head)
    items, about 535 per CTA over 148, so every CTA takes its last items from the
    walk over the candidates in global memory.  Every row must be finite; a spread
    sample of sequences and the last 40 (which only that walk reaches) are checked
    against the oracle."""
    r = np.random.default_rng(41)
    lengths = [int(x) for x in r.integers(129, 201, 3300)]
    n = int(sum(lengths))
    g = torch.Generator(device="cuda")
    g.manual_seed(42)
    q_dev = torch.randn(n, 3 * 768, generator=g, device="cuda").to(torch.bfloat16)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    ctx = torch.empty(n, 768, device="cuda", dtype=torch.bfloat16)
    assert tea.test_attention(q_dev, torch.tensor(cu, device="cuda"), max(lengths), ctx) == 0
    assert bool(torch.isfinite(ctx.float()).all())
    for s in list(range(0, 3300, 151)) + list(range(3260, 3300)):
        x = _np(q_dev[cu[s]:cu[s + 1]])
        ref = oracle.attention(x[:, :768], x[:, 768:1536], x[:, 1536:], np.ones(lengths[s], np.uint8), 12)
        _close(_np(ctx[cu[s]:cu[s + 1]]), ref, rel=2e-2, what=f"attention seq {s} L={lengths[s]}")


def test_attention_mma_sync_kernel_long_sequences():
    _attention_case([129, 256, 300, 512], seed=12, legacy=True)


def test_attention_fp32_ragged_lengths():
    _attention_case([1, 5, 36, 40, 129], fp32=True, seed=2)


@pytest.mark.parametrize("L", [50, 128, 300])
def test_attention_identical_keys_give_mean_of_values(L):
    r = np.random.default_rng(3)
    qkv = r.normal(0, 1, (L, 3 * 768))
    qkv[:, 768:1536] = qkv[0, 768:1536]
    q_dev = _bf16_t(qkv)
    ctx = torch.empty(L, 768, device="cuda", dtype=torch.bfloat16)
    cu = torch.tensor([0, L], dtype=torch.int32, device="cuda")
    assert tea.test_attention(q_dev, cu, L, ctx) == 0
    v = _np(q_dev)[:, 1536:]
    _close(_np(ctx), np.tile(v.mean(0), (L, 1)), rel=2e-2, what="identical keys")
