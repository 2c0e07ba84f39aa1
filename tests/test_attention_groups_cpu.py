"""Attention groups for sequences of at most 128 tokens (host-side model).

The prep kernels give each sequence longer than 64 tokens an attention item of
its own and pair the sequences of at most 64 tokens in batch order (1st with
2nd, 3rd with 4th, ...), each pair sharing one 128-row item as its two 64-row
halves.  The device code ranks the sequences with warp ballots, 32 per step.
This file checks that formulation, restated lane by lane in Python, against the
plain definition on many batches; the device result itself is compared with the
same definition on the GPU (tests/test_gpu_kernels.py).
"""
import numpy as np
import pytest

HALF = 64


def pair_groups(starts, lengths, half=HALF):
    """Plain definition: (start, length, partner start, partner length) -- the
    pairs of short sequences first, then the longer sequences in batch order,
    then an unpaired last short sequence."""
    short = [b for b, L in enumerate(lengths) if L <= half]
    long_ = [b for b, L in enumerate(lengths) if L > half]
    out = [(starts[a], lengths[a], starts[b], lengths[b]) for a, b in zip(short[0::2], short[1::2])]
    out += [(starts[b], lengths[b], 0, 0) for b in long_]
    if len(short) % 2:
        out.append((starts[short[-1]], lengths[short[-1]], 0, 0))
    return out


def ballot_groups(starts, lengths, half=HALF):
    """The warp formulation: a counting pass, then ranks from ballots."""
    n = len(lengths)
    n_short = 0
    for base in range(0, n, 32):
        n_short += sum(1 for lane in range(32) if base + lane < n and lengths[base + lane] <= half)
    n_pairs, n_long = n_short // 2, n - n_short
    n_groups = n_pairs + n_long + n_short % 2
    halves = {}
    groups = {}
    short_seen = long_seen = 0
    for base in range(0, n, 32):
        is_short = [base + l < n and lengths[base + l] <= half for l in range(32)]
        is_long = [base + l < n and not is_short[l] for l in range(32)]
        S = sum(1 << l for l in range(32) if is_short[l])
        Lg = sum(1 << l for l in range(32) if is_long[l])
        for lane in range(32):
            b = base + lane
            below = (1 << lane) - 1
            if is_short[lane]:
                k = short_seen + bin(S & below).count("1")
                if k < 2 * n_pairs:
                    halves[k] = (starts[b], lengths[b])
                else:
                    groups[n_pairs + n_long] = (starts[b], lengths[b], 0, 0)
            elif is_long[lane]:
                groups[n_pairs + long_seen + bin(Lg & below).count("1")] = (starts[b], lengths[b], 0, 0)
        short_seen += bin(S).count("1")
        long_seen += bin(Lg).count("1")
    for g in range(n_pairs):
        groups[g] = halves[2 * g] + halves[2 * g + 1]
    return [groups[g] for g in range(n_groups)]


def packed(lengths):
    return list(np.concatenate([[0], np.cumsum(lengths)[:-1]]).astype(int)), list(map(int, lengths))


def test_definition_on_a_small_example():
    s, L = packed([30, 100, 64, 65, 1, 128, 7])
    assert pair_groups(s, L) == [(0, 30, 130, 64), (259, 1, 388, 7), (30, 100, 0, 0), (194, 65, 0, 0),
                                 (260, 128, 0, 0)]
    s, L = packed([5, 6, 7])
    assert pair_groups(s, L) == [(0, 5, 5, 6), (11, 7, 0, 0)]


@pytest.mark.parametrize("n", [1, 2, 31, 32, 33, 63, 64, 65, 100, 256, 1000])
def test_ballot_formulation_matches_definition(n):
    r = np.random.default_rng(n)
    for trial in range(20):
        mode = trial % 4
        if mode == 0:
            L = r.integers(16, 129, n)          # the uniform [16, 128] batches
        elif mode == 1:
            L = r.integers(1, 65, n)            # all short
        elif mode == 2:
            L = r.integers(65, 129, n)          # none short
        else:
            L = r.choice([1, 63, 64, 65, 127, 128], n)
        s, L = packed(L)
        assert ballot_groups(s, L) == pair_groups(s, L)


def test_groups_cover_every_sequence_once():
    r = np.random.default_rng(5)
    for _ in range(50):
        s, L = packed(r.integers(1, 129, int(r.integers(1, 300))))
        g = ballot_groups(s, L)
        seen = sorted([a for a, _, _, _ in g] + [c for _, _, c, w in g if w > 0])
        assert seen == sorted(s)
        assert all(w == 0 or (l <= HALF and w <= HALF) for _, l, _, w in g)
        # every pair fills at most the item's 128 rows, each half at most 64
        assert len(g) == sum(1 for x in L if x > HALF) + (sum(1 for x in L if x <= HALF) + 1) // 2
