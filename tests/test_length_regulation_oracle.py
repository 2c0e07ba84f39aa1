"""Pins of the length-regulation oracle (CPU, no GPU).

The oracle follows "How Kokoro TTS Works and Where CKE Stands", section "The time
axis is where a circuit becomes difficult", and the worked example of "Qwen3-TTS and
Kokoro: Two Routes from Text to Speech", section "Path one: Kokoro decides how long
each sound lasts".  Each pin below is fixed by the pages
or by closed forms, not by re-evaluating the oracle's own formula.
"""
import os

import numpy as np

from oracle import length_regulation as lr

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "length_regulation_worked_example.txt")


def _golden():
    vals = {}
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        k, *v = line.split()
        vals[k] = [int(x) for x in v]
    return vals


def _logits_with_ones(counts, C):
    """Rows whose sigmoid channels are 1 (logit +40) for the first counts[t] channels and
    0 (logit -40) for the rest: the channel sum is counts[t] to within 1e-16."""
    z = np.full((len(counts), C), -40.0)
    for t, k in enumerate(counts):
        z[t, :k] = 40.0
    return z


def test_worked_example_from_the_pages():
    g = _golden()
    z = _logits_with_ones(g["durations"], C=4)
    feats = np.arange(3, dtype=np.float64)[:, None] * np.ones((1, 8))  # row t holds t
    d, start, cu_frames, frames = lr.length_regulate(z, 1.0, feats, [0, 3])
    assert d.tolist() == g["durations"]
    assert int(cu_frames[-1]) == g["frames"][0]
    assert frames[:, 0].astype(int).tolist() == g["aligned_tokens"]
    assert start.tolist() == [0, 2, 3]


def test_durations_clamp_to_one_frame():
    z = np.full((5, 50), -40.0)  # sigmoid sum ~ 0 -> rounds to 0 -> clamped
    assert lr.durations(z, 1.0).tolist() == [1] * 5


def test_zero_logits_are_one_half_each():
    # sigmoid(0) = 1/2 exactly: six channels sum to 3
    assert lr.durations(np.zeros((2, 6)), 1.0).tolist() == [3, 3]


def test_speed_divides_and_ties_round_to_even():
    z = _logits_with_ones([5, 3, 7, 4, 2], C=8)
    # sums 5, 3, 7, 4, 2 over speed 2: 2.5 -> 2, 1.5 -> 2, 3.5 -> 4, 2 -> 2, 1 -> 1
    assert lr.durations(z, 2.0).tolist() == [2, 2, 4, 2, 1]
    # over speed 0.5: doubled exactly
    assert lr.durations(z, 0.5).tolist() == [10, 6, 14, 8, 4]


def test_expansion_equals_numpy_repeat_and_frame_count_is_the_sum():
    r = np.random.default_rng(5)
    lens = [7, 1, 30, 12]
    cu = np.concatenate([[0], np.cumsum(lens)])
    n = int(cu[-1])
    z = r.normal(-2.9, 1.0, (n, 50))
    feats = r.normal(0, 1, (n, 16))
    d, start, cu_frames, frames = lr.length_regulate(z, 1.0, feats, cu)
    assert np.array_equal(frames, np.repeat(feats, d, axis=0))
    assert int(cu_frames[-1]) == int(d.sum()) == frames.shape[0]
    for b in range(len(lens)):
        assert cu_frames[b + 1] - cu_frames[b] == d[cu[b]:cu[b + 1]].sum()
    assert np.all(d >= 1)


def test_durations_do_not_increase_with_speed():
    r = np.random.default_rng(6)
    z = r.normal(-2.0, 1.5, (40, 50))
    d1, d2, d4 = (lr.durations(z, s) for s in (1.0, 2.0, 4.0))
    assert np.all(d1 >= d2) and np.all(d2 >= d4)
