"""TEST INFRASTRUCTURE -- fp64 CPU oracle of length regulation, the step after the
encoder on Kokoro's path.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's ``cpu_baseline`` /
``--impl reference`` legs may import this module.  It shares no code with the
CUDA library.

What it computes (sources, by page and section):
  * "How Kokoro TTS Works and Where CKE Stands", section "The time axis is where
    a circuit becomes difficult": per token, the sigmoid duration channels are
    summed, divided by the speed, rounded and clamped to at least one frame;
    A = sum_t d[t] is the number of aligned frames; token features are repeated
    according to the duration vector.
  * "Qwen3-TTS and Kokoro: Two Routes from Text to Speech", section "Path one:
    Kokoro decides how long each sound lasts": the worked example (durations
    2, 1, 3 -> six positions p1 p1 p2 p3 p3 p3) that pins the expansion order.

Readings where the pages are silent: "rounded" is round-half-to-even (IEEE
rint); the number of duration channels C is a parameter; the decision is taken
in fp64 (sigmoid, sum over channels in ascending order, then the division).
Sequences are packed back to back (token rows in cu_seqlens order) and so are
their frames.
"""
from __future__ import annotations

import numpy as np


def durations(logits, speed: float) -> np.ndarray:
    """d[t] = max(1, rint(sum_c sigmoid(logits[t, c]) / speed)), int64, in fp64."""
    z = np.asarray(logits, dtype=np.float64)
    assert z.ndim == 2 and speed > 0
    d = np.empty(z.shape[0], dtype=np.int64)
    for t in range(z.shape[0]):
        s = 0.0
        for c in range(z.shape[1]):  # ascending channel order
            x = -z[t, c]
            s += 0.0 if x > 709.0 else 1.0 / (1.0 + np.exp(x))
        d[t] = max(1, int(np.rint(s / float(speed))))
    return d


def frame_offsets(d, cu_seqlens) -> tuple[np.ndarray, np.ndarray]:
    """Frame start of every token and the frame offsets of every sequence.

    Frames of the packed batch are numbered sequence after sequence, token after
    token: token t starts at sum_{t' < t} d[t']; sequence b owns frames
    cu_frames[b] .. cu_frames[b+1]-1, so A_b = cu_frames[b+1] - cu_frames[b]."""
    d = np.asarray(d, dtype=np.int64)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    start = np.zeros(d.shape[0], dtype=np.int64)
    run = 0
    for t in range(d.shape[0]):
        start[t] = run
        run += int(d[t])
    cu_frames = np.array([start[c] if c < d.shape[0] else run for c in cu], dtype=np.int64)
    return start, cu_frames


def expand(feats, d) -> np.ndarray:
    """Frame-level rows: token t's feature row repeated d[t] times, in token order."""
    f = np.asarray(feats)
    rows = []
    for t in range(f.shape[0]):
        for _ in range(int(d[t])):
            rows.append(f[t])
    return np.stack(rows) if rows else np.zeros((0, f.shape[1]), dtype=f.dtype)


def length_regulate(logits, speed: float, feats, cu_seqlens):
    """(durations, frame starts, cu_frames, frames) of a packed batch."""
    d = durations(logits, speed)
    start, cu_frames = frame_offsets(d, cu_seqlens)
    return d, start, cu_frames, expand(feats, d)
