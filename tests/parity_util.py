"""Helpers shared by the parity tests: tolerances and oracle sampling.

Tolerances (stated for the encoder output over valid tokens):
  bf16 path: max |gpu - oracle| <= 3e-2 and per-token cosine >= 0.999;
  fp32 path: ||gpu - oracle||_inf / ||oracle||_inf <= 1e-4.
Hidden-state checkpoints (the [T, 768] LayerNorm outputs, unit variance, |x| up
to ~5) get the same cosine bar and an elementwise bar of 3e-2 + 2^-7 |ref|:
one bf16 ulp of the value on top of the output bar, for the extra bf16
rounding of z * gamma that the deferred LayerNorm carries to its consumer
(a half-ulp at |x| in [4, 8) is already 0.0156).
"""
import numpy as np

import oracle
import synth

BF16_MAX_ABS = 3e-2
BF16_MIN_COS = 0.999
FP32_REL = 1e-4


def per_token_cosine(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    a = a.astype(np.float64)
    b = b.astype(np.float64)
    return (a * b).sum(-1) / (np.linalg.norm(a, axis=-1) * np.linalg.norm(b, axis=-1) + 1e-300)


def check_bf16(gpu: np.ndarray, ref: np.ndarray, what: str = "", checkpoint: bool = False):
    diff = np.abs(gpu.astype(np.float64) - ref)
    err = float(np.max(diff))
    cos = float(np.min(per_token_cosine(gpu, ref)))
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite output"
    if checkpoint:
        excess = float(np.max(diff - (BF16_MAX_ABS + 2.0 ** -7 * np.abs(ref))))
        assert excess <= 0, f"{what}: checkpoint error {err:.3e} exceeds 3e-2 + 2^-7|ref| by {excess:.3e}"
    else:
        assert err <= BF16_MAX_ABS, f"{what}: max abs err {err:.3e} > {BF16_MAX_ABS}"
    assert cos >= BF16_MIN_COS, f"{what}: min per-token cosine {cos:.6f} < {BF16_MIN_COS}"
    return err, cos


def check_fp32(gpu: np.ndarray, ref: np.ndarray, what: str = ""):
    rel = float(np.max(np.abs(gpu.astype(np.float64) - ref)) / np.max(np.abs(ref)))
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite output"
    assert rel <= FP32_REL, f"{what}: relative error {rel:.3e} > {FP32_REL}"
    return rel


# (label, sequences, valid tokens, worst error, worst per-token cosine, error kind)
# of every whole-encoder comparison in this session, printed in the summary
PARITY_REPORT = []


def record_parity(label, n_seq, n_tok, err, cos, kind):
    PARITY_REPORT.append((label, n_seq, n_tok, err, cos, kind))


def oracle_rows(weights: dict, ids: np.ndarray, mask: np.ndarray, L: np.ndarray, seqs, n_exec=None,
                out_dim=None) -> dict:
    """Oracle outputs of the valid rows of the chosen sequences (each alone, unpadded)."""
    m = oracle.Model(weights, synth.ARCH, n_exec=n_exec, out_dim=out_dim)
    out = {}
    for b in seqs:
        n = int(L[b])
        out[b] = m.encode(ids[b, :n], mask[b, :n])
    return out
