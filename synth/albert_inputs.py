"""Seeded synthetic weights and phoneme-id batches for Kokoro's ALBERT phoneme encoder.

Architecture constants follow "ALBERT: How Kokoro's Phoneme Encoder Works, and Where
CKE Has Reached It" (shivasnotes), sections "1. Factorized embedding" (vocabulary 178,
512 positions, 2 token types, E=128, H=768) and "Inside One Real ALBERT Layer"
(12 heads of 64, FFN 2048, one shared layer run 12 times, final 768->512
projection, LayerNorm epsilon 1e-12 from "How CKE Represents It").

Recipe (the same for every consumer):
  * numpy ``default_rng(seed)`` (PCG64), weight seed 1234, drawn in PARAM_ORDER;
  * every matrix, bias and embedding table ~ N(0, 0.02);
  * LayerNorm gamma = 1, beta = 0 (``ln_affine="random"``: gamma ~ 1 + N(0, 0.1),
    beta ~ N(0, 0.1), drawn after the rest, to catch a swapped gamma/beta);
  * bf16 workloads round every parameter once to the nearest bf16 value (ties to
    even) and keep it as float32, so the GPU library and the oracle see the same
    numbers;
  * ids: 0 at slot 0 and slot L-1 (boundary ids at both ends of the sequence, from
    "How Kokoro TTS Works and Where CKE Stands", section "The whole graph"),
    interior uniform in [1, 177], padding slots 0; token type 0 everywhere;
  * lengths per workload as listed in WORKLOADS; input seed = 100 + workload index.

No arithmetic of the encoder lives here.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

ARCH = dict(
    vocab=178,
    emb=128,
    hidden=768,
    heads=12,
    ffn=2048,
    n_exec=12,
    max_pos=512,
    n_types=2,
    out_dim=512,
    ln_eps=1e-12,
)

# Parameter order = the order of the library's weight struct.  Shapes use the
# [out, in] layout of a linear layer y_j = b_j + sum_i x_i W_{j,i}.
PARAM_ORDER = (
    "word", "pos", "type", "emb_ln_g", "emb_ln_b",
    "w_in", "b_in",
    "wq", "bq", "wk", "bk", "wv", "bv",
    "wo", "bo", "ln1_g", "ln1_b",
    "w1", "b1", "w2", "b2", "ln2_g", "ln2_b",
    "w_out", "b_out",
)

_LN_NAMES = ("emb_ln_g", "emb_ln_b", "ln1_g", "ln1_b", "ln2_g", "ln2_b")


def param_shapes(arch: dict = ARCH) -> dict:
    V, E, H, F = arch["vocab"], arch["emb"], arch["hidden"], arch["ffn"]
    P, NT, O = arch["max_pos"], arch["n_types"], arch["out_dim"]
    return {
        "word": (V, E), "pos": (P, E), "type": (NT, E),
        "emb_ln_g": (E,), "emb_ln_b": (E,),
        "w_in": (H, E), "b_in": (H,),
        "wq": (H, H), "bq": (H,), "wk": (H, H), "bk": (H,), "wv": (H, H), "bv": (H,),
        "wo": (H, H), "bo": (H,), "ln1_g": (H,), "ln1_b": (H,),
        "w1": (F, H), "b1": (F,), "w2": (H, F), "b2": (H,),
        "ln2_g": (H,), "ln2_b": (H,),
        "w_out": (max(O, 0), H), "b_out": (max(O, 0),),
    }


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 value (ties to even); return float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)
    out = r.astype(np.uint32).view(np.float32)
    # NaN/Inf are never drawn here; keep them untouched if a caller passes one.
    bad = ~np.isfinite(a)
    if bad.any():
        out = out.copy()
        out[bad] = a[bad]
    return out.reshape(a.shape)


# Parameters of the transformer layer; with n_groups > 1 each holds n_groups
# stacked copies (leading axis = weight group).
LAYER_PARAMS = ("wq", "bq", "wk", "bk", "wv", "bv", "wo", "bo", "ln1_g", "ln1_b",
                "w1", "b1", "w2", "b2", "ln2_g", "ln2_b")


def make_weights(seed: int = 1234, arch: dict = ARCH, bf16: bool = True,
                 ln_affine: str = "identity", std: float = 0.02, n_groups: int = 1) -> dict:
    """Draw every parameter in PARAM_ORDER from N(0, std); LN gamma=1, beta=0 by default.
    n_groups > 1: the layer parameters get a leading axis of n_groups weight sets."""
    rng = np.random.default_rng(seed)
    shapes = dict(param_shapes(arch))
    if n_groups > 1:
        for k in LAYER_PARAMS:
            shapes[k] = (n_groups,) + tuple(shapes[k])
    w = {}
    for name in PARAM_ORDER:
        shp = shapes[name]
        if name in _LN_NAMES:
            continue
        w[name] = rng.normal(0.0, std, size=shp).astype(np.float32)
    for name in _LN_NAMES:
        shp = shapes[name]
        if name.endswith("_g"):
            w[name] = np.ones(shp, np.float32)
        else:
            w[name] = np.zeros(shp, np.float32)
    if ln_affine == "random":
        for name in _LN_NAMES:
            shp = shapes[name]
            if name.endswith("_g"):
                w[name] = (1.0 + rng.normal(0.0, 0.1, size=shp)).astype(np.float32)
            else:
                w[name] = rng.normal(0.0, 0.1, size=shp).astype(np.float32)
    elif ln_affine != "identity":
        raise ValueError(ln_affine)
    if bf16:
        w = {k: bf16_round(v) for k, v in w.items()}
    return {k: w[k] for k in PARAM_ORDER}


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: batch shape, length law, precision and output width."""
    name: str
    B: int
    T: int
    lengths: str          # "full" | "uniform" | "normal"
    lo: int = 1
    hi: int = 0
    mean: float = 0.0
    sd: float = 0.0
    dtype: str = "bf16"   # "bf16" | "fp32"
    out_dim: int = 512
    seed: int = 100

    def describe(self) -> str:
        law = {"full": f"L={self.T}",
               "uniform": f"L~U[{self.lo},{self.hi}]",
               "normal": f"L=round(N({self.mean:g},{self.sd:g})) clipped to [{self.lo},{self.hi}]"}[self.lengths]
        return f"B={self.B} T={self.T} {law} {self.dtype} out_dim={self.out_dim}"


WORKLOADS = {
    "tiny_fp32_T36": Workload("tiny_fp32_T36", 1, 36, "full", dtype="fp32", out_dim=0, seed=100),
    "b8_T128": Workload("b8_T128", 8, 128, "uniform", lo=16, hi=128, seed=101),
    "b64_T128_normal": Workload("b64_T128_normal", 64, 128, "normal", lo=8, hi=128,
                                mean=60.0, sd=25.0, seed=102),
    "b32_T512_long": Workload("b32_T512_long", 32, 512, "uniform", lo=256, hi=512, seed=103),
    "b256_T128": Workload("b256_T128", 256, 128, "uniform", lo=16, hi=128, seed=104),
    "b1_T64_latency": Workload("b1_T64_latency", 1, 64, "full", seed=105),
}


def draw_lengths(wl: Workload, rng: np.random.Generator) -> np.ndarray:
    if wl.lengths == "full":
        return np.full(wl.B, wl.T, np.int64)
    if wl.lengths == "uniform":
        return rng.integers(wl.lo, wl.hi + 1, size=wl.B).astype(np.int64)
    if wl.lengths == "normal":
        x = np.rint(rng.normal(wl.mean, wl.sd, size=wl.B))
        return np.clip(x, wl.lo, wl.hi).astype(np.int64)
    raise ValueError(wl.lengths)


def make_batch(wl: Workload, vocab: int = ARCH["vocab"], seed: int | None = None):
    """Return (ids[B,T] int64, mask[B,T] uint8, lengths[B] int64) for a workload."""
    rng = np.random.default_rng(wl.seed if seed is None else seed)
    L = draw_lengths(wl, rng)
    ids = np.zeros((wl.B, wl.T), np.int64)
    mask = np.zeros((wl.B, wl.T), np.uint8)
    for b in range(wl.B):
        n = int(L[b])
        if n > 2:
            ids[b, 1:n - 1] = rng.integers(1, vocab, size=n - 2)
        mask[b, :n] = 1
    return ids, mask, L


# Length regulation inputs: duration channels per token (pre-sigmoid).  50
# channels drawn N(-2.9, 1) give sigmoid sums near 3.5, i.e. a few frames per
# token; the channel count is a parameter of the operation.
DURATION_CHANNELS = 50


def make_duration_logits(n_tok: int, channels: int = DURATION_CHANNELS, seed: int = 7,
                         mean: float = -2.9, std: float = 1.0) -> np.ndarray:
    """Seeded fp32 duration logits [n_tok, channels]."""
    rng = np.random.default_rng(seed)
    return rng.normal(mean, std, (n_tok, channels)).astype(np.float32)


def make_features(n_tok: int, width: int = ARCH["out_dim"], seed: int = 8) -> np.ndarray:
    """Seeded bf16-representable token features [n_tok, width] (fp32 array)."""
    rng = np.random.default_rng(seed)
    return bf16_round(rng.normal(0.0, 1.0, (n_tok, width)).astype(np.float32))
