"""TEST INFRASTRUCTURE -- ctypes front end of the fp64 CPU oracle (albert_oracle.c).

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's ``cpu_baseline`` /
``--impl reference`` legs may import this package.  The product library never
calls it, and it never calls the product library.

The C file states what each function computes and which page passage it follows.
This wrapper only marshals numpy arrays: it converts parameters to float64 and
passes pointers.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "albert_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_albert.so")

PARAM_ORDER = (
    "word", "pos", "type", "emb_ln_g", "emb_ln_b",
    "w_in", "b_in",
    "wq", "bq", "wk", "bk", "wv", "bv",
    "wo", "bo", "ln1_g", "ln1_b",
    "w1", "b1", "w2", "b2", "ln2_g", "ln2_b",
    "w_out", "b_out",
)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, strict IEEE: no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared",
               "-fPIC", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


class _Cfg(C.Structure):
    _fields_ = [(n, C.c_int) for n in ("vocab", "emb", "hidden", "heads", "ffn", "n_exec",
                                       "max_pos", "n_types", "out_dim")] + [("ln_eps", C.c_double)]


class _W(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in PARAM_ORDER]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        d = C.c_void_p
        _lib.orc_linear.argtypes = [d, C.c_int, C.c_int, d, d, C.c_int, d]
        _lib.orc_layer_norm.argtypes = [d, C.c_int, C.c_int, d, d, C.c_double, d]
        _lib.orc_gelu_tanh.argtypes = [C.c_double]
        _lib.orc_gelu_tanh.restype = C.c_double
        _lib.orc_gelu_rows.argtypes = [d, C.c_long, d]
        _lib.orc_attention.argtypes = [d, d, d, C.c_int, d, C.c_int, C.c_int, C.c_int, d, C.c_int]
        _lib.orc_embed.argtypes = [C.POINTER(_Cfg), C.POINTER(_W), d, d, C.c_int, d]
        _lib.orc_layer.argtypes = [C.POINTER(_Cfg), C.POINTER(_W), d, d, C.c_int]
        _lib.orc_encode.argtypes = [C.POINTER(_Cfg), C.POINTER(_W), d, d, C.c_int, d]
        _lib.orc_encode_batch.argtypes = [C.POINTER(_Cfg), C.POINTER(_W), d, d, C.c_int,
                                          C.c_int, d]
        _lib.orc_set_threads.argtypes = [C.c_int]
        _lib.orc_num_threads.restype = C.c_int
    return _lib


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


def num_threads() -> int:
    return int(lib().orc_num_threads())


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a: np.ndarray):
    return C.c_void_p(a.ctypes.data)


class Model:
    """Holds fp64 copies of the parameters and the architecture constants."""

    def __init__(self, weights: dict, arch: dict, n_exec: int | None = None,
                 out_dim: int | None = None):
        self.cfg = _Cfg(arch["vocab"], arch["emb"], arch["hidden"], arch["heads"], arch["ffn"],
                        arch["n_exec"] if n_exec is None else n_exec, arch["max_pos"],
                        arch["n_types"], arch["out_dim"] if out_dim is None else out_dim,
                        float(arch["ln_eps"]))
        self.w64 = {k: _f64(weights[k]) for k in PARAM_ORDER}
        self.cw = _W(*[self.w64[k].ctypes.data for k in PARAM_ORDER])

    @property
    def out_width(self) -> int:
        return self.cfg.out_dim if self.cfg.out_dim > 0 else self.cfg.hidden

    def encode(self, ids, mask) -> np.ndarray:
        """ids, mask: [T] or [B, T].  Returns fp64 [.., T, out_width]."""
        ids = np.ascontiguousarray(ids, dtype=np.int64)
        mask = np.ascontiguousarray(mask, dtype=np.uint8)
        squeeze = ids.ndim == 1
        if squeeze:
            ids, mask = ids[None], mask[None]
        B, T = ids.shape
        out = np.zeros((B, T, self.out_width), np.float64)
        rc = lib().orc_encode_batch(C.byref(self.cfg), C.byref(self.cw), _p(ids), _p(mask),
                                    B, T, _p(out))
        if rc:
            raise ValueError("oracle rejected the input (id out of range, T > max_pos or "
                             "an all-masked sequence)")
        return out[0] if squeeze else out

    def embed(self, ids, mask) -> np.ndarray:
        ids = np.ascontiguousarray(ids, dtype=np.int64)
        mask = np.ascontiguousarray(mask, dtype=np.uint8)
        T = ids.shape[0]
        out = np.zeros((T, self.cfg.emb), np.float64)
        if lib().orc_embed(C.byref(self.cfg), C.byref(self.cw), _p(ids), _p(mask), T, _p(out)):
            raise ValueError("oracle rejected the input")
        return out

    def layer(self, x, mask) -> np.ndarray:
        x = _f64(x).copy()
        mask = np.ascontiguousarray(mask, dtype=np.uint8)
        if lib().orc_layer(C.byref(self.cfg), C.byref(self.cw), _p(x), _p(mask), x.shape[0]):
            raise ValueError("oracle rejected the input")
        return x


LAYER_PARAMS = ("wq", "bq", "wk", "bk", "wv", "bv", "wo", "bo", "ln1_g", "ln1_b",
                "w1", "b1", "w2", "b2", "ln2_g", "ln2_b")


def encode_grouped(weights: dict, arch: dict, ids, mask, n_groups: int, n_exec: int | None = None,
                   out_dim: int | None = None) -> np.ndarray:
    """ALBERT with grouped sharing ("ALBERT: How Kokoro's Phoneme Encoder Works",
    section "2. Cross-layer parameter sharing": several distinct weight sets, each
    reused over a block of consecutive executions).  The layer parameters hold
    n_groups stacked sets; execution i uses set floor(i * n_groups / n_exec).
    One sequence (ids, mask: [T]); returns fp64 [T, out_width], padding rows 0."""
    n_exec = arch["n_exec"] if n_exec is None else n_exec
    out_dim = arch["out_dim"] if out_dim is None else out_dim
    ids = np.asarray(ids)
    mask = np.asarray(mask, dtype=np.uint8)
    L = int(mask.sum())
    # one group: the layer parameters are not stacked
    sets = [{k: (weights[k][g] if k in LAYER_PARAMS and n_groups > 1 else weights[k]) for k in PARAM_ORDER}
            for g in range(n_groups)]
    # embedding, its LayerNorm and the 128 -> 768 projection (no execution, no final projection)
    x = Model(sets[0], arch, n_exec=0, out_dim=0).encode(ids[:L], mask[:L])
    for i in range(n_exec):
        x = Model(sets[i * n_groups // n_exec], arch, n_exec=1, out_dim=0).layer(x, mask[:L])
    if out_dim > 0:
        x = linear(x, weights["w_out"], weights["b_out"])
    out = np.zeros((ids.shape[0], x.shape[1]), np.float64)
    out[:L] = x
    return out


def linear(x, W, b=None) -> np.ndarray:
    x, W = _f64(x), _f64(W)
    b = None if b is None else _f64(b)
    rows, n_in = x.shape
    n_out = W.shape[0]
    y = np.empty((rows, n_out), np.float64)
    lib().orc_linear(_p(x), rows, n_in, _p(W), None if b is None else _p(b), n_out, _p(y))
    return y


def layer_norm(x, g, b, eps) -> np.ndarray:
    x, g, b = _f64(x), _f64(g), _f64(b)
    rows, n = x.shape
    y = np.empty_like(x)
    lib().orc_layer_norm(_p(x), rows, n, _p(g), _p(b), float(eps), _p(y))
    return y


def gelu(x) -> np.ndarray:
    x = _f64(x)
    y = np.empty_like(x)
    lib().orc_gelu_rows(_p(x), x.size, _p(y))
    return y


def gelu_scalar(x: float) -> float:
    return float(lib().orc_gelu_tanh(float(x)))


def attention(q, k, v, key_mask, heads) -> np.ndarray:
    """q, k, v: [T, heads*dh] fp64; key_mask: [T] (1 = valid key)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    key_mask = np.ascontiguousarray(key_mask, dtype=np.uint8)
    T, D = q.shape
    ctx = np.empty((T, D), np.float64)
    if lib().orc_attention(_p(q), _p(k), _p(v), D, _p(key_mask), T, heads, D // heads,
                           _p(ctx), D):
        raise ValueError("no valid key")
    return ctx
