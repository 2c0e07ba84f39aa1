"""TEST INFRASTRUCTURE -- fp64 CPU oracle of the FP8 (E4M3) variant's quantization.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's ``cpu_baseline`` /
``--impl reference`` legs may import this module.  It shares no code with the
CUDA library.

The pages evaluate a quantized build of the encoder against its FP32 outputs
("Kokoro-82M-encoder-hailo10h" model card, section "Eval results": per-sample
cosine and MSE over 16 random N(0,1) post-embedding-LayerNorm inputs of shape
[1, 128, 128]); they fix no scheme for this hardware.  The reading taken here:
both operands of a linear layer are quantized to FP8 E4M3 with one scale per
row along the reduction dimension K (per token for activations, per output
channel for weights):
  amax  = max_k |x[k]|                         (exact)
  s     = amax / 448        (fp32 division)    448 = largest E4M3 magnitude
  inv   = 448 / amax        (fp32 division)
  q[k]  = E4M3(fp32(x[k] * inv))  round to nearest, ties to even, saturating
  a row of zeros has s = 0 and q = 0,
and the product is y[i, j] = (sum_k qx[i, k] qw[j, k]) * sx[i] * sw[j] + b[j].
The code q is an integer decision taken in floating point; it is taken in fp32
here exactly as the kernel takes it (product rounded to fp32, then to E4M3).

E4M3 (the "fn" variant): 1 sign, 4 exponent bits with bias 7, 3 mantissa bits;
normal values 2^(E-7) * (1 + m/8) for E = 1..15 except the all-ones pattern
S.1111.111 (NaN), subnormals 2^-6 * m/8; largest 448, smallest 2^-9.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def e4m3_values() -> np.ndarray:
    """All finite E4M3 magnitudes, ascending (0 included), from the format definition."""
    vals = set()
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue  # NaN pattern
            v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
            vals.add(v)
    return np.array(sorted(vals), dtype=np.float64)


_GRID = e4m3_values()
# the grid is a union of binades of 8 values (the subnormals included), so the
# parity of a value's position equals the parity of its 3-bit mantissa
_EVEN = (np.arange(_GRID.size) % 2) == 0


def round_e4m3(x) -> np.ndarray:
    """Round to the nearest E4M3 value, ties to an even mantissa, saturating at +-448."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.minimum(np.searchsorted(_GRID, a, side="left"), _GRID.size - 1)  # first grid value >= a
    lo = np.maximum(hi - 1, 0)
    glo, ghi = _GRID[lo], _GRID[hi]
    dlo, dhi = a - glo, ghi - a
    pick_hi = np.where(ghi == a, True, np.where(dhi < dlo, True, np.where(dhi > dlo, False, _EVEN[hi])))
    q = np.where(pick_hi, ghi, glo)
    return np.where(x < 0, -q, q)


def e4m3_code(q) -> np.ndarray:
    """The byte encoding of E4M3 values (sign bit 7, exponent bits 6..3, mantissa
    2..0); the sign bit follows the value's sign, negative zero included."""
    q = np.asarray(q, dtype=np.float64)
    a = np.abs(q)
    idx = np.searchsorted(_GRID, a)
    assert np.all(_GRID[np.minimum(idx, _GRID.size - 1)] == a), "not an E4M3 value"
    # grid position = 8 * exponent field + mantissa field
    return (idx + np.where(np.signbit(q), 128, 0)).astype(np.uint8)


def quantize_rows(x):
    """x [rows, K] (fp32-representable) -> (q [rows, K] E4M3 values as float64,
    s [rows] fp32 scales as float64); x[i] is represented by q[i] * s[i]."""
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x32), axis=1)
    nz = amax > 0
    safe = np.where(nz, amax, np.float32(1.0))
    s = np.where(nz, safe / np.float32(E4M3_MAX), np.float32(0.0)).astype(np.float32)
    inv = np.where(nz, np.float32(E4M3_MAX) / safe, np.float32(0.0)).astype(np.float32)
    y = (x32 * inv[:, None]).astype(np.float32)
    return round_e4m3(y), s.astype(np.float64)


def fp8_linear(x, W, b=None) -> np.ndarray:
    """y = (Qx Qw^T) * sx * sw + b: both operands quantized per row along K
    (W [out, in]), products and sums in fp64."""
    qx, sx = quantize_rows(x)
    qw, sw = quantize_rows(W)
    y = (qx @ qw.T) * sx[:, None] * sw[None, :]
    return y if b is None else y + np.asarray(b, np.float64)


def dequantize_rows(q, s) -> np.ndarray:
    return np.asarray(q, np.float64) * np.asarray(s, np.float64)[:, None]
