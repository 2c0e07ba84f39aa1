"""Pins of the FP8 (E4M3, per-row scale) quantization oracle (CPU, no GPU).

Each pin is fixed by the E4M3 format definition, a closed form or an
independent implementation (torch's float8_e4m3fn conversion), not by
re-running the oracle's own arithmetic."""
import numpy as np
import torch

from oracle import fp8_quant as fq


def test_e4m3_grid_from_the_format():
    g = fq.e4m3_values()
    assert g.size == 127                       # 16 exponents x 8 mantissas - NaN, non-negative
    assert g[0] == 0.0 and g[1] == 2.0 ** -9   # smallest subnormal
    assert g[8] == 2.0 ** -6                   # smallest normal
    assert g[-1] == 448.0 and g[-2] == 416.0   # 1.75 * 2^8, 1.625 * 2^8
    t = torch.tensor(g, dtype=torch.float64).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(t, g)


def test_rounding_matches_torch_in_range():
    rng = np.random.default_rng(0)
    g = fq.e4m3_values()
    mids = (g[:-1] + g[1:]) / 2                 # exact ties: ties to even
    x = np.concatenate([rng.uniform(-448, 448, 20000), rng.normal(0, 1, 20000), rng.normal(0, 0.01, 5000),
                        mids, -mids, g, -g])
    ref = torch.tensor(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(fq.round_e4m3(x), ref)


def test_ties_go_to_the_even_mantissa_and_saturation():
    assert fq.round_e4m3(1.0625) == 1.0       # between 1.0 (m=0) and 1.125 (m=1)
    assert fq.round_e4m3(1.1875) == 1.25      # between 1.125 (m=1) and 1.25 (m=2)
    assert fq.round_e4m3(15.5) == 16.0        # between 15 (m=7) and 16 (next binade, m=0)
    assert fq.round_e4m3(1e6) == 448.0 and fq.round_e4m3(-1e6) == -448.0
    assert fq.round_e4m3(-3.0) == -3.0


def test_byte_codes_match_torch():
    g = fq.e4m3_values()
    vals = np.concatenate([g, -g])             # negative zero included
    want = torch.tensor(vals, dtype=torch.float64).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(fq.e4m3_code(vals), want)
    # a negative value that rounds to zero keeps its sign
    tiny = np.array([-1e-9, 1e-9])
    want = torch.tensor(tiny).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(fq.e4m3_code(fq.round_e4m3(tiny)), want)
    assert list(want) == [0x80, 0x00]


def test_row_scales_closed_forms():
    x = np.array([[448.0, -1.0, 2.0, 0.5], [0.0, 0.0, 0.0, 0.0], [1.0, -1.0, 0.25, 0.0]], np.float32)
    q, s = fq.quantize_rows(x)
    assert s[0] == 1.0 and np.all(q[0] == [448.0, -1.0, 2.0, 0.5])  # amax 448: scale 1, exact
    assert s[1] == 0.0 and np.all(q[1] == 0.0)                     # zero row
    assert s[2] == np.float32(1.0) / np.float32(448.0)
    assert q[2, 0] == 448.0 and q[2, 1] == -448.0 and q[2, 2] == 112.0  # 0.25 * 448
    # the row maximum always maps onto +-448
    rng = np.random.default_rng(1)
    q, s = fq.quantize_rows(rng.normal(0, 3, (50, 96)).astype(np.float32))
    assert np.all(np.max(np.abs(q), axis=1) == 448.0)


def test_relative_error_bound_of_normals():
    # E4M3 keeps 3 mantissa bits: relative error at most 2^-4 for normal values,
    # on top of one fp32 rounding of x * inv
    rng = np.random.default_rng(2)
    x = rng.normal(0, 1, (64, 256)).astype(np.float32)
    q, s = fq.quantize_rows(x)
    d = fq.dequantize_rows(q, s)
    sel = np.abs(q) >= 2.0 ** -6
    assert np.max(np.abs(d[sel] - x[sel]) / np.abs(x[sel])) <= 2.0 ** -4 * (1 + 1e-6)


def test_fp8_linear_against_a_double_loop():
    rng = np.random.default_rng(3)
    x = rng.normal(0, 1, (3, 64)).astype(np.float32)
    W = rng.normal(0, 0.05, (5, 64)).astype(np.float32)
    b = rng.normal(0, 0.1, 5)
    qx, sx = fq.quantize_rows(x)
    qw, sw = fq.quantize_rows(W)
    ref = np.array([[sum(qx[i, k] * qw[j, k] for k in range(64)) * sx[i] * sw[j] + b[j] for j in range(5)]
                    for i in range(3)])
    np.testing.assert_allclose(fq.fp8_linear(x, W, b), ref, rtol=1e-12, atol=1e-12)
    # and it approximates the unquantized product to E4M3 precision
    exact = x.astype(np.float64) @ W.astype(np.float64).T + b
    assert np.max(np.abs(fq.fp8_linear(x, W, b) - exact)) < 0.1 * np.max(np.abs(exact))
