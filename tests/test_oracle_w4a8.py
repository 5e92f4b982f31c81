"""Pins of the oracle's MXFP8 quantizer and W4A8 product (CPU only).

W4A8 per the eefocus.com article on FP4 vs INT4 (the Zhouyi X3 passage): FP4
weights with activations quantized to FP8.  The page gives no scale rule; the
oracle's readings (X1, X2) give FP8 activations the MX block structure of the
FP4 weights: 32 values share an E8M0 scale X = 2^e, the smallest power of two
with bamax <= 448 X, and each element is the E4M3 RNE of x / X.  Each check
below uses something other than the oracle's own code: a brute-force search
over every scale byte, torch's float8_e4m3fn conversion, exact round trips
and a closed form."""
import math

import numpy as np
import torch

import oracle


def scale_by_search(bamax: float) -> int:
    for s in range(255):
        if bamax <= math.ldexp(448.0, s - 127):
            return s
    raise AssertionError("no scale covers this block")


def e4m3_torch(v: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_mx8_scale_rule_by_search():
    f32 = np.float32
    vals = [0.0, float(np.finfo(f32).max), float(np.finfo(f32).smallest_subnormal), float(np.finfo(f32).tiny)]
    for k in range(-140, 120):
        edge = f32(math.ldexp(448.0, k))
        vals += [float(edge), float(np.nextafter(edge, f32(0))), float(np.nextafter(edge, f32(np.inf)))]
    vals += list(np.abs(np.random.default_rng(0).standard_normal(2000).astype(np.float32) * 1e3))
    for b in vals:
        want = 0 if b == 0.0 else min(max(scale_by_search(b), 0), 254)
        assert oracle.mx8_block_scale(b) == want, b


def test_mx8_elements_against_torch():
    """Every element is torch's E4M3 conversion of x / X (exact quotient)."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal((40, 256)).astype(np.float32) * np.exp(rng.uniform(-8, 8, (40, 1))).astype(np.float32)
    x[rng.random(x.shape) < 0.01] *= 50
    x[3, :32] = 0.0
    x[4, 5] = -0.0
    q = oracle.mx8_quantize(x)
    X = np.ldexp(1.0, q.scales.astype(np.int64) - 127).repeat(32, axis=1)
    v = (x.astype(np.float64) / X).astype(np.float32)
    assert np.array_equal(q.elems, e4m3_torch(v))
    assert q.elems[4, 5] == 0x80                       # the sign of -0 is kept
    assert np.all(np.abs(oracle.mx8_dequantize_f64(q)) <= 448.0 * X)


def test_mx8_round_trip_exact():
    """Values e * 2^k with e on the E4M3 grid come back exactly when each block
    holds 448 * 2^k (so X = 2^k)."""
    grid = np.array([oracle.e4m3_value(b) for b in range(0x7F)], np.float64)
    for k in (-20, -3, 0, 7, 60):
        x = np.zeros((2, 128), np.float32)
        x[:, ::32] = 448.0 * 2.0 ** k
        x[0, 1:32] = grid[1:32] * 2.0 ** k
        x[1, 33:64] = -grid[40:71] * 2.0 ** k
        x[0, 65:96] = grid[90:121] * 2.0 ** k
        q = oracle.mx8_quantize(x)
        assert np.all(q.scales == 127 + k)
        assert np.array_equal(oracle.mx8_dequantize_f64(q), x.astype(np.float64))


def test_w4a8_closed_form():
    """Activations all 1.0 with scale 2^0 (E4M3 0x38, E8M0 127) and weights
    all 0.5 with scale 2^2: each product is 2, Y = 2 K everywhere."""
    M, N, K = 3, 4, 96
    x = oracle.QuantizedMX8(np.full((M, K), 0x38, np.uint8), np.full((M, K // 32), 127, np.uint8), M, K)
    w = oracle.QuantizedMX(np.full((N, K // 2), 0x11, np.uint8), np.full((N, K // 32), 129, np.uint8), N, K)
    assert np.array_equal(oracle.w4a8_gemm_f64(x, w), np.full((M, N), 2.0 * K))


def test_w4a8_storage_and_sign():
    """Negating the activations negates the product."""
    rng = np.random.default_rng(2)
    xq = oracle.mx8_quantize(rng.standard_normal((2, 64)).astype(np.float32))
    wq = oracle.mx_quantize(rng.standard_normal((3, 64)).astype(np.float32))
    y = oracle.w4a8_gemm_f64(xq, wq)
    neg = oracle.QuantizedMX8(xq.elems ^ 0x80, xq.scales, xq.rows, xq.cols)
    assert np.array_equal(oracle.w4a8_gemm_f64(neg, wq), -y)
