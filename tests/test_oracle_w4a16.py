"""Pins of the oracle's W4A16 product (CPU only): 16-bit activations times
NVFP4 weights dequantized to their exact values (aixq.cc article on Unsloth
Dynamic NVFP4, section "核心差异：W4A4 vs W4A16": NVIDIA's scheme keeps the
activations in 16 bits and dequantizes the 4-bit weights before the product).
Each check uses something other than the oracle's own code: exact rationals
built from the code and scale bytes with the page's E2M1 grid and torch's
E4M3 decode, a closed form, and a symmetry."""
from fractions import Fraction

import numpy as np
import torch

import oracle

GRID = [0, 0.5, 1, 1.5, 2, 3, 4, 6]


def e4m3(byte):
    return float(torch.tensor([byte], dtype=torch.uint8).view(torch.float8_e4m3fn).float()[0])


def exact_value(q, n, k):
    byte = int(q.codes[n, k // 2])
    code = byte & 15 if k % 2 == 0 else byte >> 4
    mag = Fraction(GRID[code & 7]).limit_denominator()
    s = Fraction(e4m3(int(q.scales[n, k // 16])))
    v = mag * s * Fraction(float(np.float32(q.g)))
    return -v if code & 8 else v


def bf16_bits(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_w4a16_exact_rationals():
    rng = np.random.default_rng(3)
    M, N, K = 3, 5, 64
    xb = bf16_bits(rng.standard_normal((M, K)) * 3)
    w = rng.standard_normal((N, K)).astype(np.float32) * 0.02
    w[1, 7] = 0.9                                     # an outlier sets the tensor scale
    wq = oracle.quantize(w)
    y = oracle.w4a16_gemm_f64(xb, wq)
    xv = oracle.bf16_bits_to_f32(xb)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(xv[m, k])) * exact_value(wq, n, k) for k in range(K))
            assert abs(Fraction(y[m, n]) - exact) <= abs(exact) * Fraction(1, 10 ** 12) + Fraction(1, 10 ** 300)


def test_w4a16_closed_form_constant_weights():
    """Every weight code 1.0 (0x2), every block scale 1.0 (0x38), g = 2^-3:
    each dequantized weight is 1/8, so Y[m][n] = sum_k x[m][k] / 8."""
    M, N, K = 4, 6, 128
    q = oracle.Quantized(np.full((N, K // 2), 0x22, np.uint8), np.full((N, K // 16), 0x38, np.uint8),
                         np.float32(0.125), N, K)
    x = np.random.default_rng(5).integers(-64, 64, (M, K)).astype(np.float32) / 16   # exact in bf16
    y = oracle.w4a16_gemm_f64(bf16_bits(x), q)
    assert np.array_equal(y, np.repeat(x.sum(axis=1, keepdims=True) / 8, N, axis=1))


def test_w4a16_sign_symmetry():
    """Setting the sign bit of every weight code negates the product, and
    negating the activations does too."""
    rng = np.random.default_rng(7)
    x = bf16_bits(rng.standard_normal((2, 96)))
    wq = oracle.quantize(rng.standard_normal((3, 96)).astype(np.float32))
    y = oracle.w4a16_gemm_f64(x, wq)
    neg = oracle.Quantized(wq.codes ^ 0x88, wq.scales, wq.g, wq.rows, wq.cols)
    assert np.array_equal(oracle.w4a16_gemm_f64(x, neg), -y)
    assert np.array_equal(oracle.w4a16_gemm_f64(x ^ np.uint16(0x8000), wq), -y)
