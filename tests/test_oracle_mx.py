"""Pins of the oracle's MXFP4 functions (CPU only).

MXFP4 per the eefocus.com article on FP4 vs INT4, section
"FP4被视为下一代AI计算的核心标准": 32 consecutive E2M1 elements share one
8-bit scale, usually E8M0; about 4.25 bits per value.  The page gives no rule
for choosing the scale; the oracle's reading (M1) is the smallest power of two
2^e that brings the block's largest magnitude into the E2M1 range
(bamax <= 6 * 2^e), clamped to the E8M0 range.  Each check below uses
something other than the oracle's own code: torch's E8M0 dtype, a brute-force
search over every scale byte, a separately written nearest-code rule, exact
round trips and closed forms.
"""
import math

import numpy as np
import pytest
import torch

import oracle

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e8m0_torch(byte: int) -> float:
    return float(torch.tensor([byte], dtype=torch.uint8).view(torch.float8_e8m0fnu).float()[0])


def scale_by_search(bamax: float) -> int:
    """Smallest scale byte s (0..254) with bamax <= 6 * 2^(s - 127), exactly."""
    for s in range(255):
        if bamax <= math.ldexp(6.0, s - 127):
            return s
    raise AssertionError("no scale covers this block")


def nearest_code(v: float) -> int:
    """E2M1 code of v: nearest grid magnitude, a tie going to the even index,
    the sign of v (a negative zero included) in bit 3."""
    a = abs(v)
    d = np.abs(GRID - a)
    best = min(range(8), key=lambda i: (d[i], i % 2))
    return best | (8 if math.copysign(1.0, v) < 0 else 0)


def codes_of(q, r, c):
    byte = int(q.codes[r, c // 2])
    return byte & 15 if c % 2 == 0 else byte >> 4


def test_e8m0_decode_all_bytes_against_torch():
    for b in range(255):
        assert oracle.e8m0_value(b) == e8m0_torch(b) == math.ldexp(1.0, b - 127), b
    assert math.isnan(oracle.e8m0_value(255)) and math.isnan(e8m0_torch(255))


def _bamax_cases():
    f32 = np.float32
    vals = [0.0, float(np.finfo(f32).max), float(np.finfo(f32).smallest_subnormal),
            float(np.finfo(f32).tiny)]
    for k in range(-130, 127):
        if math.ldexp(6.0, k) > float(np.finfo(f32).max):
            continue
        edge = f32(math.ldexp(6.0, k))                       # exact: 1.5 * 2^(k+2)
        vals += [float(edge), float(np.nextafter(edge, f32(np.inf))), float(np.nextafter(edge, f32(0)))]
    rng = np.random.default_rng(7)
    vals += [float(f32(v)) for v in np.exp(rng.uniform(-100, 88, 3000))]
    return [v for v in vals if np.isfinite(np.float32(v))]


def test_scale_rule_is_the_smallest_power_of_two_that_fits():
    for v in _bamax_cases():
        assert oracle.mx_block_scale(v) == scale_by_search(v), v


def _heavy_tailed(rows, cols, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols)).astype(np.float32)
    x[rng.random(x.shape) < 0.02] *= 60
    x *= np.exp2(rng.integers(-20, 20, size=(rows, 1))).astype(np.float32)   # rows at many magnitudes
    x[0, :32] = 0.0                                                            # an all-zero block
    x[1, 32:64] = np.float32(1e-39)                                            # a subnormal block
    x[2, 5] = -np.float32(1e-3) * np.abs(x[2, :32]).max()                      # rounds to -0
    return x


def test_every_scale_and_code_against_search_and_nearest_rule():
    x = _heavy_tailed(6, 256, seed=1)
    q = oracle.mx_quantize(x)
    for r in range(x.shape[0]):
        for b in range(x.shape[1] // 32):
            blk = x[r, 32 * b:32 * b + 32].astype(np.float64)
            s = scale_by_search(float(np.abs(blk).max()))
            assert q.scales[r, b] == s, (r, b)
            scale = e8m0_torch(s)
            for i in range(32):
                assert codes_of(q, r, 32 * b + i) == nearest_code(blk[i] / scale), (r, b, i)
    assert codes_of(q, 2, 5) == 0x8                                            # sign kept at zero


def test_scale_is_tight():
    """A non-zero block above the smallest scale would saturate at the next
    smaller scale: 3 * X < bamax <= 6 * X."""
    x = _heavy_tailed(8, 512, seed=2)
    q = oracle.mx_quantize(x)
    bamax = np.abs(x.astype(np.float64)).reshape(8, 16, 32).max(axis=2)
    scale = np.vectorize(e8m0_torch)(q.scales.astype(int))
    live = (bamax > 0) & (q.scales > 0)
    assert live.sum() > 100
    assert (bamax[live] <= 6 * scale[live]).all() and (bamax[live] > 3 * scale[live]).all()


@pytest.mark.parametrize("k", [-127, -60, -1, 0, 7, 100, 125])
def test_exact_round_trip_of_every_value(k):
    """Blocks holding every signed E2M1 magnitude times 2^k, with 6 * 2^k
    present, get the scale 2^k and dequantize back exactly."""
    mags = np.concatenate([GRID, -GRID])                                      # 16 values
    blk = np.concatenate([mags, mags[::-1]]).astype(np.float64) * math.ldexp(1.0, k)
    x = np.stack([blk, -blk]).astype(np.float32)
    assert np.array_equal(x.astype(np.float64), np.stack([blk, -blk]))         # representable
    q = oracle.mx_quantize(x)
    assert (q.scales == k + 127).all()
    assert np.array_equal(oracle.mx_dequantize_f64(q), x.astype(np.float64))


def test_block_granularity():
    x = _heavy_tailed(4, 256, seed=3)
    q0 = oracle.mx_quantize(x)
    y = x.copy()
    y[2, 100] = np.float32(1e6)                                                # block 3 of row 2
    q1 = oracle.mx_quantize(y)
    changed_scales = np.argwhere(q0.scales != q1.scales)
    assert changed_scales.tolist() == [[2, 3]]
    changed_bytes = np.argwhere(q0.codes != q1.codes)
    assert len(changed_bytes) > 0
    assert all(r == 2 and 48 <= c < 64 for r, c in changed_bytes)


def test_error_bound():
    """Each dequantized value is within half an E2M1 step (at its magnitude)
    of the input, in units of the block scale."""
    x = _heavy_tailed(8, 512, seed=4).astype(np.float64)
    q = oracle.mx_quantize(x.astype(np.float32))
    d = oracle.mx_dequantize_f64(q)
    scale = np.repeat(np.vectorize(e8m0_torch)(q.scales.astype(int)), 32, axis=1)
    v = np.abs(x) / scale
    half_step = np.where(v <= 2, 0.25, np.where(v <= 4, 0.5, 1.0))
    assert (np.abs(x - d) <= half_step * scale).all()


def test_storage_accounting_matches_page(facts):
    mx = facts["mxfp4"]
    assert mx["block"] == 32
    for rows, cols in [(1, 32), (128, 4096), (17408, 5120)]:
        assert oracle.mx_storage_bytes(rows, cols) * 8 / (rows * cols) == mx["bits_per_value"]


def test_gemm_closed_form_constant_operands():
    """A = 1.5 and B = -0.75 everywhere (both exact in MXFP4): Y = -1.125 K."""
    M, N, K = 5, 7, 96
    a = oracle.mx_quantize(np.full((M, K), 1.5, np.float32))
    b = oracle.mx_quantize(np.full((N, K), -0.75, np.float32))
    assert np.array_equal(oracle.mx_gemm_f64(a, b), np.full((M, N), -1.125 * K))


def test_gemm_matches_dot_products_of_exact_values():
    """Operands built from exactly representable MXFP4 values (one scale per
    block): the GEMM is the plain fp64 product of the inputs."""
    rng = np.random.default_rng(5)
    M, N, K = 4, 6, 128

    def exact(rows):
        ks = rng.integers(-10, 10, size=(rows, K // 32))
        codes = rng.integers(0, 16, size=(rows, K))
        vals = np.where(codes >= 8, -1.0, 1.0) * GRID[codes % 8]
        vals[:, ::32] = 6.0                                                    # pin each block's scale
        return (vals * np.exp2(np.repeat(ks, 32, axis=1))).astype(np.float32)

    A, B = exact(M), exact(N)
    y = oracle.mx_gemm_f64(oracle.mx_quantize(A), oracle.mx_quantize(B))
    assert np.array_equal(y, A.astype(np.float64) @ B.astype(np.float64).T)
