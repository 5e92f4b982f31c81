"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these checks re-types the oracle's own formula: each compares the
oracle with an independent fact (a value stated on the pages, a hand-derived
fixture, an independent decoder, exact rational arithmetic, brute-force
optimality, a closed form or an invariant), chosen so that a dropped term, a
wrong sign, index or tie rule, or a transposed operand fails at least one.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import reading_vectors
from nvfp4_block_scaled_21_b200 import workloads

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")




# ---------------------------------------------------------------------------
# E2M1
# ---------------------------------------------------------------------------

def test_e2m1_grid_matches_page_facts(facts):
    grid = facts["e2m1"]["non_negative_grid"]
    vals = [oracle.e2m1_value(c) for c in range(16)]
    assert vals[:8] == grid
    # sign bit 3 mirrors the grid, including a negative zero
    for c in range(8):
        assert vals[8 + c] == -grid[c]
    assert math.copysign(1.0, vals[8]) == -1.0
    # range about +-6 (1 sign, 2 exponent, 1 mantissa bit)
    assert max(abs(v) for v in vals) == facts["e2m1"]["range"]
    assert len({abs(v) for v in vals}) == 8   # 3 magnitude bits, all distinct


def _e2m1_nearest_by_grid(v, grid):
    """Independent brute force over the page grid: nearest, ties to the even
    magnitude index, saturate beyond the largest magnitude, sign from v."""
    a = min(abs(v), grid[-1]) if abs(v) > grid[-1] else abs(v)
    best = min(range(8), key=lambda i: (abs(a - grid[i]), i % 2))
    return (8 if math.copysign(1.0, v) < 0 else 0) | best


def test_e2m1_encode_brute_force_sweep(facts):
    grid = facts["e2m1"]["non_negative_grid"]
    rng = np.random.default_rng(123)
    vs = np.concatenate([
        rng.uniform(-8, 8, 20000).astype(np.float32),
        np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 6.5, 100.0,
                  -0.25, -0.75, -5.0, -1e-30, 0.0, -0.0, 0.2499999, 0.2500001],
                 dtype=np.float32)])
    got = oracle.e2m1_encode_array(vs)
    want = np.array([_e2m1_nearest_by_grid(float(v), grid) for v in vs], np.uint8)
    np.testing.assert_array_equal(got, want)


def test_e2m1_ties_go_to_even_index():
    # midpoints and where RNE sends them (even magnitude index)
    cases = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for v, want in cases.items():
        assert oracle.e2m1_value(oracle.e2m1_encode(v)) == want
        assert oracle.e2m1_value(oracle.e2m1_encode(-v)) == -want


# ---------------------------------------------------------------------------
# E4M3
# ---------------------------------------------------------------------------

def test_e4m3_decode_all_256_against_torch():
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    got = oracle.e4m3_value_array(np.arange(256, dtype=np.uint8))
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])
    assert np.array_equal(np.signbit(got[ok]), np.signbit(ref[ok]))
    assert got[0x7E] == 448.0


def _torch_e4m3_rne(t):
    return torch.from_numpy(np.ascontiguousarray(t, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_encode_matches_torch_rne_in_range():
    rng = np.random.default_rng(7)
    t = np.concatenate([
        rng.uniform(0, 448, 300000),
        np.exp(rng.uniform(np.log(1e-4), np.log(448), 300000)),
        rng.uniform(0, 2.0 ** -6, 50000),                       # subnormal range
    ]).astype(np.float32)
    np.testing.assert_array_equal(oracle.e4m3_encode_array(t), _torch_e4m3_rne(t))


def test_e4m3_encode_midpoints_tie_to_even():
    vals = oracle.e4m3_value_array(np.arange(0x7F, dtype=np.uint8))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    assert np.all(mids.astype(np.float64) == (vals[:-1] + vals[1:]) / 2)  # exact in fp32
    got = oracle.e4m3_encode_array(mids)
    lo = np.arange(0x7E, dtype=np.uint8)
    want = np.where(lo % 2 == 0, lo, lo + 1).astype(np.uint8)
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(got, _torch_e4m3_rne(mids))
    # one ulp either side of each midpoint rounds away from the tie
    below = np.nextafter(mids, np.float32(0))
    above = np.nextafter(mids, np.float32(1e9))
    np.testing.assert_array_equal(oracle.e4m3_encode_array(below), lo)
    np.testing.assert_array_equal(oracle.e4m3_encode_array(above), lo + 1)


def test_e4m3_encode_saturates_and_flushes():
    assert oracle.e4m3_encode(448.0) == 0x7E
    assert oracle.e4m3_encode(463.9) == 0x7E
    assert oracle.e4m3_encode(1e30) == 0x7E          # satfinite, never 0x7F
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00     # half the smallest subnormal: tie to 0
    assert oracle.e4m3_encode(np.nextafter(np.float32(2.0 ** -10), np.float32(1))) == 0x01
    assert oracle.e4m3_encode(0.0) == 0x00


# ---------------------------------------------------------------------------
# Quantizer
# ---------------------------------------------------------------------------

def test_worked_example_hand_derived(golden_dir):
    with open(os.path.join(golden_dir, "worked_example_1x32.json")) as f:
        ex = json.load(f)
    x = np.array([float(v) for v in ex["x"]], np.float32).reshape(1, 32)
    q = oracle.quantize(x)
    assert float(q.g) == float(ex["g"])
    assert [f"{b:02x}" for b in q.scales[0]] == ex["scales_hex"]
    assert [f"{b:02x}" for b in q.codes[0]] == ex["packed_bytes_hex"]
    y = oracle.dequantize(q)
    want = np.array([float(v) for v in ex["dequantized"]], np.float32)
    np.testing.assert_array_equal(y[0], want)
    assert np.array_equal(np.signbit(y[0]), np.signbit(want))


def _e4m3_positive_finite():
    return [b for b in range(1, 0x7F)]  # 126 codes: 0x01..0x7E


@pytest.mark.parametrize("k", [0, -20, 30, -110])
def test_exact_round_trip_every_e2m1_x_e4m3_value(k):
    """Every positive finite E4M3 scale with every one of the 16 codes comes
    back bit-exact: codes, scales, and the dequantized values."""
    scales = _e4m3_positive_finite()
    p2k = np.float32(2.0 ** k)
    rows = []
    want_codes = []
    # row 0 carries the tensor amax 2688 * 2^k, so g = 2^k exactly
    row0 = np.zeros(16, np.float32)
    row0[0] = np.float32(2688.0) * p2k
    rows.append(row0)
    want_codes.append(None)
    order = [7] + [c for c in range(16) if c != 7]   # code 7 (6.0) forces t = dec(s)
    for s in scales:
        ds = oracle.e4m3_value(s)
        row = np.array([oracle.e2m1_value(c) * ds * 2.0 ** k for c in order], np.float64)
        assert np.all(row.astype(np.float32).astype(np.float64) == row)
        rows.append(row.astype(np.float32))
        want_codes.append(order)
    x = np.stack(rows)
    q = oracle.quantize(x)
    assert float(q.g) == 2.0 ** k
    assert q.scales[0, 0] == 0x7E
    for i, s in enumerate(scales, start=1):
        assert q.scales[i, 0] == s
        codes = [(q.codes[i, j // 2] >> (4 * (j % 2))) & 15 for j in range(16)]
        assert codes == want_codes[i]
    y = oracle.dequantize(q)
    assert np.array_equal(y.view(np.uint32), x.view(np.uint32))   # bit-for-bit, signed zeros too


def _block_view(x):
    return x.reshape(x.shape[0], -1, 16)


@pytest.fixture(scope="module")
def random_case():
    rng = np.random.default_rng(99)
    x = rng.standard_normal((48, 256)).astype(np.float32)
    x[rng.random(x.shape) < 0.01] *= 50
    x[3, 16:32] = 0.0                                  # an all-zero block
    x[5, 32:48] *= 1e-3                                # a tiny block
    x[7, :16] = -x[7, :16]
    return x


def test_scales_are_nearest_e4m3_with_even_ties(random_case):
    """Brute force: each scale byte is the E4M3 value nearest to
    t = bamax/(6g) among all finite non-negative codes (ties to even)."""
    x = random_case
    q = oracle.quantize(x)
    g = np.float32(np.abs(x).max() / np.float32(2688.0))
    assert q.g == g
    bamax = np.abs(_block_view(x)).max(axis=2)
    t = (bamax / np.float32(6.0 * g)).astype(np.float32)
    table = torch.arange(0x7F, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    for (r, b), tv in np.ndenumerate(t):
        err = np.abs(table - float(tv))
        best = np.flatnonzero(err == err.min())
        want = best[0] if len(best) == 1 else best[best % 2 == 0][0]
        if tv >= 448:
            want = 0x7E
        assert q.scales[r, b] == want, (r, b, tv)


def test_codes_are_nearest_grid_points(random_case, facts):
    """Brute force over all 16 codes: each code minimises |e - v|
    (ties to the even magnitude index, saturation at +-6)."""
    grid = np.array(facts["e2m1"]["non_negative_grid"])
    x = random_case
    q = oracle.quantize(x)
    codes = np.stack([q.codes & 15, q.codes >> 4], axis=-1).reshape(x.shape)
    sv = oracle.e4m3_value_array(q.scales)
    for r in range(x.shape[0]):
        for c in range(x.shape[1]):
            d = np.float32(np.float32(sv[r, c // 16]) * q.g)
            if d == 0:
                assert codes[r, c] == 0
                continue
            v = np.float32(x[r, c] * np.float32(np.float32(1.0) / d))
            a = min(abs(float(v)), 6.0)
            err = np.abs(grid - a)
            cand = np.flatnonzero(err == err.min())
            mag = cand[0] if len(cand) == 1 else cand[cand % 2 == 0][0]
            sign = 8 if np.signbit(v) else 0
            assert codes[r, c] == (sign | mag), (r, c, v)


def test_element_step_multiplies_by_the_rounded_reciprocal():
    """The element step is v = fl32(x * fl32(1/d)) (one correctly rounded
    reciprocal per block, then a multiply), not x / d: on vector A of
    reading_vectors the two readings round the same x to different E2M1
    codes."""
    (a, ga), *_ = reading_vectors.vectors()
    f = np.float32
    x, d = a[0, 17], ga                                  # block 1 scale is E4M3 1.0: d = g
    assert f(x / d) == f(2.5)                            # exact quotient: a tie -> even index (2.0)
    assert f(x * (f(1) / d)) > f(2.5)                    # the reciprocal reading: above the tie -> 3.0
    q = oracle.quantize(a)
    assert q.g == ga and q.scales[0, 1] == 0x38
    assert q.codes[0, 8] == 0x57                         # 6g -> 6.0 (7), 2.5g -> 3.0 (5)
    assert q.codes[0, 9] == 0x0D                         # -2.5g -> -3.0


def test_block_scale_is_a_correctly_rounded_quotient():
    """The block scale is E4M3_rne(fl32(bamax / fl32(6g))), a correctly rounded
    division: on vector B the quotient is exactly the E4M3 midpoint 1.0625,
    which ties to the even code 1.0 (0x38); a reciprocal-multiply form would
    give 1.0625001 and the code 1.125 (0x39)."""
    _, (b, gb), *_ = reading_vectors.vectors()
    f = np.float32
    six_g = f(6) * gb
    assert f(b[0, 16] / six_g) == f(1.0625)
    assert f(b[0, 16] * (f(1) / six_g)) > f(1.0625)
    q = oracle.quantize(b)
    assert q.g == gb
    assert q.scales[0, 1] == 0x38


def test_block_scale_divides_by_the_rounded_six_g():
    """The divisor of the block-scale quotient is fl32(6g), rounded before the
    division: on vector C, 6g is half an ulp below fl32(6g), and only the
    rounded divisor puts the quotient exactly on the E4M3 midpoint 1.0625."""
    _, _, (c, gc), _ = reading_vectors.vectors()
    f = np.float32
    six_g = f(6) * gc
    assert Fraction(float(six_g)) - 6 * Fraction(float(gc)) > 0            # fl32(6g) was rounded up
    assert f(c[0, 16] / six_g) == f(1.0625)
    assert f(float(Fraction(float(c[0, 16])) / (6 * Fraction(float(gc))))) > f(1.0625)
    q = oracle.quantize(c)
    assert q.g == gc
    assert q.scales[0, 1] == 0x38


def test_element_reciprocal_is_of_the_rounded_d():
    """d = fl32(dec(s) * g) is rounded before its reciprocal is taken: on
    vector D, x * fl32(1/d) is exactly the E2M1 midpoint 2.5 (code 2.0), while
    the reciprocal of the unrounded dec(s) * g would give 2.5000002 (3.0)."""
    *_, (dv, gd) = reading_vectors.vectors()
    f = np.float32
    x = dv[0, 17]
    d = f(f(1.125) * gd)
    assert Fraction(float(d)) != Fraction(9, 8) * Fraction(float(gd))       # d was rounded
    assert f(x * (f(1) / d)) == f(2.5)
    assert f(x * f(float(1 / (Fraction(9, 8) * Fraction(float(gd)))))) > f(2.5)
    q = oracle.quantize(dv)
    assert q.g == gd and q.scales[0, 1] == 0x39                             # E4M3 1.125
    assert q.codes[0, 8] == 0x47                                            # 6.0 (7), 2.0 (4)
    assert q.codes[0, 9] == 0x0C                                            # -2.0


def test_dequantize_rounds_the_scaled_code_before_g():
    """Dequantize order: y = fl32(fl32(e * dec(s)) * g), the first product
    exact.  With e = 3, dec(s) = 4.5 (0x49) and g = 0.5201722979545593 that is
    fl32(13.5 g) = 7.022326; the other order, fl32(e * fl32(dec(s) * g)),
    gives 7.0223255."""
    f = np.float32
    g = f(0.5201722979545593)
    codes = np.zeros((1, 8), np.uint8)
    codes[0, 0] = 0x05                                   # element 0: +3.0
    q = oracle.Quantized(codes, np.array([[0x49]], np.uint8), g, 1, 16)
    y = oracle.dequantize(q)
    assert y[0, 0] == f(f(13.5) * g)
    assert y[0, 0] != f(f(3) * f(f(4.5) * g))
    assert (y[0, 1:] == 0).all()


def test_code_magnitudes_bounded_by_six(random_case):
    q = oracle.quantize(random_case * 1e3)
    nibbles = np.concatenate([q.codes & 15, q.codes >> 4]).ravel()
    mags = np.array([abs(oracle.e2m1_value(c)) for c in range(16)])
    assert mags[nibbles].max() <= 6.0
    assert mags[nibbles].max() == 6.0        # the tensor amax reaches the top code


def test_quantization_error_bound(random_case, facts):
    """|x - deq| <= half the local grid gap times d, except where |v| > 6
    saturates (then the error is |x| - 6d)."""
    grid = np.array(facts["e2m1"]["non_negative_grid"])
    gaps = np.diff(grid)
    x = random_case
    q = oracle.quantize(x)
    y = oracle.dequantize(q).astype(np.float64)
    d = (oracle.e4m3_value_array(q.scales) * float(q.g)).repeat(16, axis=1)
    ax = np.abs(x.astype(np.float64))
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(d > 0, ax / d, 0)
    idx = np.clip(np.searchsorted(grid, v, side="right") - 1, 0, 6)
    half_gap = np.where(v >= 6, 0, gaps[idx] / 2)
    bound = half_gap * d + np.where(v >= 6, ax - 6 * d, 0)
    # the fp32 reciprocal and product add at most a few ulps of |x|
    slack = 4 * np.finfo(np.float32).eps * ax + 1e-30
    assert np.all(np.abs(ax - np.abs(y)) <= bound + slack)


def test_block_granularity(random_case):
    """Changing one element (without changing the tensor amax) changes only
    the scale and codes of its own 16-element block."""
    x = random_case.copy()
    q0 = oracle.quantize(x)
    r, c = 10, 37
    x[r, c] = x[r, c] * 0.5 + 0.75
    assert np.abs(x).max() == np.abs(random_case).max()
    q1 = oracle.quantize(x)
    changed_s = np.argwhere(q0.scales != q1.scales)
    changed_c = np.argwhere(q0.codes != q1.codes)
    assert all((rr, bb) == (r, c // 16) for rr, bb in changed_s)
    assert all(rr == r and bb // 8 == c // 16 for rr, bb in changed_c)
    assert len(changed_c) > 0


def test_amax_change_moves_every_block(random_case):
    x = random_case.copy()
    q0 = oracle.quantize(x)
    x[0, 0] = np.abs(x).max() * 4
    q1 = oracle.quantize(x)
    assert q1.g == np.float32(q0.g * 0 + x[0, 0] / np.float32(2688.0))
    assert (q0.scales != q1.scales).mean() > 0.9


def test_zero_tensor_and_zero_blocks():
    x = np.zeros((4, 64), np.float32)
    x[1, 20] = -0.0
    q = oracle.quantize(x)
    assert q.g == 0.0
    assert not q.scales.any() and not q.codes.any()
    assert not oracle.dequantize(q).any()


def test_tiny_magnitudes_follow_zero_block_rule():
    """amax so small that block scales round to zero or 1/d overflows: those
    blocks are zero-scale blocks with all codes 0; other blocks stay exact."""
    x = np.zeros((3, 32), np.float32)
    x[0, 0] = np.float32(2688 * 2.0 ** -120)          # g = 2^-120
    x[0, 16] = np.float32(2.0 ** -134)                # t = 2^-134/(6*2^-120) << 2^-10 -> s = 0
    x[1, 0] = np.float32(-3.0 * 2.0 ** -130)
    x[2, 5] = np.float32(-1e-38)                      # t ~ 0.0022 -> s = 2^-9 (0x01), d = 2^-129:
    q = oracle.quantize(x)                            # a non-zero d with no finite fp32 reciprocal
    assert q.g == np.float32(2.0 ** -120)
    assert q.scales[0, 1] == 0 and q.codes[0, 8:16].tolist() == [0] * 8
    with np.errstate(over="ignore"):
        assert np.isinf(np.float32(1) / (np.float32(2.0 ** -9) * q.g))
    assert q.scales[2, 0] == 0x01 and q.codes[2, 0:8].tolist() == [0] * 8
    y = oracle.dequantize(q)
    assert y[0, 0] == x[0, 0]
    assert y[0, 16] == 0.0 and y[2, 5] == 0.0


def test_negative_values_rounding_to_zero_keep_sign():
    x = np.zeros((1, 16), np.float32)
    x[0, 0] = 6.0
    x[0, 1] = -0.1
    x[0, 2] = -0.0
    x[0, 3] = 0.1
    q = oracle.quantize(x)
    codes = [(q.codes[0, j // 2] >> (4 * (j % 2))) & 15 for j in range(4)]
    assert codes == [7, 8, 8, 0]


def test_storage_accounting_matches_page(facts):
    nv = facts["nvfp4"]
    for rows, cols in [(8192, 5120), (17408, 5120), (64, 256)]:
        bits = oracle.storage_bytes(rows, cols) * 8 / (rows * cols)
        # 4 bits per code + 8 bits per 16-value block, plus the one fp32 scale
        assert bits == nv["bits_per_value"] + 32 / (rows * cols)
        assert round(bits, 2) == nv["bits_per_value"]
        assert round(16 / bits, 1) in (3.5, 3.6)      # "about 3.5x" vs FP16
        assert round(8 / bits, 1) == nv["smaller_than_fp8"]
    mx = facts["mxfp4"]
    assert (mx["block"] * 4 + 8) / mx["block"] == mx["bits_per_value"]
    q = oracle.quantize(np.ones((64, 256), np.float32))
    assert q.codes.nbytes + q.scales.nbytes + 4 == oracle.storage_bytes(64, 256)


def test_bf16_widening_is_exact():
    x = np.array([1.0, -2.5, 3.140625, 1e-30, 6e4], np.float32)
    bits = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    back = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(oracle.bf16_bits_to_f32(bits), back)


# ---------------------------------------------------------------------------
# GEMM
# ---------------------------------------------------------------------------

@pytest.fixture(scope="module")
def tiny_q():
    w = workloads.make("tiny")
    return oracle.quantize(w["X"]), oracle.quantize(w["W"])


def _exact_deq(q):
    """Dequantized operand as exact rationals, from the page grid and an
    independent E4M3 decoder (torch)."""
    e4 = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    grid = [0, Fraction(1, 2), 1, Fraction(3, 2), 2, 3, 4, 6]
    g = Fraction(float(q.g))
    out = []
    for r in range(q.rows):
        row = []
        for c in range(q.cols):
            byte = int(q.codes[r, c // 2])
            code = (byte >> 4) if c % 2 else (byte & 15)
            e = grid[code & 7] * (-1 if code & 8 else 1)
            row.append(e * Fraction(float(e4[q.scales[r, c // 16]])) * g)
        out.append(row)
    return out


def test_gemm_f64_against_exact_rationals(tiny_q):
    xq, wq = tiny_q
    y = oracle.gemm_f64(xq, wq)
    assert y.shape == (16, 64)
    A, B = _exact_deq(xq), _exact_deq(wq)
    for m in range(16):
        for n in range(0, 64, 3):
            exact = sum(a * b for a, b in zip(A[m], B[n]))
            mag = sum(abs(a * b) for a, b in zip(A[m], B[n]))
            assert abs(Fraction(y[m, n]) - exact) <= Fraction(1e-12) * (mag + 1)


def test_gemm_transpose_convention(tiny_q):
    """Y = X W^T: entry (m, n) pairs row m of X with row n of W, not column."""
    xq, wq = tiny_q
    y = oracle.gemm_f64(xq, wq)
    dx = oracle.dequantize_f64(xq)
    dw = oracle.dequantize_f64(wq)
    np.testing.assert_allclose(y, dx @ dw.T, rtol=1e-12, atol=1e-12)
    e, na, nb = oracle.gemm_entries(xq, wq, [0, 5, 15], [63, 0, 17])
    np.testing.assert_allclose(e, y[[0, 5, 15], [63, 0, 17]], rtol=1e-13, atol=0)
    np.testing.assert_allclose(na, np.linalg.norm(dx[[0, 5, 15]], axis=1), rtol=1e-12)
    np.testing.assert_allclose(nb, np.linalg.norm(dw[[63, 0, 17]], axis=1), rtol=1e-12)


def test_gemm_closed_form_constant_operands():
    # constant 2688 -> g = 1, every block scale 448, every code 6.0;
    # constant -5376 -> g = 2, scale 448, code -6.0: Y = K * 2688 * (-5376)
    a = oracle.quantize(np.full((3, 128), 2688.0, np.float32))
    b = oracle.quantize(np.full((5, 128), -5376.0, np.float32))
    assert (a.g, b.g) == (1.0, 2.0)
    assert (a.scales == 0x7E).all() and (b.scales == 0x7E).all()
    assert (a.codes == 0x77).all() and (b.codes == 0xFF).all()
    np.testing.assert_array_equal(oracle.gemm_f64(a, b), np.full((3, 5), -128 * 2688.0 * 5376.0))
    # all ones: every element dequantizes to the same d = 6*448*g, so
    # Y = K * dA * dB up to fp64 summation rounding
    a1 = oracle.quantize(np.ones((2, 256), np.float32))
    d1 = Fraction(6) * Fraction(448) * Fraction(float(a1.g))
    y1 = oracle.gemm_f64(a1, a1)
    exact = 256 * d1 * d1
    assert abs(Fraction(y1[0, 1]) - exact) <= exact * Fraction(1e-14)


# ---------------------------------------------------------------------------
# SiLU * up
# ---------------------------------------------------------------------------

def test_silu_mul_identities():
    z = np.linspace(-30, 30, 601)
    one = np.ones_like(z)
    s = oracle.silu_mul_f64(z, one)
    s_neg = oracle.silu_mul_f64(-z, one)
    np.testing.assert_allclose(s - s_neg, z, rtol=0, atol=1e-12)     # z*sig(z) - (-z)*sig(-z) = z
    assert oracle.silu_mul_f64(np.array([0.0]), np.array([5.0]))[0] == 0.0
    np.testing.assert_allclose(oracle.silu_mul_f64(np.array([40.0]), np.array([1.0])), [40.0], rtol=1e-15)
    np.testing.assert_allclose(oracle.silu_mul_f64(np.array([1.0]), np.array([3.0])),
                               [3.0 / (1.0 + math.exp(-1.0))], rtol=1e-15)
    u = np.linspace(-2, 2, 601)
    np.testing.assert_allclose(oracle.silu_mul_f64(z, u), s * u, rtol=1e-15)


# ---------------------------------------------------------------------------
# Workload generator (shared by the oracle and the CUDA path)
# ---------------------------------------------------------------------------

def test_workload_generator_is_seeded_and_shaped():
    a = workloads.make("tiny")
    b = workloads.make("tiny")
    assert a["X"].shape == (16, 256) and a["W"].shape == (64, 256)
    np.testing.assert_array_equal(a["X"], b["X"])
    assert (np.abs(a["X"]) == 40).sum() == 4 and (np.abs(a["W"]) == 40).sum() == 4
    d = workloads.make("decode", N=256, K=512)
    assert d["X"].dtype == np.uint16 and d["X"].shape == (8, 512)
    x = oracle.bf16_bits_to_f32(d["X"])
    assert (np.abs(x) > 10).sum() >= 1
