"""GPU parity of the quantizer and dequantizer against the CPU oracle:
packed codes, tiled scales (padding included) and the tensor scale must be
bit-exact."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import reading_vectors
from gpu_helpers import (assert_quantized_equal, bf16_tensor, f32_tensor, tiled_scales)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import nvfp4_block_scaled_21_b200 as nv
    return nv


def quantize_gpu(nv, x_dev, ld=None):
    rows, cols = x_dev.shape
    if ld is not None and ld != cols:
        buf = torch.zeros((rows, ld), dtype=x_dev.dtype, device=x_dev.device)
        buf[:, :cols] = x_dev
        x_dev = buf[:, :cols]
    out = nv.NVFP4Tensor.empty(rows, cols)
    ws = nv.workspace(nv.OP_QUANTIZE, rows, 0, cols)
    nv.nvfp4_quantize(x_dev, out, ws)
    return out


def test_worked_example(nv, golden_dir):
    with open(os.path.join(golden_dir, "worked_example_1x32.json")) as f:
        ex = json.load(f)
    x = np.array([float(v) for v in ex["x"]], np.float32).reshape(1, 32)
    out = quantize_gpu(nv, f32_tensor(x))
    torch.cuda.synchronize()
    assert [f"{b:02x}" for b in out.codes.cpu().numpy()[0]] == ex["packed_bytes_hex"]
    sc = out.scales.cpu().numpy()
    assert [f"{sc[0]:02x}", f"{sc[1]:02x}"] == ex["scales_hex"]
    assert out.tensor_scale[0].item() == float(ex["g"])
    assert_quantized_equal(out, oracle.quantize(x))


@pytest.mark.parametrize("k", [0, -20, 30])
def test_round_trip_every_representable_value(nv, k):
    """Every positive finite E4M3 scale with all 16 codes (same construction
    as the oracle pin) gives the same bytes on the GPU."""
    rows = [np.zeros(16, np.float32)]
    rows[0][0] = np.float32(2688.0 * 2.0 ** k)
    order = [7] + [c for c in range(16) if c != 7]
    for s in range(1, 0x7F):
        ds = oracle.e4m3_value(s)
        rows.append(np.array([oracle.e2m1_value(c) * ds * 2.0 ** k for c in order], np.float32))
    x = np.stack(rows)
    assert_quantized_equal(quantize_gpu(nv, f32_tensor(x)), oracle.quantize(x))
    # the bf16 path sees the same values (all of them are exact in bf16)
    xb = torch.from_numpy(x).to(torch.bfloat16)
    assert torch.equal(xb.float(), torch.from_numpy(x))
    assert_quantized_equal(quantize_gpu(nv, xb.cuda()), oracle.quantize(x))


def _rand(rows, cols, seed, outliers=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols)).astype(np.float32)
    if outliers:
        m = rng.random(x.shape) < 1e-3
        x[m] = (rng.standard_normal(m.sum()) * 50).astype(np.float32)
    return x


SHAPES = [(1, 16), (2, 48), (3, 80), (17, 1040), (129, 64), (300, 640), (257, 5120)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_quantize_parity(nv, shape, dtype):
    x = _rand(*shape, seed=shape[0] * 7 + shape[1])
    if dtype == "bf16":
        xt = torch.from_numpy(x).to(torch.bfloat16)
        bits = xt.view(torch.int16).numpy().view(np.uint16)
        q = oracle.quantize(bits)
        xd = xt.cuda()
    else:
        q = oracle.quantize(x)
        xd = f32_tensor(x)
    assert_quantized_equal(quantize_gpu(nv, xd), q)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_quantize_row_pitch(nv, dtype):
    x = _rand(37, 96, seed=5)
    xd = f32_tensor(x) if dtype == "f32" else f32_tensor(x).to(torch.bfloat16)
    ref = oracle.quantize(x if dtype == "f32" else xd.cpu().view(torch.int16).numpy().view(np.uint16))
    assert_quantized_equal(quantize_gpu(nv, xd, ld=160), ref)


def test_quantize_edge_cases(nv):
    # all zeros, including a negative zero
    z = np.zeros((5, 32), np.float32)
    z[2, 3] = -0.0
    assert_quantized_equal(quantize_gpu(nv, f32_tensor(z)), oracle.quantize(z))
    # zero-scale blocks next to normal ones; tiny amax
    t = np.zeros((3, 48), np.float32)
    t[0, 0] = np.float32(2688 * 2.0 ** -120)
    t[0, 16] = np.float32(2.0 ** -134)
    t[1, 0] = np.float32(-3.0 * 2.0 ** -130)
    t[2, 5] = np.float32(-1e-38)
    assert_quantized_equal(quantize_gpu(nv, f32_tensor(t)), oracle.quantize(t))
    # negative values that round to zero keep their sign; exact E2M1 ties
    s = np.zeros((1, 32), np.float32)
    s[0, :16] = [6, -0.1, -0.0, 0.1, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, -5, -0.25, 7, -7, 0]
    s[0, 16:] = np.linspace(-3, 3, 16)
    assert_quantized_equal(quantize_gpu(nv, f32_tensor(s)), oracle.quantize(s))
    # a single huge value: every other block's scale underflows towards zero
    h = _rand(4, 64, seed=9, outliers=False)
    h[0, 0] = 3e38
    assert_quantized_equal(quantize_gpu(nv, f32_tensor(h)), oracle.quantize(h))


def test_block_scale_ties_and_boundaries(nv):
    """Blocks whose quotient bamax/(6g) lands exactly on an E4M3 rounding
    midpoint (ties to even), one ulp either side of it, and on E4M3 values:
    the kernel's fast scale path must hand these to its exact division."""
    vals = [oracle.e4m3_value(c) for c in range(0x7F)]
    mids = [(a + b) / 2 for a, b in zip(vals[:-1], vals[1:])]
    rows = [np.zeros(16, np.float32)]
    rows[0][0] = np.float32(2688.0)                        # g = 1 exactly
    for m in mids + vals[1:]:
        for nudge in (0, -1, 1):
            t = np.float32(m)
            if nudge:
                t = np.nextafter(t, np.float32(nudge * 1e9))
            bamax = np.float32(np.float64(t) * 6.0)        # 6 t is exact in fp32 for these t
            if np.float64(bamax) != np.float64(t) * 6.0 or t > 448:
                continue                                   # keep the tensor amax at 2688
            row = np.linspace(-1, 1, 16).astype(np.float32) * bamax
            row[3] = bamax
            rows.append(row)
    x = np.stack(rows)
    assert_quantized_equal(quantize_gpu(nv, f32_tensor(x)), oracle.quantize(x))


def test_quotient_reading_vectors(nv):
    """The four rows of reading_vectors, where a different formation of the
    block-scale or element quotient would change a scale byte or a code: the
    GPU agrees with the oracle bit for bit (vectors B and C also take the
    encode pass's exact-division fallback for the block scale)."""
    for x, g in reading_vectors.vectors():
        q = quantize_gpu(nv, f32_tensor(x))
        qo = oracle.quantize(x)
        assert qo.g == g
        assert_quantized_equal(q, qo)


@pytest.mark.parametrize("shape", [(0, 64), (5, 0), (0, 0)])
def test_quantize_empty(nv, shape):
    """An empty tensor has no codes and no scale bytes; its amax is 0, so g = 0
    (written even though nothing else is)."""
    out = nv.NVFP4Tensor.empty(*shape)
    out.tensor_scale.fill_(7.0)
    x = torch.zeros(shape, device="cuda")
    nv.nvfp4_quantize(x, out, nv.workspace(nv.OP_QUANTIZE, shape[0], 0, shape[1]))
    torch.cuda.synchronize()
    assert out.tensor_scale[0].item() == 0.0


def test_quantize_full_size_quantize_workload(nv):
    """The 8192x5120 bf16 quantize workload (seed 1), launched exactly as the
    benchmark launches it, bit-exact over the whole tensor."""
    from nvfp4_block_scaled_21_b200 import workloads
    w = workloads.make("quantize")
    q = oracle.quantize(w["X"])
    assert_quantized_equal(quantize_gpu(nv, bf16_tensor(w["X"])), q)


@pytest.mark.parametrize("shape", [(1, 16), (7, 96), (130, 320)])
def test_dequantize_parity(nv, shape):
    x = _rand(*shape, seed=11)
    q = oracle.quantize(x)
    ref = oracle.dequantize(q)
    t = nv.NVFP4Tensor.empty(*shape)
    t.codes.copy_(torch.from_numpy(q.codes))
    t.scales.copy_(torch.from_numpy(tiled_scales(q.scales)))
    t.tensor_scale[0] = float(q.g)
    y = torch.empty(shape, dtype=torch.float32, device="cuda")
    nv.nvfp4_dequantize(t, y)
    got = y.cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    yb = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    nv.nvfp4_dequantize(t, yb)
    assert torch.equal(yb.cpu(), torch.from_numpy(ref).to(torch.bfloat16))


def test_dequantize_rounding_order(nv):
    """y = fl32(fl32(e * dec(s)) * g): e = 3 with dec(s) = 4.5 and
    g = 0.5201722979545593 is a value where the other order of the two
    roundings gives a different fp32 result; every code with that scale and g."""
    f = np.float32
    codes = np.array([[(2 * j) | ((2 * j + 1) << 4) for j in range(8)]], np.uint8)   # codes 0..15
    q = oracle.Quantized(codes, np.array([[0x49]], np.uint8), f(0.5201722979545593), 1, 16)
    ref = oracle.dequantize(q)
    assert ref[0, 5] == f(f(13.5) * q.g)
    t = nv.NVFP4Tensor.empty(1, 16)
    t.codes.copy_(torch.from_numpy(q.codes))
    t.scales.copy_(torch.from_numpy(tiled_scales(q.scales)))
    t.tensor_scale[0] = float(q.g)
    y = torch.empty((1, 16), dtype=torch.float32, device="cuda")
    nv.nvfp4_dequantize(t, y)
    assert np.array_equal(y.cpu().numpy().view(np.uint32), ref.view(np.uint32))


# The one-read cooperative quantizer (contiguous x, cols % 64 == 0, at least
# 8 MB): all of a CTA's slice on chip (16 MB bf16), a slice that spills past
# shared memory and registers and is read again (84 MB bf16), fp32 input with
# rows not a multiple of 128 (padding rows of the scale layout), and a small
# column count.  Bit-exact against the oracle and against the two-pass
# quantizer (NVFP4_QUANTIZE_ONEPASS=0).
@pytest.mark.parametrize("rows,cols,dtype", [(2048, 4096, torch.bfloat16), (8192, 5120, torch.bfloat16),
                                             (1000, 4096, torch.float32), (3000, 1536, torch.bfloat16)])
def test_quantize_onepass(nv, rows, cols, dtype, monkeypatch):
    rng = np.random.default_rng(rows + cols)
    x = rng.standard_normal((rows, cols)).astype(np.float32)
    x[rng.random(x.shape) < 1e-3] *= 50
    if dtype == torch.bfloat16:
        xt = torch.from_numpy(x).to(torch.bfloat16)
        x_or = xt.view(torch.int16).numpy().view(np.uint16)
    else:
        xt, x_or = torch.from_numpy(x), x
    xd = xt.cuda()
    outs = []
    for onepass in ("1", "0"):
        monkeypatch.setenv("NVFP4_QUANTIZE_ONEPASS", onepass)
        out = nv.NVFP4Tensor.empty(rows, cols)
        out.codes.fill_(0x77)
        out.scales.fill_(0x55)
        ws = nv.workspace(nv.OP_QUANTIZE, rows, 0, cols)
        nv.nvfp4_quantize(xd, out, ws)
        assert nv.nvfp4_get_device_status(ws) == nv.OK
        outs.append(out)
    torch.cuda.synchronize()
    assert torch.equal(outs[0].codes, outs[1].codes)
    assert torch.equal(outs[0].scales, outs[1].scales)
    assert torch.equal(outs[0].tensor_scale, outs[1].tensor_scale)
    assert_quantized_equal(outs[0], oracle.quantize(x_or))


# Small tensors (at most 32 x 256 blocks of 16) take one cooperative launch
# of a few CTAs that meet once for the tensor amax; NVFP4_QUANTIZE_MEET=0
# keeps them on the two passes.  Both bit-exact against the oracle, on shapes
# with partial scale words (cols % 64 != 0), padding rows, a row pitch wider
# than cols, and the largest size the cooperative form takes.
@pytest.mark.parametrize("rows,cols,dtype,ld", [(7, 96, torch.float32, None), (33, 80, torch.bfloat16, 96),
                                                (130, 320, torch.bfloat16, None), (8, 5120, torch.bfloat16, None),
                                                (16, 8192, torch.float32, None), (1, 16, torch.bfloat16, None)])
def test_quantize_small_cooperative_and_two_pass(nv, rows, cols, dtype, ld, monkeypatch):
    rng = np.random.default_rng(rows * 7 + cols)
    x = rng.standard_normal((rows, cols)).astype(np.float32)
    x[rng.random(x.shape) < 2e-3] *= 50
    if dtype == torch.bfloat16:
        xt = torch.from_numpy(x).to(torch.bfloat16)
        x_or = xt.view(torch.int16).numpy().view(np.uint16)
    else:
        xt, x_or = torch.from_numpy(x), x
    want = oracle.quantize(x_or)
    for meet in ("1", "0"):
        monkeypatch.setenv("NVFP4_QUANTIZE_MEET", meet)
        out = quantize_gpu(nv, xt.cuda(), ld)
        assert_quantized_equal(out, want)
