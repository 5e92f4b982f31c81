"""GPU parity of the W4A4 block-scaled GEMM against the fp64 oracle.

Each case quantizes the same seeded inputs on both sides (the GPU with its own
kernels, the oracle with its own code; quantization is bit-exact, tested
separately), runs the GPU GEMM, and compares every output (small cases) or
sampled outputs (full sizes) with the fp64 dot products of the dequantized
operands, within max relative error 2e-3 and the absolute floor
1e-3 * |row A| * |row B| / sqrt(K) (plus 2^-8 relative for a bf16 output)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (assert_gemm_close, assert_quantized_equal, bf16_tensor, f32_tensor,
                         to_numpy_f64, upload)
from nvfp4_block_scaled_21_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import nvfp4_block_scaled_21_b200 as nv
    return nv


def quantize_gpu(nv, x):
    out = nv.NVFP4Tensor.empty(*x.shape)
    nv.nvfp4_quantize(x, out, nv.workspace(nv.OP_QUANTIZE, x.shape[0], 0, x.shape[1]))
    return out


def run_gemm(nv, a, b, out_dtype, ws=None):
    # rows of y must start on 16-byte boundaries: pad the pitch (always by at
    # least one 16-byte unit, so that writes past N would be seen), then slice
    per16 = 16 // torch.empty((), dtype=out_dtype).element_size()
    ldy = -(-b.rows // per16) * per16 + per16
    buf = torch.full((a.rows, ldy), float("nan"), dtype=out_dtype, device="cuda")
    y = buf[:, :b.rows]
    if ws is None:
        ws = nv.workspace(nv.OP_GEMM, a.rows, b.rows, a.cols)
    nv.nvfp4_gemm(a, b, y, ws)
    assert nv.nvfp4_get_device_status(ws) == nv.OK
    assert torch.isnan(buf[:, b.rows:].float()).all()      # nothing written past N
    return y


def norms(q):
    return np.linalg.norm(oracle.dequantize_f64(q), axis=1)


def test_tiny_workload(nv):
    """X fp32 16x256, W fp32 64x256 (seed 0), Y = X W^T in fp32."""
    w = workloads.make("tiny")
    xq_o, wq_o = oracle.quantize(w["X"]), oracle.quantize(w["W"])
    xq, wq = quantize_gpu(nv, f32_tensor(w["X"])), quantize_gpu(nv, f32_tensor(w["W"]))
    assert_quantized_equal(xq, xq_o)
    assert_quantized_equal(wq, wq_o)
    y = run_gemm(nv, xq, wq, torch.float32)
    ref = oracle.gemm_f64(xq_o, wq_o)
    assert_gemm_close(to_numpy_f64(y), ref, norms(xq_o)[:, None], norms(wq_o)[None, :], 256, False, "tiny")


CASES = [
    # (M, N, K): swapped (M <= 64) with MMA N = 16 / 32 / 64, and unswapped
    # (M > 64) with 128-wide tiles; ragged M and N tails, K with a partial
    # last 256-column slab.
    (1, 64, 64), (8, 200, 320), (13, 384, 1024), (16, 1000, 192), (17, 130, 256),
    (33, 256, 576), (64, 129, 512), (65, 300, 256), (128, 512, 1280), (200, 384, 320),
    (300, 1000, 640),
]


@pytest.mark.parametrize("M,N,K", CASES)
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_gemm_parity(nv, M, N, K, out):
    rng = np.random.default_rng(M * 1000 + N + K)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[rng.random(x.shape) < 1e-3] *= 50
    wt = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    xq_o, wq_o = oracle.quantize(x), oracle.quantize(wt)
    xq, wq = quantize_gpu(nv, f32_tensor(x)), quantize_gpu(nv, f32_tensor(wt))
    dt = torch.bfloat16 if out == "bf16" else torch.float32
    y = run_gemm(nv, xq, wq, dt)
    ref = oracle.gemm_f64(xq_o, wq_o)
    assert_gemm_close(to_numpy_f64(y), ref, norms(xq_o)[:, None], norms(wq_o)[None, :], K,
                      out == "bf16", f"gemm {M}x{N}x{K}")


def test_gemm_from_oracle_operands(nv):
    """The GEMM fed the oracle's own codes and scales (uploaded in the tiled
    layout) agrees with the oracle: pins the nibble order and the scale layout
    the tensor cores read, independently of the GPU quantizer."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((40, 512)).astype(np.float32)
    wt = rng.standard_normal((256, 512)).astype(np.float32)
    xq_o, wq_o = oracle.quantize(x), oracle.quantize(wt)
    y = run_gemm(nv, upload(xq_o, nv), upload(wq_o, nv), torch.float32)
    ref = oracle.gemm_f64(xq_o, wq_o)
    assert_gemm_close(to_numpy_f64(y), ref, norms(xq_o)[:, None], norms(wq_o)[None, :], 512, False, "oracle operands")


def test_gemm_wide_tiles(nv):
    """Enough tiles to take the 128x256 tile path, sampled outputs."""
    M, N, K = 2304, 4608, 256
    rng = np.random.default_rng(21)
    x = rng.standard_normal((M, K)).astype(np.float32)
    wt = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    xq_o, wq_o = oracle.quantize(x), oracle.quantize(wt)
    y = run_gemm(nv, quantize_gpu(nv, f32_tensor(x)), quantize_gpu(nv, f32_tensor(wt)), torch.bfloat16)
    yc = to_numpy_f64(y)
    ms = np.concatenate([rng.integers(0, M, 3000), np.full(N, M - 1)])
    ns = np.concatenate([rng.integers(0, N, 3000), np.arange(N)])
    ref, na, nb = oracle.gemm_entries(xq_o, wq_o, ms, ns)
    assert_gemm_close(yc[ms, ns], ref, na, nb, K, True, "wide tiles")


@pytest.mark.parametrize("pair", ["0", "1"])
@pytest.mark.parametrize("M,N,K", [(2304, 4608, 256), (2000, 4700, 320), (1900, 4616, 256)])
def test_gemm_cta_pair_tiles(nv, M, N, K, pair, monkeypatch):
    """Shapes large enough for the two-CTA 256x256 tiles (NVFP4_GEMM_CTA_PAIR=0
    keeps them on the one-CTA kernel), including ragged M (the second CTA of
    the last row pair partly or wholly outside), ragged N with and without
    N % 8 == 0 (TMA-store and per-row-store epilogues) and a partial last K
    slab; sampled outputs plus the last row and column, for both kernels."""
    monkeypatch.setenv("NVFP4_GEMM_CTA_PAIR", pair)
    rng = np.random.default_rng(M + N)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[rng.random(x.shape) < 1e-3] *= 50
    wt = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    xq_o, wq_o = oracle.quantize(x), oracle.quantize(wt)
    y = run_gemm(nv, quantize_gpu(nv, f32_tensor(x)), quantize_gpu(nv, f32_tensor(wt)), torch.bfloat16)
    yc = to_numpy_f64(y)
    ms = np.concatenate([rng.integers(0, M, 4000), np.full(N, M - 1), np.arange(M)])
    ns = np.concatenate([rng.integers(0, N, 4000), np.arange(N), np.full(M, N - 1)])
    ref, na, nb = oracle.gemm_entries(xq_o, wq_o, ms, ns)
    assert_gemm_close(yc[ms, ns], ref, na, nb, K, True, f"pair {M}x{N}x{K}")
    assert np.isfinite(yc).all()


def test_gemm_cta_pair_f32_output(nv, monkeypatch):
    """The two-CTA kernel's fp32 epilogue (per-row stores; the TMA-store path
    is bf16 only), with ragged M and N: sampled outputs plus the last row and
    column, and nothing written past N."""
    monkeypatch.setenv("NVFP4_GEMM_CTA_PAIR", "1")
    M, N, K = 2000, 4616, 256
    rng = np.random.default_rng(77)
    x = rng.standard_normal((M, K)).astype(np.float32)
    wt = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    xq_o, wq_o = oracle.quantize(x), oracle.quantize(wt)
    y = run_gemm(nv, quantize_gpu(nv, f32_tensor(x)), quantize_gpu(nv, f32_tensor(wt)), torch.float32)
    yc = to_numpy_f64(y)
    ms = np.concatenate([rng.integers(0, M, 4000), np.full(N, M - 1), np.arange(M)])
    ns = np.concatenate([rng.integers(0, N, 4000), np.arange(N), np.full(M, N - 1)])
    ref, na, nb = oracle.gemm_entries(xq_o, wq_o, ms, ns)
    assert_gemm_close(yc[ms, ns], ref, na, nb, K, False, f"pair f32 {M}x{N}x{K}")
    assert np.isfinite(yc).all()


@pytest.mark.parametrize("M,N,K,dt", [(24, 1000, 1088, torch.bfloat16), (8, 17408, 5120, torch.float32),
                                      (200, 700, 2048, torch.bfloat16), (130, 520, 4096, torch.float32)])
def test_gemm_stream_k(nv, M, N, K, dt):
    """Few output tiles: CTAs split K, partial sums meet in fp32 in the
    workspace and the last contributor of each tile writes it.  Covers the
    swapped (M <= 64) and 128x128 layouts, ragged M and N, bf16 and fp32 out;
    the workspace's scratch starts full of garbage (as another operation may
    have left it) and two calls on it both match the oracle."""
    rng = np.random.default_rng(M * 7 + N)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[rng.random(x.shape) < 1e-3] *= 50
    wt = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    xq_o, wq_o = oracle.quantize(x), oracle.quantize(wt)
    xq, wq = quantize_gpu(nv, f32_tensor(x)), quantize_gpu(nv, f32_tensor(wt))
    ws = nv.workspace(nv.OP_GEMM, M, N, K)
    assert ws.numel() > 256                                  # the shape has stream-K scratch
    ws[256:] = 0x7f                                          # garbage (large finite floats)
    ms = np.concatenate([rng.integers(0, M, 3000), np.full(N, M - 1), np.arange(M)])
    ns = np.concatenate([rng.integers(0, N, 3000), np.arange(N), np.full(M, N - 1)])
    ref, na, nb = oracle.gemm_entries(xq_o, wq_o, ms, ns)
    for call in range(2):
        y = run_gemm(nv, xq, wq, dt, ws=ws)
        yc = to_numpy_f64(y)
        assert np.isfinite(yc).all()
        assert_gemm_close(yc[ms, ns], ref, na, nb, K, dt == torch.bfloat16, f"stream-K {M}x{N}x{K} call {call}")


def test_gemm_special_operands(nv):
    # all-zero activations -> exact zeros; constant operands -> closed form
    z = quantize_gpu(nv, torch.zeros((8, 128), device="cuda"))
    c = quantize_gpu(nv, torch.full((64, 128), -5376.0, device="cuda"))
    y = run_gemm(nv, z, c, torch.float32)
    assert torch.count_nonzero(y) == 0
    a = quantize_gpu(nv, torch.full((3, 128), 2688.0, device="cuda"))
    y = run_gemm(nv, a, c, torch.float32)
    assert torch.all(y == -128 * 2688.0 * 5376.0)


def test_gemm_degenerate_shapes(nv):
    """M = 0 and N = 0 launch nothing and write nothing; K = 0 is an empty
    reduction, so y is all zeros."""
    b = quantize_gpu(nv, torch.randn((40, 64), device="cuda"))
    a0 = nv.NVFP4Tensor.empty(0, 64)
    y0 = torch.empty((0, 40), dtype=torch.bfloat16, device="cuda")
    ws = nv.workspace(nv.OP_GEMM, 0, 40, 64)
    nv.nvfp4_gemm(a0, b, y0, ws)
    a = quantize_gpu(nv, torch.randn((5, 64), device="cuda"))
    b0 = nv.NVFP4Tensor.empty(0, 64)
    buf = torch.full((5, 8), float("nan"), dtype=torch.float32, device="cuda")
    nv.nvfp4_gemm(a, b0, buf[:, :0], nv.workspace(nv.OP_GEMM, 5, 0, 64))
    assert torch.isnan(buf).all()                                # nothing written
    ak, bk = nv.NVFP4Tensor.empty(5, 0), nv.NVFP4Tensor.empty(8, 0)
    yk = torch.full((5, 8), float("nan"), dtype=torch.float32, device="cuda")
    ws = nv.workspace(nv.OP_GEMM, 5, 8, 0)
    nv.nvfp4_gemm(ak, bk, yk, ws)
    torch.cuda.synchronize()
    assert torch.count_nonzero(yk) == 0
    assert nv.nvfp4_get_device_status(ws) == nv.OK


def test_decode_workload_full(nv):
    """M=8, N=17408, K=5120 (seed 2): every output against the fp64 oracle."""
    w = workloads.make("decode")
    xq_o, wq_o = oracle.quantize(w["X"]), oracle.quantize(w["W"])
    wq = quantize_gpu(nv, bf16_tensor(w["W"]))
    assert_quantized_equal(wq, wq_o)
    xq = quantize_gpu(nv, bf16_tensor(w["X"]))
    y = run_gemm(nv, xq, wq, torch.bfloat16)
    ref = oracle.gemm_f64(xq_o, wq_o)
    assert_gemm_close(to_numpy_f64(y), ref, norms(xq_o)[:, None], norms(wq_o)[None, :], 5120, True, "decode")


def test_prefill_workload_sampled(nv):
    """M=4096, N=17408, K=5120 (seed 3) in the benchmark's configuration:
    4096 random outputs plus one full row and one full column."""
    w = workloads.make("prefill")
    xq_o, wq_o = oracle.quantize(w["X"]), oracle.quantize(w["W"])
    xq, wq = quantize_gpu(nv, bf16_tensor(w["X"])), quantize_gpu(nv, bf16_tensor(w["W"]))
    y = run_gemm(nv, xq, wq, torch.bfloat16)
    yc = y.float().cpu().numpy().astype(np.float64)
    rng = np.random.default_rng(0)
    M, N = 4096, 17408
    ms = np.concatenate([rng.integers(0, M, 4096), np.full(N, 1234), np.arange(M)])
    ns = np.concatenate([rng.integers(0, N, 4096), np.arange(N), np.full(M, 17000)])
    ref, na, nb = oracle.gemm_entries(xq_o, wq_o, ms, ns)
    assert_gemm_close(yc[ms, ns], ref, na, nb, 5120, True, "prefill")
    assert np.isfinite(yc).all()
