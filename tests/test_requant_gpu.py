"""GPU parity of the re-quantized GEMM output (y as stored, quantized to
NVFP4 for the next layer): nvfp4_gemm_requant and the y_q output of
nvfp4_linear_fused's store form.

No new oracle arithmetic is involved: y_q must be exactly what the oracle's
quantizer makes of the y the GPU stored (its bf16 bits or fp32 values), so
that is compared bit for bit, codes, tiled scales (padding zero) and tensor
scale; y itself is checked against the fp64 oracle GEMM as everywhere else.
The shapes reach every epilogue that stores output: the CTA-pair kernel
(TMA-store staging, per-row fp32), the one-CTA kernel (fast drain, general
path, 256-wide tiles), the swapped kernel (tile loop and stream-K), the
stream-K finishing pass without swap, and the one-launch decode kernel."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (assert_gemm_close, assert_quantized_equal, bf16_tensor, f32_tensor, to_numpy_f64)
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


def norms(q):
    return np.linalg.norm(oracle.dequantize_f64(q), axis=1)


def stored(y):
    """y as the oracle reads it: bf16 bit patterns or fp32 values."""
    torch.cuda.synchronize()
    if y.dtype == torch.bfloat16:
        return y.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return y.contiguous().cpu().numpy()


def poisoned_yq(nv, M, N):
    yq = nv.NVFP4Tensor.empty(M, N)
    yq.codes.fill_(0x77)
    yq.scales.fill_(0x55)
    yq.tensor_scale.fill_(7.0)
    return yq


def operands(nv, M, N, K, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[rng.random(x.shape) < 1e-3] *= 50
    wt = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    xq_o, wq_o = oracle.quantize(x), oracle.quantize(wt)
    return x, xq_o, wq_o, quantize_gpu(nv, f32_tensor(x)), quantize_gpu(nv, f32_tensor(wt))


# (M, N, K, y dtype, CTA pair allowed, what)
GEMM_CASES = [
    (2048, 4608, 256, torch.bfloat16, True, "pair, TMA-store epilogue"),
    (2000, 4624, 320, torch.float32, True, "pair, per-row fp32, ragged M"),
    (300, 1024, 640, torch.bfloat16, False, "one-CTA fast drain"),
    (300, 1008, 640, torch.float32, False, "one-CTA general path, fp32"),
    (1024, 9472, 256, torch.bfloat16, False, "one-CTA 256-wide tiles"),
    (40, 17408, 512, torch.bfloat16, True, "swapped, tile loop"),
    (24, 1008, 1088, torch.float32, True, "swapped, stream-K, fp32"),
    (8, 1024, 1344, torch.bfloat16, True, "swapped, stream-K"),
    (128, 2048, 17408, torch.bfloat16, True, "stream-K, not swapped"),
]


@pytest.mark.parametrize("M,N,K,yt,pair,what", GEMM_CASES, ids=[c[5] for c in GEMM_CASES])
def test_gemm_requant(nv, M, N, K, yt, pair, what, monkeypatch):
    if not pair:
        monkeypatch.setenv("NVFP4_GEMM_CTA_PAIR", "0")
    _, xq_o, wq_o, xq, wq = operands(nv, M, N, K, M + N + K)
    y = torch.full((M, N), float("nan"), dtype=yt, device="cuda")
    yq = poisoned_yq(nv, M, N)
    ws = nv.workspace(nv.OP_GEMM_REQUANT, M, N, K)
    nv.nvfp4_gemm_requant(xq, wq, y, yq, ws)
    assert nv.nvfp4_get_device_status(ws) == nv.OK
    ys = stored(y)
    assert_quantized_equal(yq, oracle.quantize(ys))
    # y itself: every output for the small cases, a sample for the large ones
    if M * N <= 2_000_000:
        ref = oracle.gemm_f64(xq_o, wq_o)
        assert_gemm_close(to_numpy_f64(y), ref, norms(xq_o)[:, None], norms(wq_o)[None, :], K,
                          yt == torch.bfloat16, what)
    else:
        rng = np.random.default_rng(3)
        ms, ns = rng.integers(0, M, 20000), rng.integers(0, N, 20000)
        ref, na, nb = oracle.gemm_entries(xq_o, wq_o, ms, ns)
        assert_gemm_close(to_numpy_f64(y)[ms, ns], ref, na, nb, K, yt == torch.bfloat16, what)


@pytest.mark.parametrize("M,N,K,yt", [(8, 1024, 1344, torch.bfloat16), (13, 640, 320, torch.float32),
                                      (96, 384, 640, torch.bfloat16), (300, 256, 256, torch.float32)])
def test_linear_store_requant(nv, M, N, K, yt):
    """nvfp4_linear_fused(STORE) with y_q: the decode kernel for M <= 16, the
    quantizer + GEMM path otherwise; x_q and y_q both checked bit-exact."""
    x, xq_o, wq_o, _, wq = operands(nv, M, N, K, 11 * M + N)
    y = torch.full((M, N), float("nan"), dtype=yt, device="cuda")
    yq = poisoned_yq(nv, M, N)
    x_q = nv.NVFP4Tensor.empty(M, K)
    ws = nv.workspace(nv.OP_LINEAR_FUSED, M, N, K)
    nv.nvfp4_linear_fused(f32_tensor(x), wq, ws, nv.EPI_STORE, y=y, y_q=yq, x_q=x_q)
    assert nv.nvfp4_get_device_status(ws) == nv.OK
    assert_quantized_equal(x_q, xq_o)
    assert_quantized_equal(yq, oracle.quantize(stored(y)))
    ref = oracle.gemm_f64(xq_o, wq_o)
    assert_gemm_close(to_numpy_f64(y), ref, norms(xq_o)[:, None], norms(wq_o)[None, :], K,
                      yt == torch.bfloat16, "linear + y_q")


def test_requant_degenerate_shapes(nv):
    """K = 0: y = 0, so y_q is all zero with g = 0; N = 0 or M = 0: only
    y_q's g (0) is written."""
    M, N = 5, 64
    a, b = nv.NVFP4Tensor.empty(M, 0), nv.NVFP4Tensor.empty(N, 0)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    yq = poisoned_yq(nv, M, N)
    nv.nvfp4_gemm_requant(a, b, y, yq, nv.workspace(nv.OP_GEMM_REQUANT, M, N, 0))
    torch.cuda.synchronize()
    assert torch.count_nonzero(y) == 0
    assert torch.count_nonzero(yq.codes) == 0 and torch.count_nonzero(yq.scales) == 0
    assert yq.tensor_scale[0].item() == 0.0
    for (m, n) in ((0, 64), (5, 0)):
        yq0 = poisoned_yq(nv, m, n)
        y0 = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
        nv.nvfp4_gemm_requant(nv.NVFP4Tensor.empty(m, 64), nv.NVFP4Tensor.empty(n, 64), y0, yq0,
                              nv.workspace(nv.OP_GEMM_REQUANT, m, n, 64))
        torch.cuda.synchronize()
        assert yq0.tensor_scale[0].item() == 0.0
    # the linear layer's store form, K = 0
    x = torch.empty((M, 0), dtype=torch.bfloat16, device="cuda")
    yq = poisoned_yq(nv, M, N)
    ws = nv.workspace(nv.OP_LINEAR_FUSED, M, N, 0)
    nv.nvfp4_linear_fused(x, nv.NVFP4Tensor.empty(N, 0), ws, nv.EPI_STORE, y=y, y_q=yq)
    torch.cuda.synchronize()
    assert torch.count_nonzero(yq.codes) == 0 and yq.tensor_scale[0].item() == 0.0
    assert nv.nvfp4_get_device_status(ws) == nv.OK


def test_prefill_requant_workload(nv):
    """Prefill workload at full size (M=4096, N=17408, K=5120, seed 3) through
    nvfp4_linear_fused(STORE, y_q, x_q): y on 4096 sampled outputs plus a full
    row and column, y_q bit-exact against the oracle's quantization of all of
    the stored y."""
    w = workloads.make("prefill")
    M, N, K = w["M"], w["N"], w["K"]
    xq_o, wq_o = oracle.quantize(w["X"]), oracle.quantize(w["W"])
    wq = quantize_gpu(nv, bf16_tensor(w["W"]))
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    yq = poisoned_yq(nv, M, N)
    x_q = nv.NVFP4Tensor.empty(M, K)
    ws = nv.workspace(nv.OP_LINEAR_FUSED, M, N, K)
    nv.nvfp4_linear_fused(bf16_tensor(w["X"]), wq, ws, nv.EPI_STORE, y=y, y_q=yq, x_q=x_q)
    assert nv.nvfp4_get_device_status(ws) == nv.OK
    assert_quantized_equal(x_q, xq_o)
    ys = stored(y)
    assert_quantized_equal(yq, oracle.quantize(ys))
    rng = np.random.default_rng(2)
    ms = np.concatenate([rng.integers(0, M, 4096), np.full(N, 4095), np.arange(M)])
    ns = np.concatenate([rng.integers(0, N, 4096), np.arange(N), np.full(M, 17407)])
    ref, na, nb = oracle.gemm_entries(xq_o, wq_o, ms, ns)
    yc = to_numpy_f64(y)
    assert_gemm_close(yc[ms, ns], ref, na, nb, K, True, "prefill + y_q")
