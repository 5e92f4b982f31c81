"""GPU parity of the fused linear layer (activation quantize + W4A4 GEMM) and
of the MLP step SiLU(gate)*up re-quantized to NVFP4, then the down GEMM.

The MLP check has three parts, since the GPU's fp32 h is not bit-equal to the
oracle's fp64 h: (i) GPU h against fp64 SiLU(gate)*up within the propagated
GEMM tolerance; (ii) GPU h_q bit-exact against the oracle quantizer fed the
GPU's own h; (iii) the down projection against the fp64 GEMM of that h_q."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (assert_gemm_close, assert_quantized_equal, bf16_tensor, f32_tensor,
                         gemm_tolerance, to_numpy_f64)
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


@pytest.mark.parametrize("M,N,K", [(8, 512, 1024), (96, 384, 640), (300, 256, 256)])
def test_linear_store(nv, M, N, K):
    rng = np.random.default_rng(M + N + K)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[rng.random(x.shape) < 1e-3] *= 50
    xb = torch.from_numpy(x).to(torch.bfloat16)
    xbits = xb.view(torch.int16).numpy().view(np.uint16)
    wt = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    xq_o, wq_o = oracle.quantize(xbits), oracle.quantize(wt)
    wq = quantize_gpu(nv, f32_tensor(wt))
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    x_q = nv.NVFP4Tensor.empty(M, K)
    ws = nv.workspace(nv.OP_LINEAR_FUSED, M, N, K)
    nv.nvfp4_linear_fused(xb.cuda(), wq, ws, nv.EPI_STORE, y=y, x_q=x_q)
    assert nv.nvfp4_get_device_status(ws) == nv.OK
    assert_quantized_equal(x_q, xq_o)
    ref = oracle.gemm_f64(xq_o, wq_o)
    assert_gemm_close(to_numpy_f64(y), ref, norms(xq_o)[:, None], norms(wq_o)[None, :], K, True, "linear")


@pytest.mark.parametrize("M,N,K", [(12, 256, 320), (20, 200, 576)])
def test_linear_store_f32_pitch(nv, M, N, K):
    """fp32 activations with a row pitch wider than K, the quantized
    activations kept in the workspace (x_q not requested), fp32 output."""
    rng = np.random.default_rng(5 * M + N)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[rng.random(x.shape) < 1e-3] *= 50
    wt = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    xq_o, wq_o = oracle.quantize(x), oracle.quantize(wt)
    wq = quantize_gpu(nv, f32_tensor(wt))
    buf = torch.zeros((M, K + 16), dtype=torch.float32, device="cuda")
    buf[:, :K] = f32_tensor(x)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    ws = nv.workspace(nv.OP_LINEAR_FUSED, M, N, K)
    nv.nvfp4_linear_fused(buf[:, :K], wq, ws, nv.EPI_STORE, y=y)
    assert nv.nvfp4_get_device_status(ws) == nv.OK
    ref = oracle.gemm_f64(xq_o, wq_o)
    assert_gemm_close(to_numpy_f64(y), ref, norms(xq_o)[:, None], norms(wq_o)[None, :], K, False,
                      "linear fp32 pitch")


def _silu(z):
    return z / (1.0 + np.exp(-z))


def check_mlp(nv, X, Wg, Wu, Wd, M, K, N):
    """X bf16 bits [M][K]; Wg, Wu [N][K]; Wd [K][N] (bf16 bits)."""
    xq_o = oracle.quantize(X)
    wg_o, wu_o, wd_o = oracle.quantize(Wg), oracle.quantize(Wu), oracle.quantize(Wd)
    wg, wu, wd = (quantize_gpu(nv, bf16_tensor(a)) for a in (Wg, Wu, Wd))
    h = torch.empty((M, N), dtype=torch.float32, device="cuda")
    h_q = nv.NVFP4Tensor.empty(M, N)
    ws = nv.workspace(nv.OP_LINEAR_FUSED_SILU, M, N, K)
    nv.nvfp4_linear_fused(bf16_tensor(X), wg, ws, nv.EPI_SILU_MUL_REQUANT, y=h, w_up=wu, y_q=h_q)
    y = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    nv.nvfp4_gemm(h_q, wd, y, nv.workspace(nv.OP_GEMM, M, K, N))
    assert nv.nvfp4_get_device_status(ws) == nv.OK

    # (i) h against fp64 SiLU(gate) * up with the GEMM tolerance propagated
    gate = oracle.gemm_f64(xq_o, wg_o)
    up = oracle.gemm_f64(xq_o, wu_o)
    h_ref = oracle.silu_mul_f64(gate, up)
    nx = norms(xq_o)[:, None]
    tg = gemm_tolerance(gate, nx, norms(wg_o)[None, :], K, False)
    tu = gemm_tolerance(up, nx, norms(wu_o)[None, :], K, False)
    dsilu_max = 1.1   # |d/dz z*sigmoid(z)| <= 1.0998
    tol_h = dsilu_max * (np.abs(up) + tu) * tg + np.abs(_silu(gate)) * tu + 1e-6 * np.abs(h_ref)
    hc = h.cpu().numpy().astype(np.float64)
    err = np.abs(hc - h_ref)
    assert (err <= tol_h).all(), f"h: max err/tol {(err / tol_h).max():.3f}"

    # (ii) h_q bit-exact against the oracle quantizer fed the GPU's h
    hq_o = oracle.quantize(h.cpu().numpy())
    assert_quantized_equal(h_q, hq_o)

    # (iii) the down projection against the fp64 GEMM of that h_q
    ref = oracle.gemm_f64(hq_o, wd_o)
    assert_gemm_close(to_numpy_f64(y), ref, norms(hq_o)[:, None], norms(wd_o)[None, :], N, True, "down")


# h_q is formed either inside the gate/up kernel's epilogue (the default when
# the tiles fit one per SM) or by the quantizer's encode pass over h
# (NVFP4_MLP_FUSED_REQUANT=0, and always when the tiles outnumber the SMs).
@pytest.mark.parametrize("fused", ["1", "0"])
def test_mlp_small(nv, fused, monkeypatch):
    monkeypatch.setenv("NVFP4_MLP_FUSED_REQUANT", fused)
    M, K, N = 32, 512, 384
    w = workloads.make("mlp", M=M, K=K, N=N, seed=40)
    check_mlp(nv, w["X"], w["Wg"], w["Wu"], w["Wd"], M, K, N)


@pytest.mark.parametrize("fused", ["1", "0"])
def test_mlp_ragged_tiles(nv, fused, monkeypatch):
    """Two 128-row tiles with a partial second one, a partial last 128-column
    tile of h and a partial last K slab, through the fused gate/up kernel."""
    monkeypatch.setenv("NVFP4_MLP_FUSED_REQUANT", fused)
    M, K, N = 200, 320, 320
    w = workloads.make("mlp", M=M, K=K, N=N, seed=41)
    check_mlp(nv, w["X"], w["Wg"], w["Wu"], w["Wd"], M, K, N)


def test_mlp_more_tiles_than_sms(nv):
    """9 x 18 = 162 gate/up tiles, more than the SMs: the encode pass path."""
    M, K, N = 1100, 256, 2304
    w = workloads.make("mlp", M=M, K=K, N=N, seed=42)
    check_mlp(nv, w["X"], w["Wg"], w["Wu"], w["Wd"], M, K, N)


def test_mlp_fused_requant_without_h(nv, monkeypatch):
    """The in-epilogue re-quantization with h not requested (h never written)
    gives the same h_q bytes (padding included) and tensor scale as with h
    requested, and as the separate encode pass; also against the oracle's
    quantization of the GPU's h.  N = 1040: 65 blocks per row, so the scale
    rows are padded to 68 and the last tile's second half lies past them."""
    M, K, N = 160, 1024, 1040
    w = workloads.make("mlp", M=M, K=K, N=N, seed=43)
    wg, wu = quantize_gpu(nv, bf16_tensor(w["Wg"])), quantize_gpu(nv, bf16_tensor(w["Wu"]))
    x = bf16_tensor(w["X"])
    ws = nv.workspace(nv.OP_LINEAR_FUSED_SILU, M, N, K)
    outs = []
    h = torch.empty((M, N), dtype=torch.float32, device="cuda")
    for fused, with_h in (("1", False), ("1", True), ("0", True)):
        monkeypatch.setenv("NVFP4_MLP_FUSED_REQUANT", fused)
        h_q = nv.NVFP4Tensor.empty(M, N)
        h_q.codes.fill_(0x77)
        h_q.scales.fill_(0x55)
        nv.nvfp4_linear_fused(x, wg, ws, nv.EPI_SILU_MUL_REQUANT, y=h if with_h else None, w_up=wu, y_q=h_q)
        assert nv.nvfp4_get_device_status(ws) == nv.OK
        torch.cuda.synchronize()
        outs.append(h_q)
    assert_quantized_equal(outs[0], oracle.quantize(h.cpu().numpy()))
    for q in outs[1:]:
        assert torch.equal(q.codes, outs[0].codes)
        assert torch.equal(q.scales, outs[0].scales)
        assert torch.equal(q.tensor_scale, outs[0].tensor_scale)


def test_linear_degenerate_shapes(nv):
    """K = 0 is an empty reduction: the STORE form writes zeros and the
    quantized x has g = 0; the SiLU form gives h = SiLU(0) * 0 = 0, so y_q has
    all-zero codes and scales and g = 0.  With N = 0 the SiLU form writes
    only y_q's g."""
    M, N = 5, 64
    x = torch.empty((M, 0), dtype=torch.bfloat16, device="cuda")
    w, wu = nv.NVFP4Tensor.empty(N, 0), nv.NVFP4Tensor.empty(N, 0)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    xq = nv.NVFP4Tensor.empty(M, 0)
    xq.tensor_scale.fill_(7.0)
    ws = nv.workspace(nv.OP_LINEAR_FUSED, M, N, 0)
    nv.nvfp4_linear_fused(x, w, ws, nv.EPI_STORE, y=y, x_q=xq)
    torch.cuda.synchronize()
    assert torch.count_nonzero(y) == 0 and xq.tensor_scale[0].item() == 0.0
    assert nv.nvfp4_get_device_status(ws) == nv.OK

    yq = nv.NVFP4Tensor.empty(M, N)
    yq.codes.fill_(0x77)
    yq.scales.fill_(0x38)
    yq.tensor_scale.fill_(7.0)
    h = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    ws = nv.workspace(nv.OP_LINEAR_FUSED_SILU, M, N, 0)
    nv.nvfp4_linear_fused(x, w, ws, nv.EPI_SILU_MUL_REQUANT, y=h, w_up=wu, y_q=yq)
    torch.cuda.synchronize()
    assert torch.count_nonzero(h) == 0
    assert torch.count_nonzero(yq.codes) == 0 and torch.count_nonzero(yq.scales) == 0
    assert yq.tensor_scale[0].item() == 0.0
    assert nv.nvfp4_get_device_status(ws) == nv.OK

    x1 = torch.randn((M, 64), device="cuda").to(torch.bfloat16)
    yq0 = nv.NVFP4Tensor.empty(M, 0)
    yq0.tensor_scale.fill_(7.0)
    ws = nv.workspace(nv.OP_LINEAR_FUSED_SILU, M, 0, 64)
    nv.nvfp4_linear_fused(x1, nv.NVFP4Tensor.empty(0, 64), ws, nv.EPI_SILU_MUL_REQUANT,
                          w_up=nv.NVFP4Tensor.empty(0, 64), y_q=yq0)
    torch.cuda.synchronize()
    assert yq0.tensor_scale[0].item() == 0.0
    assert nv.nvfp4_get_device_status(ws) == nv.OK


def test_mlp_workload_full(nv):
    """The fused MLP workload at full size: M=128, K=5120, N=17408 (seed 4)."""
    w = workloads.make("mlp")
    check_mlp(nv, w["X"], w["Wg"], w["Wu"], w["Wd"], 128, 5120, 17408)


def test_mlp_fused_requant_reuses_one_workspace_across_grids(nv):
    """The in-epilogue form's grid meeting point lives in the workspace and must
    be back at its start after every call: one workspace serves calls whose
    grids have 3, 18 and 6 CTAs, in that order and twice, each h_q bit-exact
    against the oracle's quantization of the GPU's own h."""
    shapes = [(32, 256, 384), (160, 256, 1040), (200, 320, 320)] * 2
    big = max(nv.workspace_bytes(nv.OP_LINEAR_FUSED_SILU, M, N, K) for M, K, N in shapes)
    ws = torch.zeros(big, dtype=torch.uint8, device="cuda")
    for i, (M, K, N) in enumerate(shapes):
        w = workloads.make("mlp", M=M, K=K, N=N, seed=50 + i)
        wg, wu = quantize_gpu(nv, bf16_tensor(w["Wg"])), quantize_gpu(nv, bf16_tensor(w["Wu"]))
        h = torch.empty((M, N), dtype=torch.float32, device="cuda")
        h_q = nv.NVFP4Tensor.empty(M, N)
        nv.nvfp4_linear_fused(bf16_tensor(w["X"]), wg, ws, nv.EPI_SILU_MUL_REQUANT, y=h, w_up=wu, y_q=h_q)
        assert nv.nvfp4_get_device_status(ws) == nv.OK
        assert_quantized_equal(h_q, oracle.quantize(h.cpu().numpy()))
