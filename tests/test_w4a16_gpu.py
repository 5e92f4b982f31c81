"""GPU parity of the W4A16 linear layer: bf16 activations times NVFP4 weights
dequantized inside the kernel (aixq.cc article on Unsloth Dynamic NVFP4,
section "核心差异：W4A4 vs W4A16"), against the fp64 oracle product of the
activations and the exactly dequantized weights.

The bar is the GEMM tolerance of the W4A4 tests with the activation row's norm
taken from the bf16 activations themselves: |y - ref| <= max(2e-3 |ref|,
1e-3 |x_m| |w_n| / sqrt(K)), plus 2^-8 |ref| for a bf16 output."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_gemm_close, bf16_tensor, f32_tensor, to_numpy_f64
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


def run(nv, xbits, wq_gpu, wq_o, M, N, K, yt, pitch=None):
    x = bf16_tensor(xbits)
    if pitch:
        buf = torch.zeros((M, pitch), dtype=torch.bfloat16, device="cuda")
        buf[:, :K] = x
        x = buf[:, :K]
    y = torch.full((M, N), float("nan"), dtype=yt, device="cuda")
    ws = nv.workspace(nv.OP_W4A16, M, N, K)
    nv.nvfp4_w4a16_linear(x, wq_gpu, y, ws)
    assert nv.nvfp4_get_device_status(ws) == nv.OK
    ref = oracle.w4a16_gemm_f64(xbits, wq_o)
    nx = np.linalg.norm(oracle.bf16_bits_to_f32(xbits).astype(np.float64), axis=1)
    nw = np.linalg.norm(oracle.dequantize_f64(wq_o), axis=1)
    assert_gemm_close(to_numpy_f64(y), ref, nx[:, None], nw[None, :], K, yt == torch.bfloat16, "w4a16")


# M up to 16 (one activation tile) and beyond it (several), partial last K
# slab, ragged N, bf16 and fp32 outputs, a row pitch wider than K
@pytest.mark.parametrize("M,N,K,yt,pitch", [(8, 1024, 1344, torch.bfloat16, None), (1, 384, 64, torch.float32, None),
                                            (16, 1000, 320, torch.bfloat16, 336), (13, 256, 5120, torch.float32, None),
                                            (40, 640, 576, torch.bfloat16, None), (3, 136, 192, torch.float32, 256)])
def test_w4a16_parity(nv, M, N, K, yt, pitch):
    w = workloads.make("decode", M=M, K=K, N=N, seed=M + N)
    wq_o = oracle.quantize(w["W"])
    run(nv, w["X"], quantize_gpu(nv, bf16_tensor(w["W"])), wq_o, M, N, K, yt, pitch)


def test_w4a16_many_tiles(nv):
    """More tiles than SMs (3 activation tiles x 136 weight tiles): several
    tiles per CTA, the accumulator handed between them."""
    M, N, K = 40, 17408, 256
    w = workloads.make("decode", M=M, K=K, N=N, seed=7)
    wq_o = oracle.quantize(w["W"])
    run(nv, w["X"], quantize_gpu(nv, bf16_tensor(w["W"])), wq_o, M, N, K, torch.bfloat16)


def test_w4a16_decode_workload(nv):
    """The decode workload's shape and data (M=8, N=17408, K=5120, seed 2):
    every output against the oracle."""
    w = workloads.make("decode")
    wq_o = oracle.quantize(w["W"])
    run(nv, w["X"], quantize_gpu(nv, bf16_tensor(w["W"])), wq_o, 8, 17408, 5120, torch.bfloat16)


def test_w4a16_special_weights(nv):
    """Weights whose blocks reach the E4M3 extremes (scale 448 and the
    smallest subnormal scales) and all-zero blocks: e * s must stay exact."""
    rng = np.random.default_rng(9)
    M, N, K = 4, 128, 256
    w = rng.standard_normal((N, K)).astype(np.float32)
    w[0, :] = 0.0                                   # zero blocks
    w[1, :16] = 1e30                                # sets the tensor scale: other blocks get tiny scales
    w[2, :16] = 1e-20
    wq = quantize_gpu(nv, f32_tensor(w))
    wq_o = oracle.quantize(w)
    x = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(torch.bfloat16)
    run(nv, x.view(torch.int16).numpy().view(np.uint16), wq, wq_o, M, N, K, torch.float32)
