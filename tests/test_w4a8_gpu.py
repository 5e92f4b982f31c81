"""GPU parity of the W4A8 path: FP4 weights (MXFP4) times FP8 activations
(MXFP8: E4M3 elements, one E8M0 scale per 32), the eefocus.com article's W4A8
(the Zhouyi X3 passage), on the tensor cores' mixed block-scaled product
(kind::mxf8f6f4).

The MXFP8 quantizer must equal the oracle's bytes exactly (elements and tiled
scales, padding included); the GEMM must be within the GEMM tolerance of the
fp64 oracle product of the dequantized operands, on every kernel shape
(swapped small-M tiles with and without stream-K, one-CTA 128- and 256-wide
tiles) and through the fused linear layer."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_gemm_close, f32_tensor, to_numpy_f64
from nvfp4_block_scaled_21_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import nvfp4_block_scaled_21_b200 as nv
    return nv


def tiled(scales_rowmajor):
    R, KB = scales_rowmajor.shape
    R128, KB4 = -(-R // 128) * 128, -(-KB // 4) * 4
    out = np.zeros(R128 * KB4, np.uint8)
    r = np.arange(R)[:, None]
    kb = np.arange(KB)[None, :]
    off = ((r // 128) * (KB4 // 4) + kb // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + kb % 4
    out[off.ravel()] = scales_rowmajor.ravel()
    return out


def assert_mx8_equal(gpu, q):
    torch.cuda.synchronize()
    el = gpu.elems.cpu().numpy()
    assert np.array_equal(el, q.elems), f"{int((el != q.elems).sum())} element bytes differ"
    sc = gpu.scales.cpu().numpy()
    assert np.array_equal(sc, tiled(q.scales)), f"{int((sc != tiled(q.scales)).sum())} scale bytes differ"


def activations(rows, cols, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols)).astype(np.float32)
    x[rng.random(x.shape) < 1e-3] *= 50
    return x


@pytest.mark.parametrize("rows,cols,dt", [(8, 5120, torch.bfloat16), (77, 320, torch.float32),
                                          (300, 96, torch.bfloat16), (4096, 5120, torch.bfloat16)])
def test_mx8_quantize_bit_exact(nv, rows, cols, dt):
    x = activations(rows, cols, rows + cols)
    if dt == torch.bfloat16:
        xt = torch.from_numpy(x).to(torch.bfloat16)
        x_or = xt.view(torch.int16).numpy().view(np.uint16)
    else:
        xt, x_or = torch.from_numpy(x), x
    q = nv.MXFP8Tensor.empty(rows, cols)
    q.elems.fill_(0x77)
    q.scales.fill_(0x55)
    nv.nvfp4_mx8_quantize(xt.cuda(), q)
    assert_mx8_equal(q, oracle.mx8_quantize(x_or))


def test_mx8_quantize_special_values(nv):
    x = np.zeros((4, 96), np.float32)
    x[1, :32] = np.linspace(-448.0, 448.0, 32) * 2.0 ** 3      # bamax = 448 * 2^3 exactly
    x[1, 32:64] = np.float32(448.0 * 8) * np.float32(1 + 2 ** -23)
    x[2, :32] = np.float32(1e-40) * np.arange(32)
    x[2, 40] = -0.0
    x[3, :32] = np.finfo(np.float32).max * np.linspace(-1, 1, 32, dtype=np.float32)
    q = nv.MXFP8Tensor.empty(4, 96)
    nv.nvfp4_mx8_quantize(f32_tensor(x), q)
    assert_mx8_equal(q, oracle.mx8_quantize(x))


W4A8_CASES = [
    (8, 4096, 1408, torch.bfloat16, True),      # swapped BN = 16, partial last tile of stages
    (16, 1008, 1152, torch.float32, True),      # swapped, stream-K, ragged N
    (40, 2048, 1024, torch.bfloat16, True),     # swapped BN = 64
    (300, 1024, 640, torch.bfloat16, False),    # one-CTA 128-wide tiles, ragged M
    (1024, 9472, 256, torch.bfloat16, False),   # CTA pair (256x256 tiles)
    (1000, 9000, 512, torch.float32, False),    # CTA pair, ragged M and N, fp32 out
    (128, 2048, 5120, torch.float32, True),     # stream-K, not swapped
]


@pytest.mark.parametrize("M,N,K,yt,_", W4A8_CASES)
def test_w4a8_gemm(nv, M, N, K, yt, _):
    x = activations(M, K, 3 * M + K)
    w = (np.random.default_rng(N + K).standard_normal((N, K)) * 0.02).astype(np.float32)
    xq_o, wq_o = oracle.mx8_quantize(x), oracle.mx_quantize(w)
    xq = nv.MXFP8Tensor.empty(M, K)
    nv.nvfp4_mx8_quantize(f32_tensor(x), xq)
    wq = nv.mx_quantize(f32_tensor(w))
    y = torch.full((M, N), float("nan"), dtype=yt, device="cuda")
    ws = nv.workspace(nv.OP_GEMM, M, N, K)
    nv.nvfp4_w4a8_gemm(xq, wq, y, ws)
    assert nv.nvfp4_get_device_status(ws) == nv.OK
    ref = oracle.w4a8_gemm_f64(xq_o, wq_o)
    na = np.linalg.norm(oracle.mx8_dequantize_f64(xq_o), axis=1)
    nb = np.linalg.norm(oracle.mx_dequantize_f64(wq_o), axis=1)
    assert_gemm_close(to_numpy_f64(y), ref, na[:, None], nb[None, :], K, yt == torch.bfloat16, "w4a8")


def test_w4a8_linear_decode_workload(nv):
    """The decode workload's data (M=8, N=17408, K=5120, seed 2) with MXFP4
    weights through nvfp4_w4a8_linear: x_q bit-exact, every output in tolerance."""
    w = workloads.make("decode")
    M, N, K = w["M"], w["N"], w["K"]
    from gpu_helpers import bf16_tensor
    wq = nv.mx_quantize(bf16_tensor(w["W"]))
    xq = nv.MXFP8Tensor.empty(M, K)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = nv.workspace(nv.OP_W4A8_LINEAR, M, N, K)
    nv.nvfp4_w4a8_linear(bf16_tensor(w["X"]), wq, y, ws, x_q=xq)
    assert nv.nvfp4_get_device_status(ws) == nv.OK
    xq_o, wq_o = oracle.mx8_quantize(w["X"]), oracle.mx_quantize(w["W"])
    assert_mx8_equal(xq, xq_o)
    ref = oracle.w4a8_gemm_f64(xq_o, wq_o)
    na = np.linalg.norm(oracle.mx8_dequantize_f64(xq_o), axis=1)
    nb = np.linalg.norm(oracle.mx_dequantize_f64(wq_o), axis=1)
    assert_gemm_close(to_numpy_f64(y), ref, na[:, None], nb[None, :], K, True, "w4a8 decode")


def test_w4a8_pair_and_one_cta_kernels_agree_with_the_oracle(nv, monkeypatch):
    """The same prefill-shaped W4A8 GEMM (M = 1024: CTA-pair tiles) on the CTA
    pair and, with NVFP4_GEMM_CTA_PAIR=0, on the one-CTA kernel: both within
    the GEMM tolerance of the oracle."""
    M, N, K = 1024, 4608, 1024
    x = activations(M, K, 7)
    w = (np.random.default_rng(8).standard_normal((N, K)) * 0.02).astype(np.float32)
    xq_o, wq_o = oracle.mx8_quantize(x), oracle.mx_quantize(w)
    xq = nv.MXFP8Tensor.empty(M, K)
    nv.nvfp4_mx8_quantize(f32_tensor(x), xq)
    wq = nv.mx_quantize(f32_tensor(w))
    ref = oracle.w4a8_gemm_f64(xq_o, wq_o)
    na = np.linalg.norm(oracle.mx8_dequantize_f64(xq_o), axis=1)
    nb = np.linalg.norm(oracle.mx_dequantize_f64(wq_o), axis=1)
    for pair in ("1", "0"):
        monkeypatch.setenv("NVFP4_GEMM_CTA_PAIR", pair)
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        ws = nv.workspace(nv.OP_GEMM, M, N, K)
        nv.nvfp4_w4a8_gemm(xq, wq, y, ws)
        assert nv.nvfp4_get_device_status(ws) == nv.OK
        assert_gemm_close(to_numpy_f64(y), ref, na[:, None], nb[None, :], K, True, f"w4a8 pair={pair}")
