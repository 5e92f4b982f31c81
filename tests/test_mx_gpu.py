"""GPU parity of the MXFP4 path: the one-pass quantizer (E2M1 elements, one
UE8M0 scale per 32 elements; the eefocus.com article on FP4 vs INT4, section
"FP4被视为下一代AI计算的核心标准") bit-exact against the oracle, and the
block-scaled MXFP4 GEMM (kind::mxf4) within the GEMM tolerance of the fp64
oracle product of the dequantized operands, on every kernel shape: the
swapped small-M tiles, stream-K, the one-CTA 128- and 256-wide tiles and the
CTA pair."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_gemm_close, f32_tensor, to_numpy_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import nvfp4_block_scaled_21_b200 as nv
    return nv


def tiled_mx_scales(scales_rowmajor):
    """Oracle scales [R][KB] (KB 32-element blocks) in the padded tiled layout."""
    R, KB = scales_rowmajor.shape
    R128, KB4 = -(-R // 128) * 128, -(-KB // 4) * 4
    out = np.zeros(R128 * KB4, np.uint8)
    r = np.arange(R)[:, None]
    kb = np.arange(KB)[None, :]
    off = ((r // 128) * (KB4 // 4) + kb // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + kb % 4
    out[off.ravel()] = scales_rowmajor.ravel()
    return out


def assert_mx_equal(gpu, q):
    torch.cuda.synchronize()
    codes = gpu.codes.cpu().numpy()
    assert np.array_equal(codes, q.codes), f"{int((codes != q.codes).sum())} code bytes differ"
    sc = gpu.scales.cpu().numpy()
    want = tiled_mx_scales(q.scales)
    assert np.array_equal(sc, want), f"{int((sc != want).sum())} scale bytes differ (padding included)"


def activations(rows, cols, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols)).astype(np.float32)
    x[rng.random(x.shape) < 1e-3] *= 50
    return x


@pytest.mark.parametrize("rows,cols,dt,pitch", [(8192, 5120, torch.bfloat16, None), (1000, 4096, torch.float32, None),
                                                (77, 320, torch.bfloat16, None), (3, 32, torch.float32, None),
                                                (130, 128, torch.bfloat16, 160), (257, 96, torch.float32, 112)])
def test_mx_quantize_bit_exact(nv, rows, cols, dt, pitch):
    x = activations(rows, cols, rows + cols)
    if dt == torch.bfloat16:
        xt = torch.from_numpy(x).to(torch.bfloat16)
        x_or = xt.view(torch.int16).numpy().view(np.uint16)
    else:
        xt, x_or = torch.from_numpy(x), x
    buf = torch.zeros((rows, pitch or cols), dtype=dt, device="cuda")
    buf[:, :cols] = xt.cuda()
    q = nv.MXFP4Tensor.empty(rows, cols)
    q.codes.fill_(0x77)
    q.scales.fill_(0x55)
    nv.nvfp4_mx_quantize(buf[:, :cols], q)
    assert_mx_equal(q, oracle.mx_quantize(x_or))


def test_mx_quantize_special_values(nv):
    """Zero blocks (byte 0, codes 0), blocks whose max sits exactly on 6 * 2^k
    and just above it, fp32 subnormals and the largest finite fp32."""
    x = np.zeros((4, 128), np.float32)
    x[1, :32] = np.linspace(-6.0, 6.0, 32) * 2.0 ** 5                       # bamax = 6 * 2^5 exactly
    x[1, 32:64] = np.float32(6.0 * 2.0 ** 5) * np.float32(1 + 2 ** -23)    # just above
    x[2, :32] = np.float32(1e-40) * np.arange(32)                          # subnormals
    x[3, :32] = np.finfo(np.float32).max * np.linspace(-1, 1, 32, dtype=np.float32)
    q = nv.mx_quantize(f32_tensor(x))
    assert_mx_equal(q, oracle.mx_quantize(x))


def mx_norms(q):
    return np.linalg.norm(oracle.mx_dequantize_f64(q), axis=1)


# (M, N, K, y dtype, CTA pair allowed): swapped BN 16/32/64 (tile loop and
# stream-K), one-CTA 128- and 256-wide tiles, the CTA pair, a partial last K
# slab (K % 256 != 0) and an odd number of K steps (K % 128 == 64).
MX_CASES = [
    (8, 17408, 5120, torch.bfloat16, True),
    (16, 1008, 1344, torch.float32, True),
    (40, 2048, 1088, torch.bfloat16, True),
    (64, 4096, 320, torch.bfloat16, True),
    (300, 1024, 640, torch.bfloat16, False),
    (1024, 9472, 192, torch.bfloat16, False),
    (2048, 4608, 256, torch.bfloat16, True),
    (2000, 4624, 320, torch.float32, True),
    (4096, 17408, 5120, torch.bfloat16, True),
]


@pytest.mark.parametrize("M,N,K,yt,pair", MX_CASES)
def test_mx_gemm(nv, M, N, K, yt, pair, monkeypatch):
    if not pair:
        monkeypatch.setenv("NVFP4_GEMM_CTA_PAIR", "0")
    x = activations(M, K, M * 7 + K)
    rng = np.random.default_rng(N + K)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    xq_o, wq_o = oracle.mx_quantize(x), oracle.mx_quantize(w)
    xq, wq = nv.mx_quantize(f32_tensor(x)), nv.mx_quantize(f32_tensor(w))
    assert_mx_equal(xq, xq_o)
    y = torch.full((M, N), float("nan"), dtype=yt, device="cuda")
    ws = nv.workspace(nv.OP_GEMM, M, N, K)
    nv.nvfp4_mx_gemm(xq, wq, y, ws)
    assert nv.nvfp4_get_device_status(ws) == nv.OK
    yc = to_numpy_f64(y)
    assert np.isfinite(yc).all()
    na, nb = mx_norms(xq_o), mx_norms(wq_o)
    if M * N <= 4_000_000:
        ref = oracle.mx_gemm_f64(xq_o, wq_o)
        assert_gemm_close(yc, ref, na[:, None], nb[None, :], K, yt == torch.bfloat16, "mx gemm")
    else:
        # sampled outputs: the oracle's dot products of single dequantized rows
        da, db = oracle.mx_dequantize_f64(xq_o), oracle.mx_dequantize_f64(wq_o)
        rs = np.random.default_rng(5)
        ms = np.concatenate([rs.integers(0, M, 4096), np.full(N, M - 1)])
        ns = np.concatenate([rs.integers(0, N, 4096), np.arange(N)])
        ref = np.einsum("ik,ik->i", da[ms], db[ns])
        assert_gemm_close(yc[ms, ns], ref, na[ms], nb[ns], K, yt == torch.bfloat16, "mx gemm sampled")
