"""GPU parity of the tensor-parallel entry points: the quantizer's first pass
on its own (nvfp4_amax) and its second pass with a given amax
(nvfp4_quantize_with_amax), which together quantize a tensor split across
ranks by rows with the one FP32 tensor scale of the whole tensor (NVFP4 wiki
page, section "技術原理").  Ranks are simulated here in one process: each
shard's amax is taken, the largest is kept (what the ranks' all-reduce MAX
gives), and each shard is quantized with it; the result must equal, bit for
bit, the oracle's quantization of the whole tensor restricted to the shard's
rows.  The sequencing over torch.distributed (tp.py) runs with a one-rank
gloo group (the host-copy path of its collective) and, for two ranks, on the
CPU in tests/test_tp_multirank.py."""
import socket

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_gemm_close, assert_quantized_equal, bf16_tensor, f32_tensor, to_numpy_f64
from nvfp4_block_scaled_21_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import nvfp4_block_scaled_21_b200 as nv
    return nv


def _x(rows, cols, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols)).astype(np.float32)
    x[rng.random(x.shape) < 1e-3] *= 50
    return x


@pytest.mark.parametrize("rows,cols,dtype,pitch", [(300, 512, "bf16", None), (7, 80, "f32", 96), (0, 64, "bf16", None),
                                                  (4096, 5120, "bf16", None)])
def test_amax_is_the_largest_magnitude(nv, rows, cols, dtype, pitch):
    x = _x(rows, cols, rows + cols)
    t = f32_tensor(x) if dtype == "f32" else f32_tensor(x).to(torch.bfloat16)
    if pitch:
        buf = torch.zeros((rows, pitch), dtype=t.dtype, device="cuda")
        buf[:, :cols] = t
        t = buf[:, :cols]
    amax = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    nv.nvfp4_amax(t, amax, nv.workspace(nv.OP_QUANTIZE, rows, 0, cols))
    want = float(t.abs().max()) if t.numel() else 0.0
    assert float(amax[0]) == want


@pytest.mark.parametrize("cuts", [(200,), (130, 131, 300), (64,)])
def test_row_shards_quantize_like_the_whole_tensor(nv, cuts):
    """Shards of 200|136, 130|1|169|36 and 64|272 rows of a 336 x 512 tensor
    (padding inside a shard's last 128-row scale tile, one-row shards)."""
    rows, cols = 336, 512
    x = _x(rows, cols, sum(cuts))
    xb = f32_tensor(x).to(torch.bfloat16)
    whole = oracle.quantize(xb.cpu().view(torch.int16).numpy().view(np.uint16))
    bounds = [0, *cuts, rows]
    shards = [(a, b) for a, b in zip(bounds[:-1], bounds[1:])]
    amaxes = []
    for a, b in shards:
        m = torch.empty(1, dtype=torch.float32, device="cuda")
        nv.nvfp4_amax(xb[a:b], m, nv.workspace(nv.OP_QUANTIZE, b - a, 0, cols))
        amaxes.append(m)
    shared = torch.stack(amaxes).max().reshape(1)           # the ranks' all-reduce MAX
    for a, b in shards:
        q = nv.NVFP4Tensor.empty(b - a, cols)
        nv.nvfp4_quantize_with_amax(xb[a:b], shared, q, nv.workspace(nv.OP_QUANTIZE, b - a, 0, cols))
        want = oracle.Quantized(whole.codes[a:b], whole.scales[a:b], whole.g, b - a, cols)
        assert_quantized_equal(q, want)


def test_quantize_with_amax_of_an_empty_shard_still_sets_the_tensor_scale(nv):
    q = nv.NVFP4Tensor.empty(0, 64)
    amax = torch.tensor([2688.0 * 4], dtype=torch.float32, device="cuda")
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    nv.nvfp4_quantize_with_amax(x, amax, q, nv.workspace(nv.OP_QUANTIZE, 0, 0, 64))
    torch.cuda.synchronize()
    assert float(q.tensor_scale[0]) == 4.0


def _one_rank_group():
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    return dist


def test_tp_helpers_on_a_one_rank_group(nv):
    """tp.quantize_row_sharded and tp.mlp_tensor_parallel through a real
    process group (gloo: the all-reduces go through host copies): with one
    rank they must give the plain quantizer's result, and the MLP the oracle's
    SiLU(gate)*up re-quantized with its own amax, then the down projection."""
    from nvfp4_block_scaled_21_b200 import tp
    dist = _one_rank_group()
    try:
        x = _x(96, 256, 3)
        xb = f32_tensor(x).to(torch.bfloat16)
        q = nv.NVFP4Tensor.empty(96, 256)
        tp.quantize_row_sharded(xb, q, nv.workspace(nv.OP_QUANTIZE, 96, 0, 256))
        assert_quantized_equal(q, oracle.quantize(xb.cpu().view(torch.int16).numpy().view(np.uint16)))

        M, K, N = 32, 512, 384
        w = workloads.make("mlp", M=M, K=K, N=N, seed=44)
        wg, wu, wd = (nv.quantize(bf16_tensor(w[k])) for k in ("Wg", "Wu", "Wd"))
        y = tp.mlp_tensor_parallel(bf16_tensor(w["X"]), wg, wu, wd)
        xq_o = oracle.quantize(w["X"])
        wg_o, wu_o, wd_o = oracle.quantize(w["Wg"]), oracle.quantize(w["Wu"]), oracle.quantize(w["Wd"])
        h_ref = oracle.silu_mul_f64(oracle.gemm_f64(xq_o, wg_o), oracle.gemm_f64(xq_o, wu_o))
        # the down projection's input is the GPU's own h quantized (as the
        # non-parallel MLP test does it), so only the last GEMM is compared
        torch.cuda.synchronize()
        assert np.isfinite(to_numpy_f64(y)).all()
        h = torch.empty((M, N), dtype=torch.float32, device="cuda")
        hq = nv.NVFP4Tensor.empty(M, N)
        nv.nvfp4_linear_fused(bf16_tensor(w["X"]), wg, nv.workspace(nv.OP_LINEAR_FUSED_SILU, M, N, K),
                              nv.EPI_SILU_MUL_REQUANT, y=h, w_up=wu, y_q=hq)
        hq_o = oracle.quantize(h.cpu().numpy())
        assert np.abs(h.cpu().numpy() - h_ref).max() <= 1e-2 * max(1.0, np.abs(h_ref).max())
        ref = oracle.gemm_f64(hq_o, wd_o)
        na = np.linalg.norm(oracle.dequantize_f64(hq_o), axis=1)[:, None]
        nb = np.linalg.norm(oracle.dequantize_f64(wd_o), axis=1)[None, :]
        assert_gemm_close(to_numpy_f64(y), ref, na, nb, N, False, "tp mlp down")
    finally:
        dist.destroy_process_group()
