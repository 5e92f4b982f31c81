"""nvfp4_linear_noalloc, the linear layer for callers that cannot allocate
device memory (no workspace: the library keeps the scratch in a static device
array), must give the same answer as nvfp4_linear_fused with a caller
workspace, call after call.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it must also pass alone in a fresh
process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import gemm_tolerance

pytestmark = pytest.mark.gpu


def _inputs(M, K, N, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[rng.random(x.shape) < 1e-3] *= 50
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    return x, w


def _call_noalloc(nv, x, wq, y):
    """Through the C ABI: plain pointers, sizes and the current stream."""
    cw = wq.c()
    st = nv.lib().nvfp4_linear_noalloc(
        ctypes.c_void_p(x.data_ptr()), nv.BF16, x.shape[0], x.shape[1], x.stride(0),
        ctypes.byref(cw), ctypes.c_void_p(y.data_ptr()), nv.BF16, y.stride(0),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == nv.OK, nv.status_string(st)


@pytest.mark.parametrize("M,K,N", [(8, 5120, 1024), (130, 1024, 640)])
def test_noalloc_matches_workspace_entry_point_twice(M, K, N):
    import nvfp4_block_scaled_21_b200 as nv
    wq = None
    for call, seed in enumerate((M + 1, M + 2)):          # two calls in a row, different inputs
        x, w = _inputs(M, K, N, seed)
        if wq is None:
            wq = nv.quantize(torch.from_numpy(w).cuda())
            w_o = oracle.quantize(w)
        xb = torch.from_numpy(x).to(torch.bfloat16).cuda()
        y_ref = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        ws = nv.workspace(nv.OP_LINEAR_FUSED, M, N, K)
        nv.nvfp4_linear_fused(xb, wq, ws, nv.EPI_STORE, y=y_ref)
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        _call_noalloc(nv, xb, wq, y)
        torch.cuda.synchronize()
        ref = y_ref.float().cpu().numpy().astype(np.float64)
        got = y.float().cpu().numpy().astype(np.float64)
        x_o = oracle.quantize(xb.cpu().view(torch.int16).numpy().view(np.uint16))
        na = np.linalg.norm(oracle.dequantize_f64(x_o), axis=1)[:, None]
        nb = np.linalg.norm(oracle.dequantize_f64(w_o), axis=1)[None, :]
        tol = gemm_tolerance(ref, na, nb, K, True)
        err = np.abs(got - ref)
        assert np.isfinite(got).all(), f"call {call}: non-finite output"
        assert (err <= tol).all(), f"call {call}: max err/tol {(err / tol).max():.3f}"
        # and against the fp64 oracle itself, on sampled outputs
        rng = np.random.default_rng(call)
        ms, ns = rng.integers(0, M, 512), rng.integers(0, N, 512)
        ref_o, na_o, nb_o = oracle.gemm_entries(x_o, w_o, ms, ns)
        tol_o = gemm_tolerance(ref_o, na_o, nb_o, K, True)
        err_o = np.abs(got[ms, ns] - ref_o)
        assert (err_o <= tol_o).all(), f"call {call}: vs oracle max err/tol {(err_o / tol_o).max():.3f}"


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import nvfp4_block_scaled_21_b200 as nv
    M, K, N = 4096, 5120, 256                                # 10.5 MB of codes > 4 MiB
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    wq = nv.quantize(torch.ones((N, K), device="cuda"))
    y = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    cw = wq.c()
    st = nv.lib().nvfp4_linear_noalloc(
        ctypes.c_void_p(x.data_ptr()), nv.BF16, M, K, K, ctypes.byref(cw),
        ctypes.c_void_p(y.data_ptr()), nv.BF16, N, None)
    assert st == nv.ERR_UNSUPPORTED_SHAPE
    torch.cuda.synchronize()
    assert torch.count_nonzero(y) == 0                       # nothing was launched
