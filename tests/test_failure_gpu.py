"""Failure detection on the GPU without a fault: a device-side bounded wait on a
barrier nothing completes gives up after its limit, records NVFP4_ERR_TIMEOUT
in the workspace status word, and leaves the context usable."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    import nvfp4_block_scaled_21_b200 as nv
    ws = nv.workspace(nv.OP_GEMM, 1, 1, 64)
    assert nv.nvfp4_get_device_status(ws) == nv.OK
    nv.nvfp4_selftest_bounded_wait(ws, 2000)          # gives up after 2 ms
    assert nv.nvfp4_get_device_status(ws) == nv.ERR_TIMEOUT
    assert nv.nvfp4_get_device_status(ws) == nv.OK    # read clears the word
    # the context still runs real work afterwards
    x = torch.randn(64, 256, device="cuda")
    q = nv.quantize(x)
    y = torch.empty(64, 64, device="cuda")
    nv.nvfp4_gemm(q, q, y, ws)
    assert nv.nvfp4_get_device_status(ws) == nv.OK
    assert torch.isfinite(y).all()
    d = torch.diagonal(y)
    assert (d > 0).all()                               # x_q . x_q^T has a positive diagonal
