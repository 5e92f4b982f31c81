"""Tensor-parallel sequencing (nvfp4_block_scaled_21_b200.tp) on CPU with two
gloo ranks.

The helpers only order library calls around two collectives: an all-reduce
MAX of one float (the shared amax of a tensor split across ranks, which every
NVFP4 tensor needs for its single FP32 tensor scale: NVFP4 wiki page, section
"技術原理") and, for the MLP's row-parallel down projection, an all-reduce
SUM of the partial outputs.  Here each rank runs them against a stand-in for
the library that computes in plain fp32 on the CPU (no quantization), so the
test checks the sharding and the exchanges: every rank must quantize with the
global amax, and the summed outputs must equal the unsharded MLP.  The
library's own arithmetic on these calls is checked on the GPU
(tests/test_tp_gpu.py).
"""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


_RANK_SCRIPT = r"""
import json, os, sys
sys.path.insert(0, {root!r})
import torch
import torch.distributed as dist
from nvfp4_block_scaled_21_b200 import tp

rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", rank=rank, world_size=world)


class Q:                                   # stands in for an NVFP4Tensor: keeps fp32 values
    def __init__(self, rows, cols, values=None):
        self.rows, self.cols, self.values, self.amax = rows, cols, values, None


class Lib:                                 # stands in for the library: fp32 on the CPU
    OP_QUANTIZE, OP_GEMM, OP_LINEAR_FUSED_SILU = 0, 2, 4
    EPI_STORE, EPI_SILU_MUL_REQUANT = 0, 1
    calls = []

    class NVFP4Tensor:
        @staticmethod
        def empty(rows, cols):
            return Q(rows, cols)

    def workspace(self, *args):
        return None

    def nvfp4_amax(self, x, amax, ws, stream=None):
        self.calls.append("amax")
        amax[0] = x.abs().max() if x.numel() else 0.0

    def nvfp4_quantize_with_amax(self, x, amax, out, ws, stream=None):
        self.calls.append("quantize_with_amax")
        out.values, out.amax = x.clone(), float(amax[0])

    def nvfp4_linear_fused(self, x, w, ws, epi, y=None, w_up=None, y_q=None, x_q=None, stream=None):
        self.calls.append("linear_fused")
        assert epi == self.EPI_SILU_MUL_REQUANT
        g, u = x @ w.values.T, x @ w_up.values.T
        y.copy_(torch.nn.functional.silu(g) * u)

    def nvfp4_gemm(self, a, b, y, ws, stream=None):
        self.calls.append("gemm")
        y.copy_(a.values @ b.values.T)


gen = torch.Generator().manual_seed(7)
M, K, N, KO = 8, 64, 96, 48                # N / 2 = 48: a multiple of 16
x = torch.randn(M, K, generator=gen)
wg, wu = torch.randn(N, K, generator=gen) * 0.1, torch.randn(N, K, generator=gen) * 0.1
wd = torch.randn(KO, N, generator=gen) * 0.1
lib = Lib()

# a tensor split by rows: every rank quantizes with the largest amax
rows = x[rank * 3:(rank + 1) * 3 + rank]   # unequal shares: 3 and 4 rows
out = Q(rows.shape[0], K)
tp.quantize_row_sharded(rows, out, None, lib=lib)
full_amax = float(x[:7].abs().max())
assert out.amax == full_amax, (out.amax, full_amax)
assert torch.equal(out.values, rows)

# the MLP: gate/up split by output rows, down by its reduction columns
lib.calls.clear()
s = slice(rank * N // 2, (rank + 1) * N // 2)
y = tp.mlp_tensor_parallel(x, Q(N // 2, K, wg[s]), Q(N // 2, K, wu[s]), Q(KO, N // 2, wd[:, s]), lib=lib)
h = torch.nn.functional.silu(x @ wg.T) * (x @ wu.T)
ref = h @ wd.T
assert torch.allclose(y, ref, rtol=1e-5, atol=1e-5), float((y - ref).abs().max())
assert lib.calls == ["linear_fused", "amax", "quantize_with_amax", "gemm"], lib.calls
print(json.dumps({{"rank": rank, "h_amax_ok": True}}))
dist.destroy_process_group()
"""


def test_tp_two_gloo_ranks_share_amax_and_sum_the_down_projection():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", _RANK_SCRIPT.format(root=ROOT)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = [p.communicate(timeout=180) for p in procs]
    for p, (out, err) in zip(procs, outs):
        assert p.returncode == 0, err[-3000:]
    seen = sorted(json.loads(l)["rank"] for out, _ in outs for l in out.splitlines() if l.strip())
    assert seen == [0, 1]


def test_mlp_tensor_parallel_refuses_shares_that_split_a_block():
    """Each rank's share of the hidden size must be a multiple of 16 (one
    scale block of h must not straddle two ranks); refused before any call."""
    import pytest
    from nvfp4_block_scaled_21_b200 import tp

    class W:
        def __init__(self, rows):
            self.rows = rows

    class NoLib:
        def __getattr__(self, name):
            raise AssertionError(f"no library call expected, got {name}")

    class X:
        shape = (8, 64)
        device = "cpu"

    with pytest.raises(ValueError, match="multiple of 16"):
        tp.mlp_tensor_parallel(X(), W(40), W(40), W(64), lib=NoLib())
