"""Host-side multi-rank logic of bench.py on CPU (gloo, world size 2).

bench.py runs one process per GPU; every rank times its own independent batch
(weak scaling, no data-path collective) and the reported time is the maximum
over ranks, printed by rank 0 alone.  These tests run that plumbing without a
GPU: two gloo ranks exercise setup, the barrier and the max-over-ranks
reduction, and a torchrun launch of the reference arm checks that exactly one
result line appears and every rank exits 0.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


_RANK_SCRIPT = r"""
import os, sys
sys.path.insert(0, {root!r})
import bench
world, rank, local = bench.dist_setup(backend="gloo")
assert world == 2 and rank in (0, 1) and local == rank
bench.barrier(world)
got = bench.max_over_ranks(world, 1.5 + rank)     # rank 0: 1.5, rank 1: 2.5
assert got == 2.5, got
got = bench.max_over_ranks(world, 10.0 - rank)    # the max may come from rank 0
assert got == 10.0, got
bench.emit({{"rank_seen": rank, "max": got}}, rank)
bench.dist_teardown(world)
"""


def test_gloo_two_ranks_barrier_and_max():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2",
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", _RANK_SCRIPT.format(root=ROOT)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = [p.communicate(timeout=120) for p in procs]
    for p, (out, err) in zip(procs, outs):
        assert p.returncode == 0, err[-2000:]
    lines = [json.loads(l) for out, _ in outs for l in out.splitlines() if l.strip()]
    assert lines == [{"rank_seen": 0, "max": 10.0}]          # rank 0 alone printed


@pytest.mark.timeout(600)
def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["cores"] == min(os.cpu_count(), 8)         # 8 rows: 8 GEMM threads at most
    assert line["e2e"]["h2d_bytes_per_step"] == 0
