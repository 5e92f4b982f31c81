"""Host-side arithmetic of bench.py, no GPU: the exactly-K replay schedule and
the roofline numbers."""
import importlib
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
bench = importlib.import_module("bench")


class _Graph:
    def __init__(self, log, slots):
        self.log, self.slots = log, slots

    def replay(self):
        self.log.extend(self.slots)


@pytest.mark.parametrize("R", [1, 2, 3, 4, 6])
@pytest.mark.parametrize("K", [0, 1, 2, 5, 7, 20, 100])
def test_replay_k_times_exactly_k_steps_in_slot_order(R, K):
    log = []
    singles = [_Graph(log, [r]) for r in range(R)]
    rotation = _Graph(log, list(range(R)))
    bench._replay_k(singles, rotation, R, K)
    assert len(log) == K                       # exactly K steps
    assert log == [i % R for i in range(K)]    # every step on the next slot in turn


class _Wl:
    name = "prefill"

    def __init__(self, bound, algorithmic):
        self.dominant = {"kernel": "k", "bound": bound, "algorithmic": algorithmic, "unit": "x"}


def test_roofline_tensor_and_hbm():
    peaks = {"hbm_gbs": 6536.7, "bf16_tflops": 1656.9, "bf16_tflops_sustained": 1387.5, "source": "measured"}
    r = bench.roofline(_Wl("tensor", 730_144_440_320), 164.9, peaks)
    assert r["unit"] == "TFLOP/s" and r["bound"] == "tensor"
    assert r["peak"] == pytest.approx(4 * 1656.9, abs=0.1)     # dense FP4 = 4 x bf16
    assert r["achieved"] == pytest.approx(730_144_440_320 / 164.9e-6 / 1e12, abs=0.1)
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], abs=1e-3)
    r = bench.roofline(_Wl("hbm", 50_436_608), 12.7, peaks)
    assert r["unit"] == "GB/s" and r["peak"] == pytest.approx(6536.7)
    assert r["achieved"] == pytest.approx(50_436_608 / 12.7e-6 / 1e9, abs=0.1)
    assert "traffic" in r


class _FakeWl:
    name = "prefill"
    metric = "NVFP4 GEMM TFLOPS (prefill)"
    unit = "TFLOP/s"
    config = {"workload": "prefill W4A4 linear", "M": 4096, "N": 17408, "K": 5120, "l2": "rotating copies"}
    dominant = {"kernel": "k", "bound": "tensor", "algorithmic": 730_144_440_320, "unit": "TFLOP/s"}
    h2d, d2h, launches = 41_943_040, 142_606_336, 3


def test_result_line_has_every_contract_key():
    """The JSON line the driver parses: every key of the measurement contract
    with the right types, the roofline and e2e sub-objects, and a round trip
    through json."""
    import json
    peaks = {"hbm_gbs": 6536.7, "bf16_tflops": 1656.9, "bf16_tflops_sustained": 1387.5, "source": "measured"}
    dist = {"median": 180.0, "p10": 179.5, "p90": 181.0, "unit": "us", "rank": "local"}
    head = bench.workload_result(_FakeWl(), 4067.5, 179.5e-6, dist, 164.9, 198.7, 100, peaks)
    head["clocks"] = {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": [], "samples": 7}
    line = bench.result_line(head, {"decode": dict(head)}, 1, 100, 10, peaks)
    line["cpu_baseline"] = {"value": 0.02, "unit": "TFLOP/s", "cores": 16, "kind": "oracle", "sample": "1024 rows"}
    line = json.loads(json.dumps(line))
    for k, t in [("metric", str), ("value", float), ("unit", str), ("n_gpus", int), ("steps", int),
                 ("warmup", int), ("ms_per_step", float), ("higher_is_better", bool), ("scaling", str),
                 ("dtype", str), ("data", str), ("config", dict), ("roofline", dict), ("e2e", dict),
                 ("gpu_launches", int), ("clocks", dict), ("cpu_baseline", dict)]:
        assert isinstance(line[k], t), k
    assert line["vs_baseline"] is None and line["scaling"] == "weak" and line["higher_is_better"] is True
    assert line["gpu_launches"] == 300 and line["ms_per_step"] == pytest.approx(0.1795)
    assert "workload" in line["config"] and "model" not in line["config"]
    assert set(line["roofline"]) >= {"bound", "achieved", "peak", "unit", "frac", "traffic"}
    assert set(line["e2e"]) >= {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"}
    assert set(line["clocks"]) >= {"sm_mhz", "sm_max_mhz", "reasons"}
    assert set(line["cpu_baseline"]) >= {"value", "unit", "cores", "kind", "sample"}
    assert line["roofline"]["frac"] == pytest.approx(line["roofline"]["achieved"] / line["roofline"]["peak"], abs=1e-3)


def test_device_info_never_raises():
    """The device record in the line: every field present, None where it
    cannot be read (as on a machine without a GPU)."""
    import torch
    info = bench.device_info(torch, 0)
    assert set(info) == {"name", "cc", "cuda_runtime", "driver"}


def test_reference_arm_inputs_do_not_load_the_library():
    """The reference arm builds its inputs with the seeded generator loaded
    from its file, so the process never maps libnvfp4.so."""
    import subprocess
    import sys
    code = ("import sys; sys.path.insert(0, '.'); import bench; bench._gen('tiny'); "
            "maps = open('/proc/self/maps').read(); print('libnvfp4' in maps, 'nvfp4_block_scaled_21_b200' in sys.modules)")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.split() == ["False", "False"], r.stdout
