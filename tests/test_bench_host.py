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
