#!/usr/bin/env python
"""Benchmark of the NVFP4 hot path on B200: activation quantize + W4A4
block-scaled GEMM (prefill, decode), the standalone quantizer, and the fused
MLP step.  Prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill|decode|quantize|mlp]

A step is one pass of the hot path over one batch of synthetic input already
resident in HBM.  The headline workload (default: prefill, M=4096 N=17408
K=5120) is timed over exactly K steps (CUDA-graph replays: a graph holds one
step per rotating input slot) bracketed by a barrier and a device
synchronize; the other workloads are measured the same way and reported under
"workloads".  L2 (126 MB) is defeated by rotating enough input copies that
each step's operands were evicted by the steps before it.  Multi-GPU runs are
independent batches per rank (weak scaling, no data-path collective); the
time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 1024 * 1024
# DRAM bytes read + written per launch of each workload's dominant kernel(s),
# from one ncu capture of the current kernels (dram__bytes_read.sum +
# dram__bytes_write.sum); None where the kernel changed after its capture or
# the capture did not cover every kernel of the dominant call.
NCU_TRAFFIC = {"prefill": 157_946_112, "decode": 50_260_224, "quantize": 172_837_376, "mlp": 106_699_264,
               "prefill_requant": 401_925_888, "mx_prefill": 153_014_272, "w4a16_decode": 50_272_000,
               "w4a8_prefill": 173_520_128}
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FP4_PER_BF16 = 4.0          # dense FP4 : dense BF16 on B200 (9 : 2.25 PFLOP/s nominal)
FP8_PER_BF16 = 2.0          # dense FP8 (and FP8 x FP4) : dense BF16 (4.5 : 2.25 PFLOP/s nominal)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
            "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML)
# ---------------------------------------------------------------------------
_REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}


class ClockSampler:
    def __init__(self, device_index: int, period_s: float = 0.002):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()
        self._t = None

    def _reasons_now(self):
        n = self.nvml
        f = getattr(n, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(n, "nvmlDeviceGetCurrentClocksThrottleReasons")
        return f(self.h)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
                self.reasons |= int(self._reasons_now())
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"],
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": [name for bit, name in _REASONS.items() if self.reasons & bit],
                "samples": len(self.samples),
                "window": "the timed region and the per-step replays that follow it"}


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------

def _copies(t, n):
    return [t] + [t.clone() for _ in range(n - 1)]


def _clone_q(nv, q, n):
    out = [q]
    for _ in range(n - 1):
        out.append(nv.NVFP4Tensor(q.codes.clone(), q.scales.clone(), q.tensor_scale.clone(),
                                  q.rows, q.cols))
    return out


def _workloads():
    """The seeded input generator, loaded from its file: importing it through
    the package would load libnvfp4.so, which the reference arm must not map."""
    import importlib.util
    mod = sys.modules.get("_nvfp4_workloads")
    if mod is None:
        spec = importlib.util.spec_from_file_location(
            "_nvfp4_workloads", os.path.join(ROOT, "nvfp4_block_scaled_21_b200", "workloads.py"))
        mod = importlib.util.module_from_spec(spec)
        sys.modules["_nvfp4_workloads"] = mod
        spec.loader.exec_module(mod)
    return mod


def _gen(name):
    return _workloads().make(name)


def _bf16(torch, bits):
    import numpy as np
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


class Prefill:
    name = "prefill"
    metric = "NVFP4 GEMM TFLOPS (prefill)"
    unit = "TFLOP/s"

    def __init__(self, nv, torch, data=None):
        w = data or _gen("prefill")
        self.M, self.K, self.N = w["M"], w["K"], w["N"]
        W = _bf16(torch, w["W"])
        wq = nv.quantize(W)
        del W
        X = _bf16(torch, w["X"])
        per_step = X.numel() * 2 + wq.codes.numel() + wq.scales.numel()
        self.R = max(2, -(-2 * L2_BYTES // per_step))
        self.X = _copies(X, self.R)
        self.Wq = _clone_q(nv, wq, self.R)
        self.xq = [nv.NVFP4Tensor.empty(self.M, self.K) for _ in range(self.R)]
        self.y = torch.empty((self.M, self.N), dtype=torch.bfloat16, device="cuda")
        self.wsq = nv.workspace(nv.OP_QUANTIZE, self.M, 0, self.K)
        self.wsg = nv.workspace(nv.OP_GEMM, self.M, self.N, self.K)
        self.wsl = nv.workspace(nv.OP_LINEAR_FUSED, self.M, self.N, self.K)
        self.nv, self.torch = nv, torch
        self.flops = 2.0 * self.M * self.N * self.K
        self.units = self.flops / 1e12          # TFLOP per step
        self.launches = 3                       # amax, encode, GEMM
        self.dominant = {"kernel": "gemm_nvf4_pair_kernel (CTA pair, 256x256 tiles)", "bound": "tensor",
                         "algorithmic": self.flops, "unit": "TFLOP/s"}
        self.config = {"workload": f"prefill W4A4 linear: quantize X bf16 {self.M}x{self.K} per call, "
                                   f"GEMM with pre-quantized W {self.N}x{self.K}, bf16 out",
                       "M": self.M, "N": self.N, "K": self.K,
                       "l2": f"{self.R} rotating copies of X and W_q ({self.R * per_step / 2**20:.0f} MiB) > 126 MB L2"}

    def step(self, i):
        # the public fused call: activation quantize + GEMM
        r = i % self.R
        self.nv.nvfp4_linear_fused(self.X[r], self.Wq[r], self.wsl, self.nv.EPI_STORE, y=self.y,
                                   x_q=self.xq[r])

    def dominant_call(self, i):
        r = i % self.R
        self.nv.nvfp4_gemm(self.xq[r], self.Wq[r], self.y, self.wsg)

    def e2e_setup(self):
        self.x_host = self.X[0].cpu().pin_memory()
        self.y_host = torch_empty_pinned(self.torch, self.y)
        self.h2d = self.x_host.numel() * 2
        self.d2h = self.y.numel() * 2

    def e2e_step(self, i):
        r = i % self.R
        self.X[r].copy_(self.x_host, non_blocking=True)
        self.nv.nvfp4_linear_fused(self.X[r], self.Wq[r], self.wsl, self.nv.EPI_STORE, y=self.y)
        self.y_host.copy_(self.y, non_blocking=True)

    def value(self, seconds_per_step):
        return self.units / seconds_per_step


class Decode(Prefill):
    name = "decode"
    metric = "NVFP4 GEMM GB/s (decode)"
    unit = "GB/s"

    def __init__(self, nv, torch):
        super().__init__(nv, torch, _gen("decode"))
        M, N, K = self.M, self.N, self.K
        w_bytes = N * K // 2 + N * K // 16
        # algorithmic bytes of the step: W codes + W scales, X bf16 in, Y bf16 out
        self.bytes = w_bytes + M * K * 2 + M * N * 2
        self.units = self.bytes / 1e9
        # Per step: the quantizer (one cooperative launch at this size: its
        # CTAs meet once for the amax), then the swapped GEMM (weights on the
        # MMA's M, the 8 tokens on N = 16), which streams its first weight
        # stages before the quantizer has finished.
        self.launches = 2
        self.dominant = {"kernel": "gemm_nvf4_kernel<16, swapped> (128x16 MMA tiles, four accumulators)",
                         "bound": "hbm", "algorithmic": w_bytes + M * K // 2 + M * K // 16 + M * N * 2,
                         "unit": "GB/s"}
        self.config["workload"] = (f"decode W4A4 linear: quantize X bf16 {M}x{K} per call, GEMM with "
                                   f"pre-quantized W {N}x{K}, bf16 out")
        self.config["algorithmic_bytes_per_step"] = self.bytes


class Quantize:
    name = "quantize"
    metric = "NVFP4 quantize GB/s"
    unit = "GB/s"

    def __init__(self, nv, torch):
        w = _gen("quantize")
        self.M, self.K = w["M"], w["K"]
        X = _bf16(torch, w["X"])
        self.R = max(2, -(-2 * L2_BYTES // (X.numel() * 2)))
        self.X = _copies(X, self.R)
        self.q = [nv.NVFP4Tensor.empty(self.M, self.K) for _ in range(self.R)]
        self.ws = nv.workspace(nv.OP_QUANTIZE, self.M, 0, self.K)
        self.nv, self.torch = nv, torch
        n = self.M * self.K
        # The two-pass method reads x twice (amax pass, encode pass: x is 84 MB
        # and the second read comes from DRAM again) and writes the codes, the
        # scales and the tensor scale.  The one-read lower bound is reported
        # beside it.
        self.bytes_one_read = n * 2 + n // 2 + n // 16 + 4
        self.bytes = self.bytes_one_read + n * 2
        self.units = self.bytes / 1e9
        self.launches = 2
        self.dominant = {"kernel": "amax_partials_kernel + encode_kernel", "bound": "hbm",
                         "algorithmic": self.bytes, "unit": "GB/s"}
        self.config = {"workload": f"quantize bf16 {self.M}x{self.K} to NVFP4 (codes, tiled E4M3 scales, fp32 tensor scale)",
                       "rows": self.M, "cols": self.K,
                       "algorithmic_bytes_per_step": self.bytes,
                       "one_read_lower_bound_bytes": self.bytes_one_read,
                       "l2": f"{self.R} rotating copies of x ({self.R * n * 2 / 2**20:.0f} MiB) > 126 MB L2"}

    def step(self, i):
        r = i % self.R
        self.nv.nvfp4_quantize(self.X[r], self.q[r], self.ws)

    dominant_call = step

    def e2e_setup(self):
        self.x_host = self.X[0].cpu().pin_memory()
        self.c_host = torch_empty_pinned(self.torch, self.q[0].codes)
        self.h2d = self.x_host.numel() * 2
        self.d2h = self.q[0].codes.numel() + self.q[0].scales.numel() + 4
        self.s_host = torch_empty_pinned(self.torch, self.q[0].scales)
        self.g_host = torch_empty_pinned(self.torch, self.q[0].tensor_scale)

    def e2e_step(self, i):
        r = i % self.R
        self.X[r].copy_(self.x_host, non_blocking=True)
        self.nv.nvfp4_quantize(self.X[r], self.q[r], self.ws)
        self.c_host.copy_(self.q[r].codes, non_blocking=True)
        self.s_host.copy_(self.q[r].scales, non_blocking=True)
        self.g_host.copy_(self.q[r].tensor_scale, non_blocking=True)

    def value(self, seconds_per_step):
        return self.units / seconds_per_step


class Mlp:
    name = "mlp"
    metric = "NVFP4 fused MLP GB/s (M=128)"
    unit = "GB/s"

    def __init__(self, nv, torch):
        w = _gen("mlp")
        self.M, self.K, self.N = w["M"], w["K"], w["N"]
        M, K, N = self.M, self.K, self.N
        wg, wu, wd = (nv.quantize(_bf16(torch, w[k])) for k in ("Wg", "Wu", "Wd"))
        X = _bf16(torch, w["X"])
        per_step = 3 * (N * K // 2 + N * K // 16)
        self.R = max(2, -(-2 * L2_BYTES // per_step))
        self.X = _copies(X, self.R)
        self.wg, self.wu, self.wd = (_clone_q(nv, q, self.R) for q in (wg, wu, wd))
        self.hq = nv.NVFP4Tensor.empty(M, N)
        self.y = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
        self.wsl = nv.workspace(nv.OP_LINEAR_FUSED_SILU, M, N, K)
        self.wsg = nv.workspace(nv.OP_GEMM, M, K, N)
        self.nv, self.torch = nv, torch
        hq_bytes = M * N // 2 + M * N // 16
        self.bytes = per_step + M * K * 2 + M * K * 2 + 2 * hq_bytes
        self.units = self.bytes / 1e9
        # amax and encode passes on x; gate+up GEMM, which re-quantizes h in
        # its epilogue (its 136 tiles fit the SMs); down GEMM
        self.launches = 4
        # The largest share of the step is the gate+up kernel (ncu: 31.7 us
        # against 28.9 us for the down projection).  It runs inside the
        # fused call together with the two quantizer passes on x, so the
        # roofline is taken over that call: gate and up weights, x in, h_q out.
        self.dominant = {"kernel": "gemm_nvf4_dual_kernel (gate+up, SiLU*up epilogue re-quantizing h) in the "
                                   "fused call with the quantizer passes on x",
                         "bound": "hbm",
                         "algorithmic": 2 * (N * K // 2 + N * K // 16) + M * K * 2 + hq_bytes,
                         "unit": "GB/s"}
        self.config = {"workload": f"fused MLP M={M}: quantize X, gate/up K={K} N={N}, SiLU(gate)*up "
                                   f"re-quantized to NVFP4, down K={N} N={K}, bf16 out",
                       "M": M, "K": K, "N": N, "algorithmic_bytes_per_step": self.bytes,
                       "flops_per_step": 2.0 * M * N * K * 3,
                       "l2": f"{self.R} rotating copies of the three weight matrices > 126 MB L2"}

    def step(self, i):
        r = i % self.R
        nv = self.nv
        nv.nvfp4_linear_fused(self.X[r], self.wg[r], self.wsl, nv.EPI_SILU_MUL_REQUANT,
                              w_up=self.wu[r], y_q=self.hq)
        nv.nvfp4_gemm(self.hq, self.wd[r], self.y, self.wsg)

    def dominant_call(self, i):
        r = i % self.R
        self.nv.nvfp4_linear_fused(self.X[r], self.wg[r], self.wsl, self.nv.EPI_SILU_MUL_REQUANT,
                                   w_up=self.wu[r], y_q=self.hq)

    def e2e_setup(self):
        self.x_host = self.X[0].cpu().pin_memory()
        self.y_host = torch_empty_pinned(self.torch, self.y)
        self.h2d = self.x_host.numel() * 2
        self.d2h = self.y.numel() * 2

    def e2e_step(self, i):
        r = i % self.R
        self.X[r].copy_(self.x_host, non_blocking=True)
        self.step(i)
        self.y_host.copy_(self.y, non_blocking=True)

    def value(self, seconds_per_step):
        return self.units / seconds_per_step


class PrefillRequant(Prefill):
    """The prefill linear layer whose bf16 output is also re-quantized to
    NVFP4 for the next layer (y_q of nvfp4_linear_fused's store form)."""
    name = "prefill_requant"
    metric = "NVFP4 GEMM TFLOPS (prefill, output re-quantized)"

    def __init__(self, nv, torch):
        super().__init__(nv, torch)
        self.yq = nv.NVFP4Tensor.empty(self.M, self.N)
        self.launches = 4                       # amax, encode (x); GEMM; encode (y)
        # y (bf16, 142.6 MB) is read once more by the encode pass, which also
        # writes y_q's codes and scales
        self.requant_bytes = self.M * self.N * 2 + self.M * self.N // 2 + self.M * self.N // 16 + 4
        self.dominant = {"kernel": "the fused call: x quantizer passes, gemm_nvf4_pair_kernel with per-CTA "
                                   "max |y|, y encode pass", "bound": "tensor", "algorithmic": self.flops,
                         "unit": "TFLOP/s"}
        self.config = dict(self.config, workload=f"prefill W4A4 linear with y re-quantized: quantize X bf16 "
                                                 f"{self.M}x{self.K}, GEMM with W {self.N}x{self.K}, bf16 y "
                                                 f"and NVFP4 y_q", requant_pass_bytes=self.requant_bytes)

    def step(self, i):
        r = i % self.R
        self.nv.nvfp4_linear_fused(self.X[r], self.Wq[r], self.wsl, self.nv.EPI_STORE, y=self.y, y_q=self.yq,
                                   x_q=self.xq[r])

    dominant_call = step

    def e2e_setup(self):
        super().e2e_setup()
        self.c_host = torch_empty_pinned(self.torch, self.yq.codes)
        self.d2h += self.yq.codes.numel()

    def e2e_step(self, i):
        r = i % self.R
        self.X[r].copy_(self.x_host, non_blocking=True)
        self.nv.nvfp4_linear_fused(self.X[r], self.Wq[r], self.wsl, self.nv.EPI_STORE, y=self.y, y_q=self.yq)
        self.y_host.copy_(self.y, non_blocking=True)
        self.c_host.copy_(self.yq.codes, non_blocking=True)


class MxPrefill:
    """MXFP4 variant of the prefill GEMM: one-pass MXFP4 quantize of X
    (32-value blocks, E8M0 scales, no tensor scale) and the kind::mxf4
    block-scaled GEMM with pre-quantized MXFP4 weights."""
    name = "mx_prefill"
    metric = "MXFP4 GEMM TFLOPS (prefill)"
    unit = "TFLOP/s"

    def __init__(self, nv, torch):
        w = _gen("prefill")
        self.M, self.K, self.N = w["M"], w["K"], w["N"]
        W = _bf16(torch, w["W"])
        wq = nv.mx_quantize(W)
        del W
        X = _bf16(torch, w["X"])
        per_step = X.numel() * 2 + wq.codes.numel() + wq.scales.numel()
        self.R = max(2, -(-2 * L2_BYTES // per_step))
        self.X = _copies(X, self.R)
        self.Wq = [wq] + [nv.MXFP4Tensor(wq.codes.clone(), wq.scales.clone(), wq.rows, wq.cols)
                          for _ in range(self.R - 1)]
        self.xq = [nv.MXFP4Tensor.empty(self.M, self.K) for _ in range(self.R)]
        self.y = torch.empty((self.M, self.N), dtype=torch.bfloat16, device="cuda")
        self.ws = nv.workspace(nv.OP_GEMM, self.M, self.N, self.K)
        self.nv, self.torch = nv, torch
        self.flops = 2.0 * self.M * self.N * self.K
        self.units = self.flops / 1e12
        self.launches = 2                       # MX quantize, GEMM
        self.dominant = {"kernel": "gemm_nvf4_pair_kernel<MX> (kind::mxf4, CTA pair, 256x256 tiles)",
                         "bound": "tensor", "algorithmic": self.flops, "unit": "TFLOP/s"}
        self.config = {"workload": f"MXFP4 prefill linear: quantize X bf16 {self.M}x{self.K} to MXFP4 per call, "
                                   f"GEMM with pre-quantized MXFP4 W {self.N}x{self.K}, bf16 out",
                       "M": self.M, "N": self.N, "K": self.K,
                       "l2": f"{self.R} rotating copies of X and W_q > 126 MB L2"}

    def step(self, i):
        r = i % self.R
        self.nv.nvfp4_mx_quantize(self.X[r], self.xq[r])
        self.nv.nvfp4_mx_gemm(self.xq[r], self.Wq[r], self.y, self.ws)

    def dominant_call(self, i):
        r = i % self.R
        self.nv.nvfp4_mx_gemm(self.xq[r], self.Wq[r], self.y, self.ws)

    def e2e_setup(self):
        self.x_host = self.X[0].cpu().pin_memory()
        self.y_host = torch_empty_pinned(self.torch, self.y)
        self.h2d = self.x_host.numel() * 2
        self.d2h = self.y.numel() * 2

    def e2e_step(self, i):
        r = i % self.R
        self.X[r].copy_(self.x_host, non_blocking=True)
        self.step(i)
        self.y_host.copy_(self.y, non_blocking=True)

    def value(self, seconds_per_step):
        return self.units / seconds_per_step


class W4A8Prefill:
    """W4A8 at the prefill shape: MXFP4 weights times MXFP8 activations (E4M3
    elements, one E8M0 scale per 32), the activations quantized per call
    inside nvfp4_w4a8_linear, then the kind::mxf8f6f4 block-scaled GEMM, which
    runs at the FP8 tensor rate."""
    name = "w4a8_prefill"
    metric = "W4A8 GEMM TFLOPS (prefill)"
    unit = "TFLOP/s"

    def __init__(self, nv, torch):
        w = _gen("prefill")
        self.M, self.K, self.N = w["M"], w["K"], w["N"]
        W = _bf16(torch, w["W"])
        wq = nv.mx_quantize(W)
        del W
        X = _bf16(torch, w["X"])
        per_step = X.numel() * 2 + wq.codes.numel() + wq.scales.numel()
        self.R = max(2, -(-2 * L2_BYTES // per_step))
        self.X = _copies(X, self.R)
        self.Wq = [wq] + [nv.MXFP4Tensor(wq.codes.clone(), wq.scales.clone(), wq.rows, wq.cols)
                          for _ in range(self.R - 1)]
        self.xq = [nv.MXFP8Tensor.empty(self.M, self.K) for _ in range(self.R)]
        self.y = torch.empty((self.M, self.N), dtype=torch.bfloat16, device="cuda")
        self.wsl = nv.workspace(nv.OP_W4A8_LINEAR, self.M, self.N, self.K)
        self.wsg = nv.workspace(nv.OP_GEMM, self.M, self.N, self.K)
        self.nv, self.torch = nv, torch
        self.flops = 2.0 * self.M * self.N * self.K
        self.units = self.flops / 1e12
        self.launches = 2                       # MXFP8 quantize, GEMM
        self.dominant = {"kernel": "gemm_nvf4_pair_kernel<W4A8> (kind::mxf8f6f4, CTA pair, 256x256 tiles)",
                         "bound": "tensor", "algorithmic": self.flops, "unit": "TFLOP/s",
                         "per_bf16": FP8_PER_BF16, "peak_name": "dense FP8"}
        self.config = {"workload": f"W4A8 prefill linear: quantize X bf16 {self.M}x{self.K} to MXFP8 per call, "
                                   f"GEMM with pre-quantized MXFP4 W {self.N}x{self.K}, bf16 out",
                       "M": self.M, "N": self.N, "K": self.K,
                       "l2": f"{self.R} rotating copies of X and W_q > 126 MB L2"}

    def step(self, i):
        r = i % self.R
        self.nv.nvfp4_w4a8_linear(self.X[r], self.Wq[r], self.y, self.wsl, x_q=self.xq[r])

    def dominant_call(self, i):
        r = i % self.R
        self.nv.nvfp4_w4a8_gemm(self.xq[r], self.Wq[r], self.y, self.wsg)

    def e2e_setup(self):
        self.x_host = self.X[0].cpu().pin_memory()
        self.y_host = torch_empty_pinned(self.torch, self.y)
        self.h2d = self.x_host.numel() * 2
        self.d2h = self.y.numel() * 2

    def e2e_step(self, i):
        r = i % self.R
        self.X[r].copy_(self.x_host, non_blocking=True)
        self.step(i)
        self.y_host.copy_(self.y, non_blocking=True)

    def value(self, seconds_per_step):
        return self.units / seconds_per_step


class W4A16Decode:
    """The W4A16 comparison scheme at the decode shape: bf16 activations, the
    same NVFP4 weights dequantized inside the kernel before bf16 MMAs."""
    name = "w4a16_decode"
    metric = "W4A16 GEMM GB/s (decode)"
    unit = "GB/s"

    def __init__(self, nv, torch):
        w = _gen("decode")
        self.M, self.K, self.N = w["M"], w["K"], w["N"]
        M, N, K = self.M, self.N, self.K
        W = _bf16(torch, w["W"])
        wq = nv.quantize(W)
        del W
        X = _bf16(torch, w["X"])
        w_bytes = N * K // 2 + N * K // 16
        self.R = max(2, -(-2 * L2_BYTES // w_bytes))
        self.X = _copies(X, self.R)
        self.Wq = _clone_q(nv, wq, self.R)
        self.y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        self.ws = nv.workspace(nv.OP_W4A16, M, N, K)
        self.nv, self.torch = nv, torch
        self.bytes = w_bytes + M * K * 2 + M * N * 2
        self.units = self.bytes / 1e9
        self.launches = 1
        self.dominant = {"kernel": "gemm_w4a16_kernel (weights dequantized into tensor memory, bf16 MMA)",
                         "bound": "hbm", "algorithmic": self.bytes, "unit": "GB/s"}
        self.config = {"workload": f"W4A16 decode linear: bf16 X {M}x{K}, NVFP4 W {N}x{K} dequantized in-kernel, "
                                   f"bf16 out", "M": M, "N": N, "K": K, "algorithmic_bytes_per_step": self.bytes,
                       "l2": f"{self.R} rotating copies of W_q > 126 MB L2"}

    def step(self, i):
        r = i % self.R
        self.nv.nvfp4_w4a16_linear(self.X[r], self.Wq[r], self.y, self.ws)

    dominant_call = step

    def e2e_setup(self):
        self.x_host = self.X[0].cpu().pin_memory()
        self.y_host = torch_empty_pinned(self.torch, self.y)
        self.h2d = self.x_host.numel() * 2
        self.d2h = self.y.numel() * 2

    def e2e_step(self, i):
        r = i % self.R
        self.X[r].copy_(self.x_host, non_blocking=True)
        self.step(i)
        self.y_host.copy_(self.y, non_blocking=True)

    def value(self, seconds_per_step):
        return self.units / seconds_per_step


WORKLOADS = {"prefill": Prefill, "decode": Decode, "quantize": Quantize, "mlp": Mlp,
             "prefill_requant": PrefillRequant, "mx_prefill": MxPrefill, "w4a16_decode": W4A16Decode,
             "w4a8_prefill": W4A8Prefill}


def torch_empty_pinned(torch, like):
    return torch.empty(like.shape, dtype=like.dtype, pin_memory=True)


# ---------------------------------------------------------------------------
# measurement
# ---------------------------------------------------------------------------

def dist_setup(backend=None):
    """One process per GPU from torchrun's environment.  NCCL on GPUs; gloo
    (CPU tensors) when asked for or when there is no GPU (host-side tests)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        if backend is None:
            backend = "nccl" if torch.cuda.is_available() else "gloo"
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, value):
    """The largest of every rank's value (each rank's device time)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def emit(line, rank):
    """Rank 0 alone prints the result line."""
    if rank == 0:
        print(json.dumps(line), flush=True)


def dist_teardown(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def _capture(torch, fn, n):
    """One CUDA graph per rotation slot, each holding one call of fn(slot)."""
    graphs = []
    for r in range(n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn(r)
        graphs.append(g)
    torch.cuda.synchronize()
    return graphs


def _capture_rotation(torch, fn, n):
    """One CUDA graph holding fn(0), fn(1), ..., fn(n-1): a full rotation of
    the input slots, so consecutive steps run without a graph launch between
    them (as consecutive layers would inside one captured forward pass)."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for r in range(n):
            fn(r)
    torch.cuda.synchronize()
    return g


def _replay_k(singles, rotation, R, K):
    """Exactly K steps starting at slot 0: full rotations, then single steps."""
    for _ in range(K // R):
        rotation.replay()
    for i in range(K % R):
        singles[i].replay()


def measure(wl, torch, K, W, world, local, sample_clocks=False):
    """Device time of exactly K steps (CUDA-graph replays of whole rotations of
    the input slots, then single steps for K mod R), bracketed by barrier +
    synchronize; the per-step distribution from K single-step replays, each
    between its own events; then the dominant kernel alone over K calls the
    same way."""
    for i in range(W):                       # eager warm-up (also resolves lazy set-up)
        wl.step(i)
    torch.cuda.synchronize()
    steps = _capture(torch, wl.step, wl.R)
    kern = _capture(torch, wl.dominant_call, wl.R)
    steps_rot = _capture_rotation(torch, wl.step, wl.R)
    kern_rot = _capture_rotation(torch, wl.dominant_call, wl.R)
    for i in range(W):
        steps[i % wl.R].replay()
    steps_rot.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    # NVML clocks are sampled from the start of the timed region to the end of
    # the per-step replays that follow it under the same load (the timed
    # region alone can be a few milliseconds, shorter than one sample period)
    sampler = ClockSampler(local) if sample_clocks else None
    if sampler:
        sampler.__enter__()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    _replay_k(steps, steps_rot, wl.R, K)
    end.record()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    elapsed = max_over_ranks(world, start.elapsed_time(end) / 1e3)
    # per-step distribution (this rank): K more replays, each between its own events
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for i in range(K):
        evs[i][0].record()
        steps[(W + i) % wl.R].replay()
        evs[i][1].record()
    torch.cuda.synchronize()
    if sampler:
        sampler.__exit__(None, None, None)
    per = sorted(a.elapsed_time(b) * 1e3 for a, b in evs)
    dist = {"median": round(per[K // 2], 2), "p10": round(per[int(0.1 * (K - 1))], 2),
            "p90": round(per[int(0.9 * (K - 1))], 2), "unit": "us", "rank": "local"}
    for i in range(W):
        kern[i % wl.R].replay()
    kern_rot.replay()
    torch.cuda.synchronize()
    ks, ke = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ks.record()
    _replay_k(kern, kern_rot, wl.R, K)
    ke.record()
    torch.cuda.synchronize()
    kern_us = max_over_ranks(world, ks.elapsed_time(ke) * 1e3 / K)
    del steps, kern, steps_rot, kern_rot
    return elapsed, kern_us, (sampler.summary() if sampler else None), dist


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def measure_e2e(wl, torch, K, world):
    wl.e2e_setup()
    for i in range(2):
        wl.e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(K):
        wl.e2e_step(i)
    end.record()
    torch.cuda.synchronize()
    barrier(world)
    return max_over_ranks(world, start.elapsed_time(end) / 1e3)


def roofline(wl, kern_us, peaks):
    d = wl.dominant
    if d["bound"] == "tensor":
        ratio = d.get("per_bf16", FP4_PER_BF16)
        achieved = d["algorithmic"] / (kern_us * 1e-6) / 1e12
        peak = peaks["bf16_tflops"] * ratio
        unit = "TFLOP/s"
        peak_note = (f"{d.get('peak_name', 'dense FP4')} = {ratio:g} x {peaks['source']} bf16 burst "
                     f"{peaks['bf16_tflops']:.1f} TFLOP/s")
    else:
        achieved = d["algorithmic"] / (kern_us * 1e-6) / 1e9
        peak = peaks["hbm_gbs"]
        unit = "GB/s"
        peak_note = f"{peaks['source']} HBM copy bandwidth"
    return {"bound": d["bound"], "achieved": round(achieved, 1), "peak": round(peak, 1),
            "unit": unit, "frac": round(achieved / peak, 4), "traffic": NCU_TRAFFIC.get(wl.name),
            "kernel": d["kernel"], "kernel_us": round(kern_us, 2),
            "algorithmic_per_launch": d["algorithmic"], "peak_source": peak_note}


# ---------------------------------------------------------------------------
# CPU baseline: the oracle as it stands, on a bounded sample
# ---------------------------------------------------------------------------

def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def cpu_oracle_prefill(rows: int):
    """Oracle time for quantizing `rows` activation rows and their fp64 GEMM
    against the whole pre-quantized weight (prefill workload, seed 3)."""
    import numpy as np
    import oracle
    w = _gen("prefill")
    wq = oracle.quantize(w["W"])                     # pre-quantized weights: untimed
    xs = w["X"][:rows]
    t0 = time.perf_counter()
    xq = oracle.quantize(xs)
    oracle.gemm_f64(xq, wq)
    dt = time.perf_counter() - t0
    flops = 2.0 * rows * w["N"] * w["K"]
    threads = oracle_threads(rows)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": threads,
            "cpu_model": _cpu_model(), "kind": "oracle", "seconds": round(dt, 2),
            "sample": f"prefill workload: oracle quantize of {rows} of 4096 X rows + fp64 GEMM of "
                      f"those rows against all 17408 pre-quantized W rows (K=5120); the GEMM on "
                      f"{threads} threads, quantize and dequantize on one"}


def oracle_threads(rows: int) -> int:
    """Threads the oracle's fp64 GEMM runs on: it splits output rows over at
    most one thread per host core (its quantize and dequantize use one)."""
    return max(1, min(os.cpu_count() or 1, rows))


def reference_arm(args):
    """--impl reference: the CPU oracle timed on this host, K steps of a
    bounded sample of the headline workload."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    w = _gen(args.workload if args.workload in ("prefill", "decode") else "prefill")
    wq = oracle.quantize(w["W"])                  # pre-quantized weights: untimed, as on the GPU
    # Each step is a bounded sample of the workload: `rows` activation rows
    # against one eighth of W, rotating through both, so that the default
    # 110 steps end within about a minute (the oracle's GEMM dequantizes its
    # whole weight operand to fp64 on one thread on every call).
    rows, w_rows = min(8, w["M"]), w["N"] // 8
    times = []
    for i in range(args.warmup + args.steps):
        r0 = (i * rows) % w["M"]
        n0 = (i % 8) * w_rows
        wslice = oracle.Quantized(wq.codes[n0:n0 + w_rows], wq.scales[n0:n0 + w_rows], wq.g, w_rows, w["K"])
        t0 = time.perf_counter()
        xq = oracle.quantize(w["X"][r0:r0 + rows])
        oracle.gemm_f64(xq, wslice)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    per_step = sum(times) / len(times)
    flops = 2.0 * rows * w_rows * w["K"]
    v = flops / per_step / 1e12
    line = {"impl": "reference", "metric": "NVFP4 GEMM TFLOPS (prefill)", "value": v,
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": per_step * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded numpy PCG64)",
            "config": {"workload": f"{w['name']} W4A4 linear, CPU oracle: each step quantizes "
                                   f"{rows} X rows and runs their fp64 GEMM against {w_rows} of the "
                                   f"{w['N']} pre-quantized W rows (K={w['K']})"},
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": oracle_threads(rows),
                             "cpu_model": _cpu_model(), "kind": "oracle",
                             "sample": f"{rows} X rows x {w_rows} W rows per step, rotating over the "
                                       f"workload; the GEMM on {oracle_threads(rows)} threads, quantize "
                                       f"and dequantize on one"},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    emit(line, rank)
    return 0


def device_info(torch, index):
    """Name, compute capability, CUDA runtime and driver of the measured GPU
    (for the record; any field that cannot be read is None)."""
    info = {"name": None, "cc": None, "cuda_runtime": getattr(torch.version, "cuda", None), "driver": None}
    try:
        info["name"] = torch.cuda.get_device_name(index)
        info["cc"] = "%d.%d" % torch.cuda.get_device_capability(index)
    except Exception:
        pass
    try:
        import pynvml
        pynvml.nvmlInit()
        d = pynvml.nvmlSystemGetDriverVersion()
        info["driver"] = d.decode() if isinstance(d, bytes) else d
    except Exception:
        pass
    return info


def workload_result(wl, value, sps, dist, kern_us, e2e_value, steps, peaks):
    """One workload's measured entry: metric value, step time and spread, the
    dominant kernel's roofline, the end-to-end figure and the launch count."""
    return {"metric": wl.metric, "value": round(value, 2), "unit": wl.unit,
            "ms_per_step": round(sps * 1e3, 4), "step_us": dist, "config": wl.config,
            "roofline": roofline(wl, kern_us, peaks),
            "e2e": {"value": round(e2e_value, 3), "unit": wl.unit,
                    "h2d_bytes_per_step": wl.h2d, "d2h_bytes_per_step": wl.d2h},
            "gpu_launches": wl.launches * steps}


def result_line(head, results, world, steps, warmup, peaks):
    """The one JSON line: the headline workload's measurement (`head`, one
    entry of the per-workload results) with the run's parameters; the other
    workloads under "workloads"."""
    return {"metric": head["metric"], "value": head["value"], "unit": head["unit"],
            "n_gpus": world, "steps": steps, "warmup": warmup,
            "ms_per_step": head["ms_per_step"], "step_us": head["step_us"],
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4",
            "data": "synthetic (seeded numpy PCG64: N(0,1) activations with 0.1% x50 outliers, "
                    "N(0,0.02) weights, bf16)",
            "config": dict(head["config"], parallelism=f"independent batch per GPU x{world}"),
            "roofline": head["roofline"], "e2e": head["e2e"], "gpu_launches": head["gpu_launches"],
            "clocks": head["clocks"], "workloads": results,
            "peaks": peaks}


def _build_library():
    """Compile libnvfp4.so in-tree if it is missing or stale (nvcc)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_nvfp4_build", os.path.join(ROOT, "nvfp4_block_scaled_21_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(WORKLOADS), default="prefill")
    ap.add_argument("--only", action="store_true", help="measure the headline workload only")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=1024)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return reference_arm(args)

    world, rank, local = dist_setup()
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}; using {world}", file=sys.stderr)
    import torch
    torch.cuda.set_device(local)
    _build_library()
    import nvfp4_block_scaled_21_b200 as nv

    peaks = load_peaks()
    names = [args.workload] + ([] if args.only else [n for n in WORKLOADS if n != args.workload])
    results = {}
    head = None
    for n in names:
        wl = WORKLOADS[n](nv, torch)
        is_head = n == args.workload
        elapsed, kern_us, clocks, dist = measure(wl, torch, args.steps, args.warmup, world, local,
                                                 sample_clocks=is_head)
        sps = elapsed / args.steps
        value = wl.value(sps) * world
        e2e_steps = min(args.steps, 20)
        e2e_elapsed = measure_e2e(wl, torch, e2e_steps, world)
        e2e_value = wl.value(e2e_elapsed / e2e_steps) * world
        res = workload_result(wl, value, sps, dist, kern_us, e2e_value, args.steps, peaks)
        if is_head:
            head = res
            head["clocks"] = clocks
        else:
            results[n] = res
        del wl
        torch.cuda.empty_cache()

    line = result_line(head, results, world, args.steps, args.warmup, peaks)
    line["device"] = device_info(torch, local)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.workload == "prefill":
        line["cpu_baseline"] = cpu_oracle_prefill(args.cpu_rows)
    emit(line, rank)
    dist_teardown(world)
    return 0


if __name__ == "__main__":
    sys.exit(main())
