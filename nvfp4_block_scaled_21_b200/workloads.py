"""Seeded synthetic inputs for the five NVFP4 workloads.

This module holds the shapes, seeds and value distributions of the workloads
and nothing of the quantization or GEMM arithmetic; it feeds both the CUDA path
and the CPU oracle.  The distributions follow the pages' motivation for FP4:
bell-shaped values plus heavy-tail outliers that a 4-bit floating grid with a
fine block scale captures better than INT4 (eefocus.com article on FP4 vs INT4,
section "为什么FP4是更合适的压缩方案？").

Draw recipe (numpy ``Generator(PCG64(seed))``, in this order):
  weights first, then activations; each tensor is float64 normals scaled by its
  standard deviation, cast to fp32, then (bf16 workloads) rounded to bf16 by
  round-to-nearest-even.  Activation outliers: ``k = round(1e-3 * numel)``
  positions from ``rng.choice(numel, k, replace=False)`` take
  ``rng.standard_normal(k) * 50``.  The tiny workload instead sets 4 positions
  per tensor to ``40 * rng.choice([-1, 1], 4)``.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    M: int          # activation rows (tokens)
    K: int          # reduction length
    N: int          # weight rows (output features); 0 for quantize-only
    dtype: str      # "f32" or "bf16" input precision
    description: str
    extra: dict = field(default_factory=dict)


TINY = Workload("tiny", 0, 16, 256, 64, "f32",
                "X fp32 16x256, W fp32 64x256, N(0,1) with 4 +-40 outliers each; Y = X W^T fp32")
QUANTIZE = Workload("quantize", 1, 8192, 5120, 0, "bf16",
                    "bf16 8192x5120, N(0,1) with 0.1% N(0,1)*50 outliers -> NVFP4")
DECODE = Workload("decode", 2, 8, 5120, 17408, "bf16",
                  "W4A4 GEMM M=8 K=5120 N=17408; W N(0,0.02) pre-quantized; X N(0,1)+0.1% x50 quantized per call; bf16 out")
PREFILL = Workload("prefill", 3, 4096, 5120, 17408, "bf16",
                   "W4A4 GEMM M=4096 K=5120 N=17408; X quantized per call; bf16 out")
MLP = Workload("mlp", 4, 128, 5120, 17408, "bf16",
               "fused MLP M=128: gate/up K=5120 N=17408, SiLU(gate)*up re-quantized, down K=17408 N=5120 -> bf16")

ALL = {w.name: w for w in (TINY, QUANTIZE, DECODE, PREFILL, MLP)}


def _to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (RNE, by torch) and return the uint16 bit patterns."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x32, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _normal(rng, shape, std):
    return (rng.standard_normal(shape) * std).astype(np.float32)


def _with_outliers(rng, x32: np.ndarray, frac: float = 1e-3, mult: float = 50.0):
    k = int(round(frac * x32.size))
    if k:
        idx = rng.choice(x32.size, k, replace=False)
        x32.reshape(-1)[idx] = (rng.standard_normal(k) * mult).astype(np.float32)
    return x32


def _tiny_tensor(rng, shape):
    x = _normal(rng, shape, 1.0)
    idx = rng.choice(x.size, 4, replace=False)
    x.reshape(-1)[idx] = (40.0 * rng.choice([-1, 1], 4)).astype(np.float32)
    return x


def activations(rng, M: int, K: int, dtype: str = "bf16"):
    x = _with_outliers(rng, _normal(rng, (M, K), 1.0))
    return _to_bf16_bits(x) if dtype == "bf16" else x


def weights(rng, N: int, K: int, dtype: str = "bf16", std: float = 0.02):
    w = _normal(rng, (N, K), std)
    return _to_bf16_bits(w) if dtype == "bf16" else w


def make(name: str, M: int | None = None, K: int | None = None,
         N: int | None = None, seed: int | None = None) -> dict:
    """Inputs of a workload as numpy arrays (bf16 as uint16 bit patterns).

    Sizes and seed may be overridden to make reduced parity cases with the
    same distributions.  Returns a dict with the arrays and their shapes.
    """
    w = ALL[name]
    M = w.M if M is None else M
    K = w.K if K is None else K
    N = w.N if N is None else N
    seed = w.seed if seed is None else seed
    rng = np.random.Generator(np.random.PCG64(seed))
    out = {"name": name, "M": M, "K": K, "N": N, "seed": seed, "dtype": w.dtype}
    if name == "tiny":
        out["W"] = _tiny_tensor(rng, (N, K))
        out["X"] = _tiny_tensor(rng, (M, K))
    elif name == "quantize":
        out["X"] = activations(rng, M, K, w.dtype)
    elif name in ("decode", "prefill"):
        out["W"] = weights(rng, N, K, w.dtype)
        out["X"] = activations(rng, M, K, w.dtype)
    elif name == "mlp":
        out["Wg"] = weights(rng, N, K, w.dtype)
        out["Wu"] = weights(rng, N, K, w.dtype)
        out["Wd"] = weights(rng, K, N, w.dtype)
        out["X"] = activations(rng, M, K, w.dtype)
    else:
        raise KeyError(name)
    return out
