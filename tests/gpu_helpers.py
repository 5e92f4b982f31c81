"""Helpers shared by the GPU parity tests (test side only).

The tiled scale layout is re-derived here with the test's own index function,
independently of the CUDA kernels: block kb of row r lives at
((r//128)*(KB4//4) + kb//4)*512 + (r%32)*16 + ((r//32)%4)*4 + kb%4.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle


def tiled_scales(scales_rowmajor: np.ndarray) -> np.ndarray:
    """Map oracle scales [R][KB] to the padded tiled byte layout."""
    R, KB = scales_rowmajor.shape
    R128 = -(-R // 128) * 128
    KB4 = -(-KB // 4) * 4
    out = np.zeros(R128 * KB4, np.uint8)
    r = np.arange(R)[:, None]
    kb = np.arange(KB)[None, :]
    off = ((r // 128) * (KB4 // 4) + kb // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + kb % 4
    out[off.ravel()] = scales_rowmajor.ravel()
    return out


def untile_scales(tiled: np.ndarray, R: int, KB: int) -> np.ndarray:
    KB4 = -(-KB // 4) * 4
    r = np.arange(R)[:, None]
    kb = np.arange(KB)[None, :]
    off = ((r // 128) * (KB4 // 4) + kb // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + kb % 4
    return tiled[off]


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def f32_tensor(x: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


def upload(q: "oracle.Quantized", nv, device="cuda"):
    """An NVFP4Tensor on the GPU holding the oracle's quantization (for tests
    that feed oracle operands to the GEMM)."""
    t = nv.NVFP4Tensor.empty(q.rows, q.cols, device=device)
    t.codes.copy_(torch.from_numpy(q.codes))
    t.scales.copy_(torch.from_numpy(tiled_scales(q.scales)))
    t.tensor_scale[0] = float(q.g)
    return t


def assert_quantized_equal(gpu, q: "oracle.Quantized"):
    """Bit-exact comparison of a GPU NVFP4Tensor with the oracle's result."""
    torch.cuda.synchronize()
    g = gpu.tensor_scale[0:1].cpu().numpy()
    assert g.view(np.uint32)[0] == np.float32(q.g).view(np.uint32), (g[0], q.g)
    codes = gpu.codes.cpu().numpy()
    if not np.array_equal(codes, q.codes):
        bad = np.argwhere(codes != q.codes)
        r, c = bad[0]
        raise AssertionError(f"{len(bad)} code bytes differ; first at [{r},{c}]: "
                             f"gpu {codes[r, c]:#04x} oracle {q.codes[r, c]:#04x}")
    sc = gpu.scales.cpu().numpy()
    want = tiled_scales(q.scales)
    if not np.array_equal(sc, want):
        bad = np.flatnonzero(sc != want)
        raise AssertionError(f"{len(bad)} scale bytes differ; first at {bad[0]}: "
                             f"gpu {sc[bad[0]]:#04x} oracle {want[bad[0]]:#04x}")


def gemm_tolerance(ref, a_norm, b_norm, K, out_bf16):
    """The parity bar: max relative error 2e-3 with an absolute floor
    1e-3 * |row of A| * |row of B| / sqrt(K) (dequantized norms), stated for
    the fp32 result; a bf16 output adds its own rounding, 2^-8 relative."""
    tol = np.maximum(2e-3 * np.abs(ref), 1e-3 * a_norm * b_norm / np.sqrt(K))
    if out_bf16:
        tol = tol + 2.0 ** -8 * np.abs(ref)
    return tol


def assert_gemm_close(y, ref, a_norm, b_norm, K, out_bf16, what=""):
    y = np.asarray(y, np.float64)
    tol = gemm_tolerance(ref, a_norm, b_norm, K, out_bf16)
    err = np.abs(y - ref)
    bad = err > tol
    if bad.any():
        idx = np.argwhere(bad)[0] if bad.ndim > 1 else np.flatnonzero(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance; first at {idx}: "
                             f"gpu {y[tuple(np.atleast_1d(idx))]} ref {ref[tuple(np.atleast_1d(idx))]} "
                             f"tol {tol[tuple(np.atleast_1d(idx))]}; max err/tol {(err / tol).max():.3f}")
    return float((err / tol).max()) if err.size else 0.0


def to_numpy_f64(y: torch.Tensor) -> np.ndarray:
    return y.float().cpu().numpy().astype(np.float64)
