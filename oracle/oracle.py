"""numpy front end of the C oracle (``nvfp4_oracle.c``).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
this module.  The product package never imports it and shares no code with it.

Parity status of each function (what pins it is in ``tests/test_oracle.py``):

* ``e2m1_value``, ``e2m1_encode``    pinned: bit formula, page range +-6, brute
                                      force nearest with tie rule, sweep.
* ``e4m3_value``, ``e4m3_encode``    pinned: all 256 bytes against
                                      torch.float8_e4m3fn; RNE against torch's
                                      converter for in-range values and every
                                      midpoint; saturation.
* ``quantize``, ``dequantize``       pinned: exact round trip of every
                                      E2M1 x E4M3 value, brute-force optimality
                                      of each scale and code, error bound, block
                                      granularity, zero tensor, golden fixture.
* ``gemm_f64``, ``gemm_entries``     pinned: exact rational arithmetic on the
                                      tiny case, closed form for constant
                                      operands.
* ``silu_mul_f64``                   pinned: closed-form identities of SiLU.
* ``w4a16_gemm_f64`` (16-bit          pinned: exact rational arithmetic from
  activations x NVFP4 weights)        the code and scale bytes, a closed form
                                      for constant weights, sign symmetry.
* ``mx_*`` (MXFP4: 32-value blocks,  pinned: E8M0 decode of all 256 bytes
  E8M0 scales, no tensor scale)      against torch.float8_e8m0fnu; the scale
                                      rule by brute force over every byte;
                                      exact round trip; nearest-code check;
                                      block granularity; 4.25-bit storage;
                                      closed-form GEMM.
* ``mx8_*``, ``w4a8_gemm_f64``       pinned: the scale rule by brute force over
  (MXFP8 activations, W4A8)           every byte; elements against torch's E4M3
                                      conversion; exact round trip; closed-form
                                      W4A8 product.
* tiled scale layout, nibble order   parity unpinned by the pages: fixed by the
                                      tensor-core operand format and checked only
                                      through GPU GEMM parity.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

# Compiler flags: plain IEEE fp32/fp64, no contraction of a*b+c into an FMA,
# no fast-math reassociation.
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
          "-shared", "-pthread"]


def build(force: bool = False) -> str:
    """Compile ``nvfp4_oracle.c`` into ``liboracle.so`` beside it."""
    if force or not os.path.exists(_LIB_PATH) or (
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


_P = ctypes.c_void_p
_I64 = ctypes.c_int64


def _declare(L):
    L.oracle_e2m1_value.argtypes = [ctypes.c_uint]
    L.oracle_e2m1_value.restype = ctypes.c_double
    L.oracle_e2m1_encode.argtypes = [ctypes.c_float]
    L.oracle_e2m1_encode.restype = ctypes.c_uint
    L.oracle_e4m3_value.argtypes = [ctypes.c_uint]
    L.oracle_e4m3_value.restype = ctypes.c_double
    L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
    L.oracle_e4m3_encode.restype = ctypes.c_uint
    L.oracle_amax.argtypes = [_P, _I64, _I64, _I64]
    L.oracle_amax.restype = ctypes.c_float
    L.oracle_tensor_scale.argtypes = [ctypes.c_float]
    L.oracle_tensor_scale.restype = ctypes.c_float
    L.oracle_block_scale.argtypes = [ctypes.c_float, ctypes.c_float]
    L.oracle_block_scale.restype = ctypes.c_uint
    L.oracle_quantize.argtypes = [_P, _I64, _I64, _I64, _P, _P, _P]
    L.oracle_quantize.restype = ctypes.c_int
    L.oracle_dequantize.argtypes = [_P, _P, ctypes.c_float, _I64, _I64, _P]
    L.oracle_dequantize.restype = ctypes.c_int
    L.oracle_dequantize_f64.argtypes = [_P, _P, ctypes.c_float, _I64, _I64, _P]
    L.oracle_dequantize_f64.restype = ctypes.c_int
    L.oracle_gemm_f64.argtypes = [_P, _P, _I64, _I64, _I64, _P, ctypes.c_int]
    L.oracle_gemm_f64.restype = ctypes.c_int
    L.oracle_gemm_entries_f64.argtypes = [_P, _P, ctypes.c_float, _P, _P,
                                          ctypes.c_float, _I64, _P, _P, _I64,
                                          _P, _P, _P]
    L.oracle_gemm_entries_f64.restype = ctypes.c_int
    L.oracle_silu_mul_f64.argtypes = [_P, _P, _I64, _P]
    L.oracle_silu_mul_f64.restype = None
    L.oracle_storage_bytes.argtypes = [_I64, _I64]
    L.oracle_storage_bytes.restype = _I64
    L.oracle_e2m1_encode_array.argtypes = [_P, _I64, _P]
    L.oracle_e4m3_encode_array.argtypes = [_P, _I64, _P]
    L.oracle_e4m3_value_array.argtypes = [_P, _I64, _P]
    L.oracle_bf16_to_f32.argtypes = [_P, _I64, _P]
    L.oracle_e8m0_value.argtypes = [ctypes.c_uint]
    L.oracle_e8m0_value.restype = ctypes.c_double
    L.oracle_mx_block_scale.argtypes = [ctypes.c_float]
    L.oracle_mx_block_scale.restype = ctypes.c_uint
    L.oracle_mx_quantize.argtypes = [_P, _I64, _I64, _I64, _P, _P]
    L.oracle_mx_quantize.restype = ctypes.c_int
    L.oracle_mx_dequantize_f64.argtypes = [_P, _P, _I64, _I64, _P]
    L.oracle_mx_dequantize_f64.restype = ctypes.c_int
    L.oracle_mx_storage_bytes.argtypes = [_I64, _I64]
    L.oracle_mx_storage_bytes.restype = _I64
    L.oracle_mx8_block_scale.argtypes = [ctypes.c_float]
    L.oracle_mx8_block_scale.restype = ctypes.c_uint
    L.oracle_e4m3_encode_signed.argtypes = [ctypes.c_float]
    L.oracle_e4m3_encode_signed.restype = ctypes.c_uint
    L.oracle_mx8_quantize.argtypes = [_P, _I64, _I64, _I64, _P, _P]
    L.oracle_mx8_quantize.restype = ctypes.c_int
    L.oracle_mx8_dequantize_f64.argtypes = [_P, _P, _I64, _I64, _P]
    L.oracle_mx8_dequantize_f64.restype = ctypes.c_int


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# Codecs
# --------------------------------------------------------------------------

def e2m1_value(code: int) -> float:
    """Value of a 4-bit E2M1 code (sign in bit 3)."""
    return lib().oracle_e2m1_value(int(code))


def e2m1_encode(v: float) -> int:
    return lib().oracle_e2m1_encode(float(v))


def e2m1_encode_array(v) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().oracle_e2m1_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e4m3_value(byte: int) -> float:
    return lib().oracle_e4m3_value(int(byte))


def e4m3_value_array(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint8)
    out = np.empty(b.shape, np.float64)
    lib().oracle_e4m3_value_array(_ptr(b), b.size, _ptr(out))
    return out


def e4m3_encode(t: float) -> int:
    return lib().oracle_e4m3_encode(float(t))


def e4m3_encode_array(t) -> np.ndarray:
    t = np.ascontiguousarray(t, dtype=np.float32)
    out = np.empty(t.shape, np.uint8)
    lib().oracle_e4m3_encode_array(_ptr(t), t.size, _ptr(out))
    return out


def bf16_bits_to_f32(x_bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to fp32."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    out = np.empty(x_bits.shape, np.float32)
    lib().oracle_bf16_to_f32(_ptr(x_bits), x_bits.size, _ptr(out))
    return out


# --------------------------------------------------------------------------
# Quantizer
# --------------------------------------------------------------------------

class Quantized:
    """One quantized tensor as the oracle emits it.

    codes:  uint8 [rows][cols/2], element 2j in the low nibble of byte j
    scales: uint8 [rows][cols/16], row-major E4M3 block scales
    g:      fp32 tensor scale
    """

    def __init__(self, codes, scales, g, rows, cols):
        self.codes, self.scales, self.g = codes, scales, np.float32(g)
        self.rows, self.cols = rows, cols

    def storage_bytes(self) -> int:
        return int(lib().oracle_storage_bytes(self.rows, self.cols))


def tensor_scale(amax: float) -> np.float32:
    return np.float32(lib().oracle_tensor_scale(float(amax)))


def block_scale(bamax: float, g: float) -> int:
    return lib().oracle_block_scale(float(bamax), float(g))


def quantize(x: np.ndarray) -> Quantized:
    """Quantize a 2-D fp32 array (or bf16 given as its uint16 bit patterns)."""
    if x.dtype == np.uint16:
        x = bf16_bits_to_f32(x)
    x = np.ascontiguousarray(x, dtype=np.float32)
    if x.ndim != 2:
        raise ValueError("quantize expects a 2-D array")
    rows, cols = x.shape
    if cols % 16:
        raise ValueError("cols must be a multiple of 16")
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 16), np.uint8)
    g = np.zeros(1, np.float32)
    rc = lib().oracle_quantize(_ptr(x), rows, cols, cols, _ptr(codes),
                               _ptr(scales), _ptr(g))
    if rc != 0:
        raise ValueError("oracle_quantize rejected the input (non-finite?)")
    return Quantized(codes, scales, g[0], rows, cols)


def dequantize(q: Quantized) -> np.ndarray:
    y = np.empty((q.rows, q.cols), np.float32)
    rc = lib().oracle_dequantize(_ptr(q.codes), _ptr(q.scales), float(q.g),
                                 q.rows, q.cols, _ptr(y))
    assert rc == 0
    return y


def dequantize_f64(q: Quantized) -> np.ndarray:
    y = np.empty((q.rows, q.cols), np.float64)
    rc = lib().oracle_dequantize_f64(_ptr(q.codes), _ptr(q.scales), float(q.g),
                                     q.rows, q.cols, _ptr(y))
    assert rc == 0
    return y


# --------------------------------------------------------------------------
# GEMM and the fused MLP middle step
# --------------------------------------------------------------------------

def gemm_f64(a: Quantized, b: Quantized, nthreads: int | None = None) -> np.ndarray:
    """Y = deq(A) . deq(B)^T in fp64, A [M][K], B [N][K]."""
    if a.cols != b.cols:
        raise ValueError("K mismatch")
    da = dequantize_f64(a)
    db = dequantize_f64(b)
    y = np.empty((a.rows, b.rows), np.float64)
    nt = nthreads or os.cpu_count() or 1
    rc = lib().oracle_gemm_f64(_ptr(da), _ptr(db), a.rows, b.rows, a.cols,
                               _ptr(y), int(nt))
    assert rc == 0
    return y


def gemm_entries(a: Quantized, b: Quantized, ms, ns):
    """Selected entries Y[ms[i], ns[i]] plus the fp64 norms of the dequantized
    row of A and row of B used by each entry."""
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    out = np.empty(ms.shape, np.float64)
    na = np.empty(ms.shape, np.float64)
    nb = np.empty(ms.shape, np.float64)
    rc = lib().oracle_gemm_entries_f64(
        _ptr(a.codes), _ptr(a.scales), float(a.g), _ptr(b.codes),
        _ptr(b.scales), float(b.g), a.cols, _ptr(ms), _ptr(ns), ms.size,
        _ptr(out), _ptr(na), _ptr(nb))
    assert rc == 0
    return out, na, nb


def w4a16_gemm_f64(x: np.ndarray, w: Quantized, nthreads: int | None = None) -> np.ndarray:
    """W4A16: Y = X . deq(W)^T in fp64 with 16-bit activations X [M][K] taken
    as they are (bf16 given as uint16 bit patterns, or fp32) and NVFP4 weights
    W [N][K] dequantized exactly (e * s * g).  The weights are 4-bit, the
    activations stay 16-bit, and the product uses the dequantized weights
    (aixq.cc article on Unsloth Dynamic NVFP4, section "核心差异：W4A4 vs
    W4A16")."""
    if x.dtype == np.uint16:
        x = bf16_bits_to_f32(x)
    xa = np.ascontiguousarray(x, dtype=np.float64)
    if xa.ndim != 2 or xa.shape[1] != w.cols:
        raise ValueError("x must be [M][K] with the weights' K")
    dw = dequantize_f64(w)
    y = np.empty((xa.shape[0], w.rows), np.float64)
    nt = nthreads or os.cpu_count() or 1
    rc = lib().oracle_gemm_f64(_ptr(xa), _ptr(dw), xa.shape[0], w.rows, w.cols, _ptr(y), int(nt))
    assert rc == 0
    return y


def silu_mul_f64(gate: np.ndarray, up: np.ndarray) -> np.ndarray:
    gate = np.ascontiguousarray(gate, dtype=np.float64)
    up = np.ascontiguousarray(up, dtype=np.float64)
    h = np.empty(gate.shape, np.float64)
    lib().oracle_silu_mul_f64(_ptr(gate), _ptr(up), gate.size, _ptr(h))
    return h


def storage_bytes(rows: int, cols: int) -> int:
    return int(lib().oracle_storage_bytes(rows, cols))


def mlp_chain_f64(x_q: Quantized, wg: Quantized, wu: Quantized):
    """Gate and up projections of the fused MLP step, then SiLU(gate)*up, all
    in fp64.  The quantization of h and the down projection reuse
    ``quantize`` and ``gemm_f64``."""
    gate = gemm_f64(x_q, wg)
    up = gemm_f64(x_q, wu)
    return silu_mul_f64(gate, up)


# --------------------------------------------------------------------------
# MXFP4 (32-value blocks, E8M0 scales, no tensor scale; readings M1-M4 in
# nvfp4_oracle.c)
# --------------------------------------------------------------------------

class QuantizedMX:
    """One MXFP4 tensor as the oracle emits it.

    codes:  uint8 [rows][cols/2], element 2j in the low nibble of byte j
    scales: uint8 [rows][cols/32], row-major E8M0 block scales
    """

    def __init__(self, codes, scales, rows, cols):
        self.codes, self.scales, self.rows, self.cols = codes, scales, rows, cols


def e8m0_value(byte: int) -> float:
    return lib().oracle_e8m0_value(int(byte))


def mx_block_scale(bamax: float) -> int:
    return lib().oracle_mx_block_scale(float(bamax))


def mx_quantize(x: np.ndarray) -> QuantizedMX:
    """Quantize a 2-D fp32 array (or bf16 given as its uint16 bit patterns) to MXFP4."""
    if x.dtype == np.uint16:
        x = bf16_bits_to_f32(x)
    x = np.ascontiguousarray(x, dtype=np.float32)
    if x.ndim != 2:
        raise ValueError("mx_quantize expects a 2-D array")
    rows, cols = x.shape
    if cols % 32:
        raise ValueError("cols must be a multiple of 32")
    codes = np.zeros((rows, cols // 2), np.uint8)
    scales = np.zeros((rows, cols // 32), np.uint8)
    rc = lib().oracle_mx_quantize(_ptr(x), rows, cols, cols, _ptr(codes), _ptr(scales))
    if rc != 0:
        raise ValueError("oracle_mx_quantize rejected the input (non-finite?)")
    return QuantizedMX(codes, scales, rows, cols)


def mx_dequantize_f64(q: QuantizedMX) -> np.ndarray:
    y = np.empty((q.rows, q.cols), np.float64)
    rc = lib().oracle_mx_dequantize_f64(_ptr(q.codes), _ptr(q.scales), q.rows, q.cols, _ptr(y))
    assert rc == 0
    return y


def mx_gemm_f64(a: QuantizedMX, b: QuantizedMX, nthreads: int | None = None) -> np.ndarray:
    """Y = deq(A) . deq(B)^T in fp64, A [M][K], B [N][K], both MXFP4."""
    if a.cols != b.cols:
        raise ValueError("K mismatch")
    da = mx_dequantize_f64(a)
    db = mx_dequantize_f64(b)
    y = np.empty((a.rows, b.rows), np.float64)
    nt = nthreads or os.cpu_count() or 1
    rc = lib().oracle_gemm_f64(_ptr(da), _ptr(db), a.rows, b.rows, a.cols, _ptr(y), int(nt))
    assert rc == 0
    return y


def mx_storage_bytes(rows: int, cols: int) -> int:
    return int(lib().oracle_mx_storage_bytes(rows, cols))


# --------------------------------------------------------------------------
# MXFP8 activations and the W4A8 product (readings X1-X2 in nvfp4_oracle.c):
# FP4 weights (MXFP4) times FP8 activations (E4M3 elements, one E8M0 scale per
# 32 values), the eefocus.com article's W4A8 (section on the Zhouyi X3 NPU).
# --------------------------------------------------------------------------

class QuantizedMX8:
    """One MXFP8 tensor as the oracle emits it.

    elems:  uint8 [rows][cols], E4M3 bytes
    scales: uint8 [rows][cols/32], row-major E8M0 block scales
    """

    def __init__(self, elems, scales, rows, cols):
        self.elems, self.scales, self.rows, self.cols = elems, scales, rows, cols


def mx8_block_scale(bamax: float) -> int:
    return lib().oracle_mx8_block_scale(float(bamax))


def e4m3_encode_signed(v: float) -> int:
    return lib().oracle_e4m3_encode_signed(float(v))


def mx8_quantize(x: np.ndarray) -> QuantizedMX8:
    """Quantize a 2-D fp32 array (or bf16 given as its uint16 bit patterns) to MXFP8."""
    if x.dtype == np.uint16:
        x = bf16_bits_to_f32(x)
    x = np.ascontiguousarray(x, dtype=np.float32)
    if x.ndim != 2:
        raise ValueError("mx8_quantize expects a 2-D array")
    rows, cols = x.shape
    if cols % 32:
        raise ValueError("cols must be a multiple of 32")
    elems = np.zeros((rows, cols), np.uint8)
    scales = np.zeros((rows, cols // 32), np.uint8)
    rc = lib().oracle_mx8_quantize(_ptr(x), rows, cols, cols, _ptr(elems), _ptr(scales))
    if rc != 0:
        raise ValueError("oracle_mx8_quantize rejected the input (non-finite?)")
    return QuantizedMX8(elems, scales, rows, cols)


def mx8_dequantize_f64(q: QuantizedMX8) -> np.ndarray:
    y = np.empty((q.rows, q.cols), np.float64)
    rc = lib().oracle_mx8_dequantize_f64(_ptr(q.elems), _ptr(q.scales), q.rows, q.cols, _ptr(y))
    assert rc == 0
    return y


def w4a8_gemm_f64(x: QuantizedMX8, w: QuantizedMX, nthreads: int | None = None) -> np.ndarray:
    """W4A8: Y = deq(X) . deq(W)^T in fp64, X MXFP8 [M][K], W MXFP4 [N][K]."""
    if x.cols != w.cols:
        raise ValueError("K mismatch")
    dx = mx8_dequantize_f64(x)
    dw = mx_dequantize_f64(w)
    y = np.empty((x.rows, w.rows), np.float64)
    nt = nthreads or os.cpu_count() or 1
    rc = lib().oracle_gemm_f64(_ptr(dx), _ptr(dw), x.rows, w.rows, x.cols, _ptr(y), int(nt))
    assert rc == 0
    return y
