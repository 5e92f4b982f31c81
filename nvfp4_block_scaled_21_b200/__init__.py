"""Python binding of the B200 NVFP4 library (``libnvfp4.so``, C ABI in
``include/nvfp4.h``).

Argument marshalling only: every step of quantization, dequantization and the
W4A4 block-scaled GEMM runs in the library's CUDA kernels.  PyTorch supplies
device memory and the current stream.  There is no CPU fallback: importing
this package fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_PKG = os.path.dirname(os.path.abspath(__file__))
# NVFP4_LIBRARY=debug loads the debug build, whose kernels check every direct
# global store against its buffer (ERR_BOUNDS in the status word on a miss).
DEBUG_BUILD = os.environ.get("NVFP4_LIBRARY", "") == "debug"
LIB_PATH = os.path.join(_PKG, "libnvfp4_debug.so" if DEBUG_BUILD else "libnvfp4.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m nvfp4_block_scaled_21_b200.build` "
        "(nvcc, sm_100a). The package has no CPU fallback.")

_lib = ctypes.CDLL(LIB_PATH)

# status codes (include/nvfp4.h)
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED_SHAPE, ERR_MISALIGNED, ERR_WORKSPACE, ERR_CUDA, \
    ERR_TIMEOUT, ERR_ARCH, ERR_BOUNDS = range(9)
F32, BF16 = 0, 1
OP_QUANTIZE, OP_DEQUANTIZE, OP_GEMM, OP_LINEAR_FUSED, OP_LINEAR_FUSED_SILU, OP_GEMM_REQUANT, OP_W4A16, \
    OP_W4A8_LINEAR = range(8)
EPI_STORE, EPI_SILU_MUL_REQUANT = 0, 1

EXPORTED = (
    "nvfp4_codes_bytes", "nvfp4_scales_bytes", "nvfp4_workspace_bytes", "nvfp4_quantize",
    "nvfp4_dequantize", "nvfp4_gemm", "nvfp4_linear_fused", "nvfp4_get_device_status",
    "nvfp4_selftest_bounded_wait", "nvfp4_set_wait_timeout_us", "nvfp4_status_string",
    "nvfp4_version", "nvfp4_linear_noalloc", "nvfp4_gemm_requant", "nvfp4_mx_scales_bytes",
    "nvfp4_mx_quantize", "nvfp4_mx_gemm", "nvfp4_w4a16_linear", "nvfp4_mx8_quantize", "nvfp4_w4a8_gemm",
    "nvfp4_w4a8_linear", "nvfp4_amax", "nvfp4_quantize_with_amax",
)


class CTensor(ctypes.Structure):
    """``nvfp4_tensor`` of the C ABI."""
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("tensor_scale", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64)]


class CMXTensor(ctypes.Structure):
    """``nvfp4_mx_tensor`` of the C ABI."""
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64)]


class CMX8Tensor(ctypes.Structure):
    """``nvfp4_mx8_tensor`` of the C ABI."""
    _fields_ = [("elems", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64)]


_P, _I64, _SZ, _I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
_T = ctypes.POINTER(CTensor)
_TM = ctypes.POINTER(CMXTensor)
_T8 = ctypes.POINTER(CMX8Tensor)

_lib.nvfp4_codes_bytes.argtypes = [_I64, _I64]
_lib.nvfp4_codes_bytes.restype = _SZ
_lib.nvfp4_scales_bytes.argtypes = [_I64, _I64]
_lib.nvfp4_scales_bytes.restype = _SZ
_lib.nvfp4_workspace_bytes.argtypes = [_I, _I64, _I64, _I64]
_lib.nvfp4_workspace_bytes.restype = _SZ
_lib.nvfp4_quantize.argtypes = [_P, _I, _I64, _I64, _I64, _T, _P, _SZ, _P]
_lib.nvfp4_quantize.restype = _I
_lib.nvfp4_amax.argtypes = [_P, _I, _I64, _I64, _I64, _P, _P, _SZ, _P]
_lib.nvfp4_amax.restype = _I
_lib.nvfp4_quantize_with_amax.argtypes = [_P, _I, _I64, _I64, _I64, _P, _T, _P, _SZ, _P]
_lib.nvfp4_quantize_with_amax.restype = _I
_lib.nvfp4_dequantize.argtypes = [_T, _P, _I, _I64, _P]
_lib.nvfp4_dequantize.restype = _I
_lib.nvfp4_gemm.argtypes = [_T, _T, _P, _I, _I64, _P, _SZ, _P]
_lib.nvfp4_gemm.restype = _I
_lib.nvfp4_gemm_requant.argtypes = [_T, _T, _P, _I, _I64, _T, _P, _SZ, _P]
_lib.nvfp4_gemm_requant.restype = _I
_lib.nvfp4_mx_scales_bytes.argtypes = [_I64, _I64]
_lib.nvfp4_mx_scales_bytes.restype = _SZ
_lib.nvfp4_mx_quantize.argtypes = [_P, _I, _I64, _I64, _I64, _TM, _P]
_lib.nvfp4_mx_quantize.restype = _I
_lib.nvfp4_mx_gemm.argtypes = [_TM, _TM, _P, _I, _I64, _P, _SZ, _P]
_lib.nvfp4_mx_gemm.restype = _I
_lib.nvfp4_w4a16_linear.argtypes = [_P, _I, _I64, _I64, _I64, _T, _P, _I, _I64, _P, _SZ, _P]
_lib.nvfp4_w4a16_linear.restype = _I
_lib.nvfp4_mx8_quantize.argtypes = [_P, _I, _I64, _I64, _I64, _T8, _P]
_lib.nvfp4_mx8_quantize.restype = _I
_lib.nvfp4_w4a8_gemm.argtypes = [_T8, _TM, _P, _I, _I64, _P, _SZ, _P]
_lib.nvfp4_w4a8_gemm.restype = _I
_lib.nvfp4_w4a8_linear.argtypes = [_P, _I, _I64, _I64, _I64, _TM, _P, _I, _I64, _T8, _P, _SZ, _P]
_lib.nvfp4_w4a8_linear.restype = _I
_lib.nvfp4_linear_fused.argtypes = [_P, _I, _I64, _I64, _I64, _T, _T, _I, _P, _I, _I64, _T, _T,
                                    _P, _SZ, _P]
_lib.nvfp4_linear_fused.restype = _I
_lib.nvfp4_linear_noalloc.argtypes = [_P, _I, _I64, _I64, _I64, _T, _P, _I, _I64, _P]
_lib.nvfp4_linear_noalloc.restype = _I
_lib.nvfp4_get_device_status.argtypes = [_P, _P]
_lib.nvfp4_get_device_status.restype = _I
_lib.nvfp4_selftest_bounded_wait.argtypes = [_P, ctypes.c_uint32, _P]
_lib.nvfp4_selftest_bounded_wait.restype = _I
_lib.nvfp4_set_wait_timeout_us.argtypes = [ctypes.c_uint32]
_lib.nvfp4_set_wait_timeout_us.restype = ctypes.c_uint32
_lib.nvfp4_status_string.argtypes = [_I]
_lib.nvfp4_status_string.restype = ctypes.c_char_p
_lib.nvfp4_version.argtypes = []
_lib.nvfp4_version.restype = _I


class NVFP4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def status_string(status: int) -> str:
    return _lib.nvfp4_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != OK:
        raise NVFP4Error(status, where)


def version() -> int:
    return _lib.nvfp4_version()


def lib() -> ctypes.CDLL:
    """The loaded ``libnvfp4.so`` (raw C ABI)."""
    return _lib


# ---------------------------------------------------------------------------
# torch marshalling
# ---------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _stream(stream) -> int:
    if stream is None:
        return _torch().cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


@dataclass
class NVFP4Tensor:
    """Device buffers of one NVFP4 tensor [rows][cols] (see ``nvfp4_tensor``)."""
    codes: "object"          # uint8 [rows, cols/2]
    scales: "object"         # uint8 [nvfp4_scales_bytes]
    tensor_scale: "object"   # float32 [4] (element 0 is g; 16-byte slot)
    rows: int
    cols: int

    @staticmethod
    def empty(rows: int, cols: int, device="cuda") -> "NVFP4Tensor":
        torch = _torch()
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=device)
        scales = torch.empty(int(_lib.nvfp4_scales_bytes(rows, cols)), dtype=torch.uint8,
                             device=device)
        g = torch.zeros(4, dtype=torch.float32, device=device)
        return NVFP4Tensor(codes, scales, g, rows, cols)

    def c(self) -> CTensor:
        return CTensor(self.codes.data_ptr(), self.scales.data_ptr(),
                       self.tensor_scale.data_ptr(), self.rows, self.cols)


@dataclass
class MXFP4Tensor:
    """Device buffers of one MXFP4 tensor [rows][cols] (see ``nvfp4_mx_tensor``)."""
    codes: "object"          # uint8 [rows, cols/2]
    scales: "object"         # uint8 [nvfp4_mx_scales_bytes]
    rows: int
    cols: int

    @staticmethod
    def empty(rows: int, cols: int, device="cuda") -> "MXFP4Tensor":
        torch = _torch()
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=device)
        scales = torch.empty(int(_lib.nvfp4_mx_scales_bytes(rows, cols)), dtype=torch.uint8, device=device)
        return MXFP4Tensor(codes, scales, rows, cols)

    def c(self) -> CMXTensor:
        return CMXTensor(self.codes.data_ptr(), self.scales.data_ptr(), self.rows, self.cols)


@dataclass
class MXFP8Tensor:
    """Device buffers of one MXFP8 tensor [rows][cols] (see ``nvfp4_mx8_tensor``)."""
    elems: "object"          # uint8 [rows, cols] (E4M3 bytes)
    scales: "object"         # uint8 [nvfp4_mx_scales_bytes]
    rows: int
    cols: int

    @staticmethod
    def empty(rows: int, cols: int, device="cuda") -> "MXFP8Tensor":
        torch = _torch()
        elems = torch.empty((rows, cols), dtype=torch.uint8, device=device)
        scales = torch.empty(int(_lib.nvfp4_mx_scales_bytes(rows, cols)), dtype=torch.uint8, device=device)
        return MXFP8Tensor(elems, scales, rows, cols)

    def c(self) -> CMX8Tensor:
        return CMX8Tensor(self.elems.data_ptr(), self.scales.data_ptr(), self.rows, self.cols)


def _rows(*ts) -> None:
    """2-D tensors whose rows are contiguous (any row pitch): the layout the C
    ABI describes with a pointer and a row pitch.  A plain check, not an assert,
    so that it also holds under python -O."""
    for t in ts:
        if t is not None and (t.dim() != 2 or (t.numel() != 0 and t.stride(1) != 1)):
            raise ValueError(f"nvfp4: expected a 2-D tensor with contiguous rows, got shape "
                             f"{tuple(t.shape)} strides {tuple(t.stride())}")


def _buffers(*qs) -> None:
    """The C ABI passes an NVFP4 tensor's buffers as bare pointers, so the
    library cannot see their sizes: each must be contiguous and hold at least
    what nvfp4_codes_bytes / nvfp4_scales_bytes give for its shape (and one
    fp32 tensor scale), or the kernels would read or write past it."""
    for q in qs:
        if q is None:
            continue
        if isinstance(q, MXFP8Tensor):
            for t, need, what in ((q.elems, q.rows * q.cols, "elems"), (q.scales, mx_scales_bytes(q.rows, q.cols), "scales")):
                have = t.numel() * t.element_size()
                if not t.is_contiguous() or have < need:
                    raise ValueError(f"nvfp4: {what} of a {q.rows}x{q.cols} MXFP8 tensor needs {need} contiguous "
                                     f"bytes; got {have} bytes")
            continue
        if isinstance(q, MXFP4Tensor):
            for t, need, what in ((q.codes, codes_bytes(q.rows, q.cols), "codes"),
                                  (q.scales, mx_scales_bytes(q.rows, q.cols), "scales")):
                have = t.numel() * t.element_size()
                if not t.is_contiguous() or have < need:
                    raise ValueError(f"nvfp4: {what} of a {q.rows}x{q.cols} MXFP4 tensor needs {need} contiguous "
                                     f"bytes; got {have} bytes")
            continue
        if q.tensor_scale.dtype != _torch().float32:
            raise TypeError(f"nvfp4: tensor_scale must be float32, got {q.tensor_scale.dtype}")
        for t, need, what in ((q.codes, codes_bytes(q.rows, q.cols), "codes"),
                              (q.scales, scales_bytes(q.rows, q.cols), "scales"),
                              (q.tensor_scale, 4, "tensor_scale")):
            have = t.numel() * t.element_size()
            if not t.is_contiguous() or have < need:
                raise ValueError(f"nvfp4: {what} of a {q.rows}x{q.cols} NVFP4 tensor needs {need} contiguous "
                                 f"bytes; got {have} bytes{'' if t.is_contiguous() else ' (not contiguous)'}")


def _shape(y, rows: int, cols: int) -> None:
    """The library writes rows x cols elements at y's row pitch: y must have that shape."""
    if y is not None and tuple(y.shape) != (rows, cols):
        raise ValueError(f"nvfp4: output of shape {tuple(y.shape)}, expected ({rows}, {cols})")


def _ws_bytes(ws) -> int:
    if not ws.is_contiguous():
        raise ValueError("nvfp4: the workspace must be contiguous")
    return ws.numel() * ws.element_size()


def _on_device(*objs) -> None:
    """Every buffer the library dereferences must live on the current CUDA
    device: a host tensor's pointer, or another GPU's, would be read by the
    kernels.  Raises before anything reaches the library."""
    cur = None
    for o in objs:
        if o is None:
            continue
        for t in ((o.codes, o.scales, o.tensor_scale) if isinstance(o, NVFP4Tensor) else
                  (o.codes, o.scales) if isinstance(o, MXFP4Tensor) else
                  (o.elems, o.scales) if isinstance(o, MXFP8Tensor) else (o,)):
            if not t.is_cuda:
                raise TypeError(f"nvfp4: got a tensor on {t.device}; the library needs CUDA tensors")
            if cur is None:
                cur = _torch().cuda.current_device()
            if t.device.index != cur:
                raise ValueError(f"nvfp4: tensor on {t.device} but the current device is cuda:{cur}")


def codes_bytes(rows: int, cols: int) -> int:
    return int(_lib.nvfp4_codes_bytes(rows, cols))


def scales_bytes(rows: int, cols: int) -> int:
    return int(_lib.nvfp4_scales_bytes(rows, cols))


def mx_scales_bytes(rows: int, cols: int) -> int:
    return int(_lib.nvfp4_mx_scales_bytes(rows, cols))


def workspace_bytes(op: int, M: int, N: int, K: int) -> int:
    return int(_lib.nvfp4_workspace_bytes(op, M, N, K))


def workspace(op: int, M: int, N: int, K: int, device="cuda"):
    """A zero-filled workspace for ``op`` at this shape."""
    torch = _torch()
    return torch.zeros(workspace_bytes(op, M, N, K), dtype=torch.uint8, device=device)


def nvfp4_quantize(x, out: NVFP4Tensor, ws, stream=None) -> NVFP4Tensor:
    """Quantize a 2-D bf16/fp32 CUDA tensor (row pitch x.stride(0)) into out."""
    _rows(x)
    _buffers(out)
    _on_device(x, out, ws)
    ct = out.c()
    st = _lib.nvfp4_quantize(x.data_ptr(), _dtype_code(x), x.shape[0], x.shape[1], _ld(x),
                             ctypes.byref(ct), ws.data_ptr(), _ws_bytes(ws), _stream(stream))
    _check(st, "nvfp4_quantize")
    return out


def _ld(x) -> int:
    """Row pitch (elements) of a 2-D tensor; an empty one is never read, and
    its strides may be anything, so it gets the plain pitch cols."""
    return x.stride(0) if x.numel() != 0 else x.shape[1]


def _amax_buffer(amax) -> None:
    """One fp32 on the device: the library writes or reads exactly that."""
    if amax.dtype != _torch().float32 or amax.numel() < 1 or not amax.is_contiguous():
        raise ValueError("nvfp4: amax must be a contiguous fp32 tensor of at least one element")


def nvfp4_amax(x, amax, ws, stream=None):
    """amax[0] = max |x| over a 2-D bf16/fp32 CUDA tensor (the quantizer's
    first pass, reduced on the device): this rank's share of a tensor split
    across ranks by rows, before an all-reduce MAX."""
    _rows(x)
    _amax_buffer(amax)
    _on_device(x, amax, ws)
    st = _lib.nvfp4_amax(x.data_ptr(), _dtype_code(x), x.shape[0], x.shape[1], _ld(x), amax.data_ptr(),
                         ws.data_ptr(), _ws_bytes(ws), _stream(stream))
    _check(st, "nvfp4_amax")
    return amax


def nvfp4_quantize_with_amax(x, amax, out: NVFP4Tensor, ws, stream=None) -> NVFP4Tensor:
    """nvfp4_quantize with the tensor amax given (amax[0], device fp32) instead
    of computed from x: g = amax / 2688."""
    _rows(x)
    _amax_buffer(amax)
    _buffers(out)
    _on_device(x, amax, out, ws)
    ct = out.c()
    st = _lib.nvfp4_quantize_with_amax(x.data_ptr(), _dtype_code(x), x.shape[0], x.shape[1], _ld(x),
                                       amax.data_ptr(), ctypes.byref(ct), ws.data_ptr(), _ws_bytes(ws),
                                       _stream(stream))
    _check(st, "nvfp4_quantize_with_amax")
    return out


def nvfp4_dequantize(q: NVFP4Tensor, y, stream=None):
    _rows(y)
    _buffers(q)
    _shape(y, q.rows, q.cols)
    _on_device(q, y)
    ct = q.c()
    st = _lib.nvfp4_dequantize(ctypes.byref(ct), y.data_ptr(), _dtype_code(y), y.stride(0),
                               _stream(stream))
    _check(st, "nvfp4_dequantize")
    return y


def nvfp4_gemm(a: NVFP4Tensor, b: NVFP4Tensor, y, ws, stream=None):
    """y[M][N] = (a . b^T) * ga * gb."""
    _rows(y)
    _buffers(a, b)
    _shape(y, a.rows, b.rows)
    _on_device(a, b, y, ws)
    ca, cb = a.c(), b.c()
    st = _lib.nvfp4_gemm(ctypes.byref(ca), ctypes.byref(cb), y.data_ptr(), _dtype_code(y),
                         y.stride(0), ws.data_ptr(), _ws_bytes(ws), _stream(stream))
    _check(st, "nvfp4_gemm")
    return y


def nvfp4_gemm_requant(a: NVFP4Tensor, b: NVFP4Tensor, y, y_q: NVFP4Tensor, ws, stream=None):
    """y[M][N] = (a . b^T) * ga * gb, and y as stored quantized to NVFP4 into y_q."""
    _rows(y)
    _buffers(a, b, y_q)
    _shape(y, a.rows, b.rows)
    if (y_q.rows, y_q.cols) != (a.rows, b.rows):
        raise ValueError(f"nvfp4: y_q is {y_q.rows}x{y_q.cols}, expected {a.rows}x{b.rows}")
    _on_device(a, b, y, y_q, ws)
    ca, cb, cq = a.c(), b.c(), y_q.c()
    st = _lib.nvfp4_gemm_requant(ctypes.byref(ca), ctypes.byref(cb), y.data_ptr(), _dtype_code(y),
                                 y.stride(0), ctypes.byref(cq), ws.data_ptr(), _ws_bytes(ws), _stream(stream))
    _check(st, "nvfp4_gemm_requant")
    return y


def nvfp4_linear_fused(x, w: NVFP4Tensor, ws, epilogue: int = EPI_STORE, y=None,
                       w_up: NVFP4Tensor | None = None, y_q: NVFP4Tensor | None = None,
                       x_q: NVFP4Tensor | None = None, stream=None):
    """Quantize x on the device and run the W4A4 linear layer (see nvfp4.h)."""
    _rows(x, y)
    _buffers(w, w_up, y_q, x_q)
    _shape(y, x.shape[0], w.rows)
    _on_device(x, w, ws, y, w_up, y_q, x_q)
    cw = w.c()
    cwu = w_up.c() if w_up is not None else None
    cyq = y_q.c() if y_q is not None else None
    cxq = x_q.c() if x_q is not None else None
    yt = _dtype_code(y) if y is not None else F32
    ldy = y.stride(0) if y is not None else 0
    st = _lib.nvfp4_linear_fused(
        x.data_ptr(), _dtype_code(x), x.shape[0], x.shape[1], x.stride(0), ctypes.byref(cw),
        ctypes.byref(cwu) if cwu is not None else None, epilogue, _ptr(y), yt, ldy,
        ctypes.byref(cyq) if cyq is not None else None,
        ctypes.byref(cxq) if cxq is not None else None, ws.data_ptr(), _ws_bytes(ws),
        _stream(stream))
    _check(st, "nvfp4_linear_fused")
    return y


def nvfp4_linear_noalloc(x, w: NVFP4Tensor, y, stream=None):
    """W4A4 linear layer (quantize x, GEMM with w) using the library's own
    static scratch instead of a caller workspace; for callers that cannot
    allocate device memory.  See nvfp4_linear_noalloc in nvfp4.h for the size
    limit and the rule that calls must not overlap on the GPU."""
    _rows(x, y)
    _buffers(w)
    _shape(y, x.shape[0], w.rows)
    _on_device(x, w, y)
    cw = w.c()
    st = _lib.nvfp4_linear_noalloc(x.data_ptr(), _dtype_code(x), x.shape[0], x.shape[1],
                                   x.stride(0), ctypes.byref(cw), y.data_ptr(), _dtype_code(y),
                                   y.stride(0), _stream(stream))
    _check(st, "nvfp4_linear_noalloc")
    return y


def nvfp4_mx_quantize(x, out: MXFP4Tensor, stream=None) -> MXFP4Tensor:
    """Quantize a 2-D bf16/fp32 CUDA tensor (row pitch x.stride(0)) to MXFP4 into out."""
    _rows(x)
    _buffers(out)
    _on_device(x, out)
    ct = out.c()
    st = _lib.nvfp4_mx_quantize(x.data_ptr(), _dtype_code(x), x.shape[0], x.shape[1], x.stride(0),
                                ctypes.byref(ct), _stream(stream))
    _check(st, "nvfp4_mx_quantize")
    return out


def nvfp4_mx_gemm(a: MXFP4Tensor, b: MXFP4Tensor, y, ws, stream=None):
    """y[M][N] = a . b^T for MXFP4 operands (workspace as for OP_GEMM)."""
    _rows(y)
    _buffers(a, b)
    _shape(y, a.rows, b.rows)
    _on_device(a, b, y, ws)
    ca, cb = a.c(), b.c()
    st = _lib.nvfp4_mx_gemm(ctypes.byref(ca), ctypes.byref(cb), y.data_ptr(), _dtype_code(y), y.stride(0),
                            ws.data_ptr(), _ws_bytes(ws), _stream(stream))
    _check(st, "nvfp4_mx_gemm")
    return y


def nvfp4_w4a16_linear(x, w: NVFP4Tensor, y, ws, stream=None):
    """W4A16: y = x . deq(w)^T with bf16 activations x [M][K] and NVFP4 weights."""
    _rows(x, y)
    _buffers(w)
    _shape(y, x.shape[0], w.rows)
    _on_device(x, w, y, ws)
    cw = w.c()
    st = _lib.nvfp4_w4a16_linear(x.data_ptr(), _dtype_code(x), x.shape[0], x.shape[1], x.stride(0), ctypes.byref(cw),
                                 y.data_ptr(), _dtype_code(y), y.stride(0), ws.data_ptr(), _ws_bytes(ws),
                                 _stream(stream))
    _check(st, "nvfp4_w4a16_linear")
    return y


def nvfp4_mx8_quantize(x, out: MXFP8Tensor, stream=None) -> MXFP8Tensor:
    """Quantize a 2-D bf16/fp32 CUDA tensor to MXFP8 (E4M3 elements, E8M0 scales per 32) into out."""
    _rows(x)
    _buffers(out)
    _on_device(x, out)
    ct = out.c()
    st = _lib.nvfp4_mx8_quantize(x.data_ptr(), _dtype_code(x), x.shape[0], x.shape[1], x.stride(0),
                                 ctypes.byref(ct), _stream(stream))
    _check(st, "nvfp4_mx8_quantize")
    return out


def nvfp4_w4a8_gemm(a: MXFP8Tensor, b: MXFP4Tensor, y, ws, stream=None):
    """y[M][N] = a . b^T for MXFP8 activations and MXFP4 weights (workspace as OP_GEMM)."""
    _rows(y)
    _buffers(a, b)
    _shape(y, a.rows, b.rows)
    _on_device(a, b, y, ws)
    ca, cb = a.c(), b.c()
    st = _lib.nvfp4_w4a8_gemm(ctypes.byref(ca), ctypes.byref(cb), y.data_ptr(), _dtype_code(y), y.stride(0),
                              ws.data_ptr(), _ws_bytes(ws), _stream(stream))
    _check(st, "nvfp4_w4a8_gemm")
    return y


def nvfp4_w4a8_linear(x, w: MXFP4Tensor, y, ws, x_q: MXFP8Tensor | None = None, stream=None):
    """W4A8 linear layer: quantize x to MXFP8 on the device, y = x_q . w^T."""
    _rows(x, y)
    _buffers(w, x_q)
    _shape(y, x.shape[0], w.rows)
    _on_device(x, w, y, ws, x_q)
    cw = w.c()
    cq = x_q.c() if x_q is not None else None
    st = _lib.nvfp4_w4a8_linear(x.data_ptr(), _dtype_code(x), x.shape[0], x.shape[1], x.stride(0), ctypes.byref(cw),
                                y.data_ptr(), _dtype_code(y), y.stride(0),
                                ctypes.byref(cq) if cq is not None else None, ws.data_ptr(), _ws_bytes(ws),
                                _stream(stream))
    _check(st, "nvfp4_w4a8_linear")
    return y


def mx_quantize(x, stream=None) -> MXFP4Tensor:
    """Allocate an MXFP4Tensor and quantize x into it."""
    return nvfp4_mx_quantize(x, MXFP4Tensor.empty(x.shape[0], x.shape[1], device=x.device), stream)


def nvfp4_get_device_status(ws, stream=None) -> int:
    _on_device(ws)
    return int(_lib.nvfp4_get_device_status(ws.data_ptr(), _stream(stream)))


def nvfp4_selftest_bounded_wait(ws, timeout_us: int, stream=None) -> None:
    _on_device(ws)
    _check(_lib.nvfp4_selftest_bounded_wait(ws.data_ptr(), int(timeout_us), _stream(stream)),
           "nvfp4_selftest_bounded_wait")


def nvfp4_set_wait_timeout_us(timeout_us: int) -> int:
    return int(_lib.nvfp4_set_wait_timeout_us(int(timeout_us)))


# convenience -----------------------------------------------------------------

def quantize(x, ws=None, stream=None) -> NVFP4Tensor:
    """Allocate an NVFP4Tensor and quantize x into it."""
    out = NVFP4Tensor.empty(x.shape[0], x.shape[1], device=x.device)
    if ws is None:
        ws = workspace(OP_QUANTIZE, x.shape[0], 0, x.shape[1], device=x.device)
    return nvfp4_quantize(x, out, ws, stream)
