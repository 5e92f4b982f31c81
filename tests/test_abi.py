"""CPU-side checks of the C ABI: the library loads, exports every function the
header declares, reports sizes, and rejects bad arguments synchronously
without touching the GPU."""
import ctypes
import os
import re

import pytest

import nvfp4_block_scaled_21_b200 as nv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "nvfp4.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_four_entry_points():
    names = declared_functions()
    for n in ("nvfp4_quantize", "nvfp4_dequantize", "nvfp4_gemm", "nvfp4_linear_fused"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = nv.lib()
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(nv.EXPORTED) == set(declared_functions())


def test_sizes():
    assert nv.codes_bytes(8192, 5120) == 8192 * 5120 // 2
    assert nv.scales_bytes(8192, 5120) == 8192 * 320
    assert nv.scales_bytes(8, 5120) == 128 * 320          # rows padded to 128
    assert nv.scales_bytes(1, 16) == 128 * 4              # blocks padded to 4
    assert nv.scales_bytes(130, 80) == 256 * 8
    assert nv.workspace_bytes(nv.OP_GEMM, 1, 1, 64) >= 256
    assert nv.workspace_bytes(nv.OP_QUANTIZE, 10, 0, 16) >= 256 + 4 * 1184
    assert nv.version() >= 100


def test_workspace_sizes_follow_the_kernel_choices():
    """GEMM-bearing ops reserve fp32 stream-K scratch (the padded output tile
    grid plus one counter per 128x128 tile) only for shapes with at most 1024
    output tiles; the fused MLP keeps fp32 h; quantize keeps the pass-1
    partial maxima."""
    a256 = lambda v: (v + 255) // 256 * 256
    # decode-shaped (M <= 64, swapped): roundup(N,128) x 64 floats + ceil(N/128) counters
    M, N, K = 8, 17408, 5120
    assert nv.workspace_bytes(nv.OP_GEMM, M, N, K) == 256 + a256(17408 * 64 * 4) + a256(136 * 4)
    # 128-row activations: roundup(M,128) x roundup(N,128) floats + tiles counters
    M, N = 128, 5120
    assert nv.workspace_bytes(nv.OP_GEMM, M, N, 17408) == 256 + a256(128 * 5120 * 4) + a256(40 * 4)
    # prefill-sized: 32 x 136 = 4352 tiles > 1024, no scratch
    assert nv.workspace_bytes(nv.OP_GEMM, 4096, 17408, 5120) == 256
    # the fused MLP: status + partials, x_q (codes, scales, g) and fp32 h, no stream-K scratch
    M, N, K = 128, 17408, 5120
    xq = a256(M * K // 2) + a256(((M + 127) // 128 * 128) * (K // 16)) + 256
    assert nv.workspace_bytes(nv.OP_LINEAR_FUSED_SILU, M, N, K) == 256 + 4096 * 4 + xq + a256(M * N * 4)
    # the plain linear layer adds the GEMM's stream-K scratch after x_q
    M, N = 128, 5120
    xq = a256(M * K // 2) + a256(128 * (K // 16)) + 256
    assert nv.workspace_bytes(nv.OP_LINEAR_FUSED, M, N, K) == 256 + 4096 * 4 + xq + a256(128 * 5120 * 4) + a256(40 * 4)
    # the re-quantizing GEMM: status + partial maxima of |y|, then the GEMM's stream-K scratch
    assert nv.workspace_bytes(nv.OP_GEMM_REQUANT, 4096, 17408, 5120) == 256 + 4096 * 4
    assert nv.workspace_bytes(nv.OP_GEMM_REQUANT, M, N, 17408) == 256 + 4096 * 4 + a256(128 * 5120 * 4) + a256(40 * 4)


def test_status_strings():
    assert nv.status_string(nv.OK) == "ok"
    assert "timed out" in nv.status_string(nv.ERR_TIMEOUT)
    assert nv.status_string(99) == "unknown status"


def _t(codes=16, scales=16, g=16, rows=4, cols=64):
    return nv.CTensor(codes, scales, g, rows, cols)


def test_quantize_rejects_bad_arguments_without_launch():
    lib = nv.lib()
    ws = 4096
    out = _t()
    q = lambda x, xt, r, c, ld, o, w, wb: lib.nvfp4_quantize(x, xt, r, c, ld, ctypes.byref(o) if o else None, w, wb, None)
    assert q(None, nv.BF16, 4, 64, 64, out, ws, 1 << 20) == nv.ERR_INVALID_ARG
    assert q(16, 7, 4, 64, 64, out, ws, 1 << 20) == nv.ERR_INVALID_ARG
    assert q(16, nv.BF16, 4, 64, 32, out, ws, 1 << 20) == nv.ERR_INVALID_ARG      # ld < cols
    assert q(16, nv.BF16, 4, 64, 64, None, ws, 1 << 20) == nv.ERR_INVALID_ARG
    assert q(16, nv.BF16, 4, 64, 64, _t(rows=5), ws, 1 << 20) == nv.ERR_INVALID_ARG
    assert q(16, nv.BF16, 4, 24, 24, _t(cols=24), ws, 1 << 20) == nv.ERR_UNSUPPORTED_SHAPE
    assert q(18, nv.BF16, 4, 64, 64, out, ws, 1 << 20) == nv.ERR_MISALIGNED
    assert q(16, nv.BF16, 4, 64, 68, out, ws, 1 << 20) == nv.ERR_MISALIGNED       # row pitch
    assert q(16, nv.BF16, 4, 64, 64, _t(codes=24), ws, 1 << 20) == nv.ERR_MISALIGNED
    assert q(16, nv.BF16, 4, 64, 64, out, None, 1 << 20) == nv.ERR_WORKSPACE
    assert q(16, nv.BF16, 4, 64, 64, out, ws, 100) == nv.ERR_WORKSPACE


def test_amax_and_quantize_with_amax_reject_bad_arguments_without_launch():
    lib = nv.lib()
    ws, amax = 4096, 1024
    a = lambda x, xt, r, c, ld, am, w, wb: lib.nvfp4_amax(x, xt, r, c, ld, am, w, wb, None)
    assert a(None, nv.BF16, 4, 64, 64, amax, ws, 1 << 20) == nv.ERR_INVALID_ARG
    assert a(16, nv.BF16, 4, 64, 64, None, ws, 1 << 20) == nv.ERR_INVALID_ARG
    assert a(16, 7, 4, 64, 64, amax, ws, 1 << 20) == nv.ERR_INVALID_ARG
    assert a(16, nv.BF16, 4, 64, 32, amax, ws, 1 << 20) == nv.ERR_INVALID_ARG        # ld < cols
    assert a(16, nv.BF16, 4, 24, 24, amax, ws, 1 << 20) == nv.ERR_UNSUPPORTED_SHAPE
    assert a(18, nv.BF16, 4, 64, 64, amax, ws, 1 << 20) == nv.ERR_MISALIGNED
    assert a(16, nv.BF16, 4, 64, 64, amax + 2, ws, 1 << 20) == nv.ERR_MISALIGNED
    assert a(16, nv.BF16, 4, 64, 64, amax, None, 1 << 20) == nv.ERR_WORKSPACE
    assert a(16, nv.BF16, 4, 64, 64, amax, ws, 100) == nv.ERR_WORKSPACE
    out = _t()
    q = lambda x, xt, r, c, ld, am, o, w, wb: lib.nvfp4_quantize_with_amax(
        x, xt, r, c, ld, am, ctypes.byref(o) if o else None, w, wb, None)
    assert q(16, nv.BF16, 4, 64, 64, None, out, ws, 1 << 20) == nv.ERR_INVALID_ARG
    assert q(16, nv.BF16, 4, 64, 64, amax, None, ws, 1 << 20) == nv.ERR_INVALID_ARG
    assert q(16, nv.BF16, 4, 64, 64, amax, _t(rows=5), ws, 1 << 20) == nv.ERR_INVALID_ARG
    assert q(16, nv.BF16, 4, 24, 24, amax, _t(cols=24), ws, 1 << 20) == nv.ERR_UNSUPPORTED_SHAPE
    assert q(16, nv.BF16, 4, 64, 64, amax + 1, out, ws, 1 << 20) == nv.ERR_MISALIGNED
    assert q(16, nv.BF16, 4, 64, 64, amax, out, ws, 100) == nv.ERR_WORKSPACE


def test_gemm_rejects_bad_arguments_without_launch():
    lib = nv.lib()
    a, b = _t(rows=8, cols=128), _t(rows=32, cols=128)
    g = lambda a, b, y, yt, ldy, ws, wb: lib.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), y, yt, ldy, ws, wb, None)
    assert g(a, b, None, nv.BF16, 32, 4096, 256) == nv.ERR_INVALID_ARG
    assert g(a, _t(rows=32, cols=64), 16, nv.BF16, 32, 4096, 256) == nv.ERR_INVALID_ARG   # K mismatch
    assert g(_t(rows=8, cols=96), _t(rows=32, cols=96), 16, nv.BF16, 32, 4096, 256) == nv.ERR_UNSUPPORTED_SHAPE
    assert g(a, b, 16, nv.BF16, 16, 4096, 256) == nv.ERR_INVALID_ARG                       # ldy < N
    assert g(a, b, 16, nv.BF16, 36, 4096, 256) == nv.ERR_MISALIGNED                        # pitch
    assert g(a, b, 16, nv.BF16, 32, 4096, 8) == nv.ERR_WORKSPACE


def test_gemm_requant_rejects_bad_arguments_without_launch():
    """Each call breaks exactly one rule of nvfp4_gemm_requant and stops at it."""
    lib = nv.lib()
    a, b = _t(rows=8, cols=128), _t(rows=32, cols=128)

    def g(a_=a, b_=b, y=16, yt=nv.BF16, ldy=32, yq=_t(rows=8, cols=32), ws=4096, wb=1 << 20):
        return lib.nvfp4_gemm_requant(ctypes.byref(a_), ctypes.byref(b_), y, yt, ldy,
                                      ctypes.byref(yq) if yq else None, ws, wb, None)

    assert g(yq=None) == nv.ERR_INVALID_ARG                                         # y_q missing
    assert g(yq=_t(rows=8, cols=48)) == nv.ERR_INVALID_ARG                          # y_q shape
    assert g(b_=_t(rows=24, cols=128), ldy=24, yq=_t(rows=8, cols=24)) == nv.ERR_UNSUPPORTED_SHAPE  # N % 16
    assert g(yq=_t(rows=8, cols=32, scales=24)) == nv.ERR_MISALIGNED
    assert g(y=None) == nv.ERR_INVALID_ARG
    assert g(ldy=36) == nv.ERR_MISALIGNED
    assert g(wb=256) == nv.ERR_WORKSPACE                                            # needs the partials too
    assert g(ws=None) == nv.ERR_WORKSPACE


def test_linear_fused_rejects_bad_arguments_without_launch():
    lib = nv.lib()
    w = _t(rows=32, cols=128)
    f = lambda epi, wu, yq, y: lib.nvfp4_linear_fused(16, nv.BF16, 8, 128, 128, ctypes.byref(w),
                                                      ctypes.byref(wu) if wu else None, epi, y,
                                                      nv.BF16, 32, ctypes.byref(yq) if yq else None,
                                                      None, 4096, 1 << 30, None)
    assert f(nv.EPI_STORE, None, None, None) == nv.ERR_INVALID_ARG                  # y missing
    assert f(5, None, None, 16) == nv.ERR_INVALID_ARG
    assert f(nv.EPI_SILU_MUL_REQUANT, None, _t(rows=8, cols=32), None) == nv.ERR_INVALID_ARG
    assert f(nv.EPI_SILU_MUL_REQUANT, _t(rows=16, cols=128), _t(rows=8, cols=32), None) == nv.ERR_INVALID_ARG


def test_dequantize_rejects_bad_arguments_without_launch():
    lib = nv.lib()
    q = _t(rows=4, cols=64)
    d = lambda t, y, yt, ldy: lib.nvfp4_dequantize(ctypes.byref(t) if t else None, y, yt, ldy, None)
    assert d(None, 16, nv.F32, 64) == nv.ERR_INVALID_ARG
    assert d(q, 16, 7, 64) == nv.ERR_INVALID_ARG                                    # dtype
    assert d(q, None, nv.F32, 64) == nv.ERR_INVALID_ARG                             # y missing
    assert d(q, 16, nv.F32, 32) == nv.ERR_INVALID_ARG                               # ldy < cols
    assert d(q, 24, nv.F32, 64) == nv.ERR_MISALIGNED                                # y
    assert d(q, 16, nv.BF16, 66) == nv.ERR_MISALIGNED                               # row pitch
    assert d(_t(rows=4, cols=24), 16, nv.F32, 24) == nv.ERR_UNSUPPORTED_SHAPE       # cols % 16
    assert d(_t(codes=None, rows=4, cols=64), 16, nv.F32, 64) == nv.ERR_INVALID_ARG
    assert d(_t(scales=24), 16, nv.F32, 64) == nv.ERR_MISALIGNED


def test_linear_fused_rejects_more_bad_arguments_without_launch():
    """Each call breaks exactly one rule of nvfp4_linear_fused and stops at it."""
    lib = nv.lib()
    w, wu = _t(rows=32, cols=128), _t(rows=32, cols=128)

    def f(x=16, xt=nv.BF16, M=8, K=128, ldx=128, w_=w, wu_=None, epi=nv.EPI_STORE, y=16, yt=nv.BF16, ldy=32,
          yq=None, xq=None, ws=4096, wb=1 << 30):
        return lib.nvfp4_linear_fused(x, xt, M, K, ldx, ctypes.byref(w_), ctypes.byref(wu_) if wu_ else None, epi,
                                      y, yt, ldy, ctypes.byref(yq) if yq else None,
                                      ctypes.byref(xq) if xq else None, ws, wb, None)

    assert f(x=None) == nv.ERR_INVALID_ARG                                          # x missing
    assert f(xt=9) == nv.ERR_INVALID_ARG
    assert f(M=-1) == nv.ERR_INVALID_ARG
    assert f(ldx=64) == nv.ERR_INVALID_ARG                                          # ldx < K
    assert f(w_=_t(rows=32, cols=64)) == nv.ERR_INVALID_ARG                         # w's K differs
    assert f(K=96, ldx=96, w_=_t(rows=32, cols=96)) == nv.ERR_UNSUPPORTED_SHAPE     # K % 64
    assert f(x=24) == nv.ERR_MISALIGNED
    assert f(ldx=132) == nv.ERR_MISALIGNED                                          # 264-byte pitch
    assert f(ldy=16) == nv.ERR_INVALID_ARG                                          # ldy < N
    assert f(yt=5) == nv.ERR_INVALID_ARG
    assert f(y=24) == nv.ERR_MISALIGNED
    assert f(ldy=36) == nv.ERR_MISALIGNED                                           # 72-byte pitch
    silu = dict(epi=nv.EPI_SILU_MUL_REQUANT, wu_=wu, yq=_t(rows=8, cols=32), yt=nv.F32)
    assert f(**{**silu, "yt": nv.BF16}) == nv.ERR_INVALID_ARG                       # h must be fp32
    assert f(**{**silu, "y": 24}) == nv.ERR_MISALIGNED
    assert f(**{**silu, "wu_": _t(rows=16, cols=128)}) == nv.ERR_INVALID_ARG        # w_up rows differ
    assert f(xq=_t(rows=8, cols=64)) == nv.ERR_INVALID_ARG                          # x_q shape
    assert f(yq=_t(rows=8, cols=48)) == nv.ERR_INVALID_ARG                          # STORE y_q shape
    assert f(yq=_t(rows=8, cols=32, codes=24)) == nv.ERR_MISALIGNED
    assert f(ws=None) == nv.ERR_WORKSPACE
    assert f(wb=64) == nv.ERR_WORKSPACE
    assert f(ws=4100) == nv.ERR_MISALIGNED


def test_gemm_rejects_sizes_beyond_its_index_range_and_bad_dtype():
    """Rows above 2^30 - 1 or K above 2^31 leave the kernels' 32-bit row and
    tile-coordinate range: refused, not wrapped."""
    lib = nv.lib()
    a, b = _t(rows=8, cols=128), _t(rows=32, cols=128)
    for x, w in [(_t(rows=2 ** 30, cols=128), b), (a, _t(rows=2 ** 30, cols=128)),
                 (_t(rows=8, cols=2 ** 31 + 64), _t(rows=32, cols=2 ** 31 + 64))]:
        assert lib.nvfp4_gemm(ctypes.byref(x), ctypes.byref(w), 16, nv.BF16, 2 ** 30 + 64, 4096, 1 << 30,
                              None) == nv.ERR_UNSUPPORTED_SHAPE
    ok = _t(rows=2 ** 30 - 1, cols=128)                     # the largest row count passes this check
    assert lib.nvfp4_gemm(ctypes.byref(ok), ctypes.byref(b), 16, nv.BF16, 32, 4096, 8, None) == nv.ERR_WORKSPACE
    assert lib.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), 16, 3, 32, 4096, 1 << 30, None) == nv.ERR_INVALID_ARG


def test_linear_layers_reject_sizes_beyond_the_gemm_index_range():
    lib = nv.lib()
    w, K = _t(rows=32, cols=128), 128
    big_k = 2 ** 31 + 64
    wk = _t(rows=32, cols=big_k)
    fused = lambda x_rows, kk, ww: lib.nvfp4_linear_fused(16, nv.BF16, x_rows, kk, kk, ctypes.byref(ww), None,
                                                          nv.EPI_STORE, 16, nv.BF16, ww.rows, None, None, 4096,
                                                          1 << 62, None)
    assert fused(2 ** 30, K, w) == nv.ERR_UNSUPPORTED_SHAPE                         # M
    assert fused(8, K, _t(rows=2 ** 30, cols=128)) == nv.ERR_UNSUPPORTED_SHAPE     # N
    assert fused(8, big_k, wk) == nv.ERR_UNSUPPORTED_SHAPE                          # K
    assert lib.nvfp4_linear_noalloc(16, nv.BF16, 8, big_k, big_k, ctypes.byref(wk), 16, nv.BF16, 32,
                                    None) == nv.ERR_UNSUPPORTED_SHAPE


def test_selftest_and_timeout_setter_host_paths():
    lib = nv.lib()
    assert lib.nvfp4_selftest_bounded_wait(None, 1000, None) == nv.ERR_WORKSPACE
    assert lib.nvfp4_selftest_bounded_wait(8, 1000, None) == nv.ERR_MISALIGNED
    old = lib.nvfp4_set_wait_timeout_us(1234)
    try:
        assert lib.nvfp4_set_wait_timeout_us(0) == 1234                              # 0 is stored as 1
        assert lib.nvfp4_set_wait_timeout_us(old) == 1
    finally:
        lib.nvfp4_set_wait_timeout_us(old)


def test_noalloc_rejects_bad_arguments_and_oversized_shapes_without_launch():
    """nvfp4_linear_noalloc checks its arguments and the size of its static
    scratch before its first device call (the scratch address lookup)."""
    lib = nv.lib()
    w = _t(rows=32, cols=128)

    def f(x=16, xt=nv.BF16, M=8, K=128, ldx=128, w_=w, y=16, yt=nv.BF16, ldy=32):
        return lib.nvfp4_linear_noalloc(x, xt, M, K, ldx, ctypes.byref(w_), y, yt, ldy, None)

    assert f(x=None) == nv.ERR_INVALID_ARG
    assert f(xt=4) == nv.ERR_INVALID_ARG
    assert f(ldx=100) == nv.ERR_INVALID_ARG                                         # ldx < K
    assert f(w_=_t(rows=32, cols=64)) == nv.ERR_INVALID_ARG                         # w's K differs
    assert f(K=96, ldx=96, w_=_t(rows=32, cols=96)) == nv.ERR_UNSUPPORTED_SHAPE     # K % 64
    assert f(y=None) == nv.ERR_INVALID_ARG
    assert f(ldy=8) == nv.ERR_INVALID_ARG                                           # ldy < N
    assert f(yt=2) == nv.ERR_INVALID_ARG
    assert f(x=40) == nv.ERR_MISALIGNED
    assert f(y=40) == nv.ERR_MISALIGNED
    # quantized activations beyond the 4 MiB static scratch: 8192 x 5120 needs 21 MB
    w5k = _t(rows=32, cols=5120)
    assert f(M=8192, K=5120, ldx=5120, w_=w5k) == nv.ERR_UNSUPPORTED_SHAPE


def test_empty_operands_skip_pointer_and_pitch_checks():
    """An empty matrix is never read or written: a NULL pointer and any pitch
    at least its row length pass validation.  Each call below then stops at
    the too-small workspace, before any launch."""
    lib = nv.lib()
    small = 8                                                    # below every workspace size
    out = _t(codes=None, scales=None, rows=5, cols=0)            # quantize 5 x 0, x = NULL, pitch 1
    assert lib.nvfp4_quantize(None, nv.F32, 5, 0, 1, ctypes.byref(out), 4096, small, None) == nv.ERR_WORKSPACE
    a, b0 = _t(rows=8, cols=128), _t(codes=None, scales=None, rows=0, cols=128)   # GEMM with N = 0
    assert lib.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b0), None, nv.BF16, 1, 4096, small, None) == nv.ERR_WORKSPACE
    w0 = _t(codes=None, scales=None, rows=32, cols=0)            # linear layer with K = 0, x = NULL
    assert lib.nvfp4_linear_fused(None, nv.BF16, 8, 0, 1, ctypes.byref(w0), None, nv.EPI_STORE, 16, nv.BF16,
                                  32, None, None, 4096, small, None) == nv.ERR_WORKSPACE
    q0 = _t(codes=None, scales=None, rows=0, cols=64)            # dequantize of 0 x 64, y = NULL
    assert lib.nvfp4_dequantize(ctypes.byref(q0), None, nv.F32, 64, None) in (nv.OK, nv.ERR_CUDA, nv.ERR_ARCH)
    # a non-empty operand still has its pitch checked
    assert lib.nvfp4_quantize(16, nv.F32, 5, 16, 17, ctypes.byref(_t(rows=5, cols=16)), 4096, small,
                              None) == nv.ERR_MISALIGNED


def test_binding_refuses_host_tensors_before_the_library():
    """A host tensor's pointer would be dereferenced by the kernels: every
    wrapper raises before it calls into the library."""
    import torch
    x = torch.zeros((4, 64), dtype=torch.float32)
    q = nv.NVFP4Tensor(torch.zeros((4, 32), dtype=torch.uint8), torch.zeros(512, dtype=torch.uint8),
                       torch.zeros(4), 4, 64)
    ws = torch.zeros(1 << 16, dtype=torch.uint8)
    y = torch.zeros((4, 4), dtype=torch.float32)
    calls = [
        lambda: nv.nvfp4_quantize(x, q, ws),
        lambda: nv.quantize(x),
        lambda: nv.nvfp4_dequantize(q, torch.zeros((4, 64))),
        lambda: nv.nvfp4_gemm(q, q, y, ws),
        lambda: nv.nvfp4_linear_fused(x, q, ws, nv.EPI_STORE, y=y),
        lambda: nv.nvfp4_linear_noalloc(x, q, y),
        lambda: nv.nvfp4_get_device_status(ws),
        lambda: nv.nvfp4_selftest_bounded_wait(ws, 1000),
    ]
    for call in calls:
        with pytest.raises(TypeError, match="CUDA tensors"):
            call()


def test_binding_refuses_matrices_without_contiguous_rows():
    """The C ABI describes a matrix by pointer and row pitch: a view whose
    elements within a row are not adjacent is refused (a plain check, so it
    also holds under python -O)."""
    import torch
    x = torch.zeros((8, 128))
    q = nv.NVFP4Tensor(torch.zeros((8, 32), dtype=torch.uint8), torch.zeros(512, dtype=torch.uint8),
                       torch.zeros(4), 8, 64)
    ws = torch.zeros(1 << 16, dtype=torch.uint8)
    for call in (lambda: nv.nvfp4_quantize(x[:, ::2], q, ws), lambda: nv.nvfp4_quantize(x.t(), q, ws),
                 lambda: nv.nvfp4_linear_fused(x[:, ::2], q, ws, nv.EPI_STORE, y=x[:, :8]),
                 lambda: nv.nvfp4_linear_fused(x[:, :64], q, ws, nv.EPI_STORE, y=x[:, ::16]),
                 lambda: nv.nvfp4_gemm(q, q, x[:, ::16], ws)):
        with pytest.raises(ValueError, match="contiguous rows"):
            call()


def test_binding_refuses_short_buffers_and_wrong_output_shapes():
    """The C ABI cannot see buffer sizes or an output's row count: the binding
    refuses an NVFP4 tensor whose buffers are too small or not contiguous, and
    an output whose shape is not the one the call writes."""
    import torch

    def q(rows=8, cols=64, codes=None, scales=None, g=None):
        return nv.NVFP4Tensor(codes if codes is not None else torch.zeros((rows, cols // 2), dtype=torch.uint8),
                              scales if scales is not None else torch.zeros(nv.scales_bytes(rows, cols),
                                                                            dtype=torch.uint8),
                              g if g is not None else torch.zeros(4), rows, cols)

    x, ws = torch.zeros((8, 64)), torch.zeros(1 << 16, dtype=torch.uint8)
    with pytest.raises(ValueError, match="scales"):
        nv.nvfp4_quantize(x, q(scales=torch.zeros(100, dtype=torch.uint8)), ws)
    with pytest.raises(ValueError, match="codes"):
        nv.nvfp4_quantize(x, q(codes=torch.zeros((8, 31), dtype=torch.uint8)), ws)
    with pytest.raises(ValueError, match="not contiguous"):
        nv.nvfp4_quantize(x, q(codes=torch.zeros((32, 8), dtype=torch.uint8).t()), ws)
    with pytest.raises(TypeError, match="float32"):
        nv.nvfp4_quantize(x, q(g=torch.zeros(4, dtype=torch.float64)), ws)
    a, b = q(8, 64), q(16, 64)
    with pytest.raises(ValueError, match="expected \\(8, 16\\)"):
        nv.nvfp4_gemm(a, b, torch.zeros((7, 16)), ws)
    with pytest.raises(ValueError, match="expected \\(8, 64\\)"):
        nv.nvfp4_dequantize(a, torch.zeros((8, 32)))
    with pytest.raises(ValueError, match="expected \\(8, 16\\)"):
        nv.nvfp4_linear_fused(x, b, ws, nv.EPI_STORE, y=torch.zeros((8, 15)))
    with pytest.raises(ValueError, match="expected \\(8, 16\\)"):
        nv.nvfp4_linear_noalloc(x, b, torch.zeros((9, 16)))
    with pytest.raises(ValueError, match="scales"):
        nv.nvfp4_linear_fused(x, b, ws, nv.EPI_SILU_MUL_REQUANT, w_up=b,
                              y_q=q(8, 16, scales=torch.zeros(8, dtype=torch.uint8)))


_C_CALLER = r"""
#include <stdio.h>
#include <string.h>
#include "nvfp4.h"

int main(void) {
    nvfp4_tensor t;
    memset(&t, 0, sizeof t);
    if (nvfp4_scales_bytes(8, 5120) != (size_t)128 * 320) return 1;
    if (nvfp4_codes_bytes(8192, 5120) != (size_t)8192 * 2560) return 2;
    if (nvfp4_version() <= 0) return 3;
    if (strcmp(nvfp4_status_string(NVFP4_ERR_INVALID_ARG), "invalid argument") != 0) return 4;
    /* argument errors return before any device call */
    if (nvfp4_quantize(NULL, NVFP4_BF16, 4, 64, 64, &t, NULL, 0, NULL) != NVFP4_ERR_INVALID_ARG) return 5;
    if (nvfp4_gemm(NULL, NULL, NULL, NVFP4_BF16, 0, NULL, 0, NULL) != NVFP4_ERR_INVALID_ARG) return 6;
    puts("ok");
    return 0;
}
"""


def test_header_is_plain_c_and_a_c_program_links_and_calls_the_library(tmp_path):
    """The boundary is a C ABI: a C99 program built with warnings as errors
    includes the header, links libnvfp4.so and makes host-only calls (sizes,
    version, status strings, argument errors); the header also parses as C++."""
    import shutil
    import subprocess
    if not shutil.which("gcc"):
        pytest.skip("gcc not available")
    src = tmp_path / "caller.c"
    src.write_text(_C_CALLER)
    exe = tmp_path / "caller"
    pkg = os.path.join(ROOT, "nvfp4_block_scaled_21_b200")
    inc = os.path.join(ROOT, "include")
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", inc, str(src),
                        "-L", pkg, "-lnvfp4", f"-Wl,-rpath,{pkg}", "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and run.stdout.strip() == "ok", (run.returncode, run.stdout, run.stderr)
    if shutil.which("g++"):
        cxx = subprocess.run(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-x", "c++",
                              "-I", inc, str(src)], capture_output=True, text=True)
        assert cxx.returncode == 0, cxx.stderr


def test_package_fails_loudly_without_library(tmp_path):
    """The binding refuses to import when libnvfp4.so is absent: no CPU fallback."""
    import subprocess
    import sys
    import shutil
    pkg = tmp_path / "nvfp4_block_scaled_21_b200"
    shutil.copytree(os.path.join(ROOT, "nvfp4_block_scaled_21_b200"), pkg,
                    ignore=shutil.ignore_patterns("*.so", "csrc", "__pycache__"))
    r = subprocess.run([sys.executable, "-c", "import nvfp4_block_scaled_21_b200"], cwd=tmp_path,
                       capture_output=True, text=True)
    assert r.returncode != 0 and "libnvfp4.so is missing" in r.stderr


def _mx(codes=16, scales=16, rows=4, cols=64):
    return nv.CMXTensor(codes, scales, rows, cols)


def test_mx_sizes_and_argument_checks_without_launch():
    """MXFP4: scale bytes roundup(rows,128) x roundup(cols/32,4); each call
    below breaks exactly one rule of nvfp4_mx_quantize / nvfp4_mx_gemm."""
    assert nv.mx_scales_bytes(8192, 5120) == 8192 * 160
    assert nv.mx_scales_bytes(1, 32) == 128 * 4
    assert nv.mx_scales_bytes(130, 96) == 256 * 4
    lib = nv.lib()

    def q(x=16, xt=nv.BF16, r=4, c=64, ld=64, o=_mx()):
        return lib.nvfp4_mx_quantize(x, xt, r, c, ld, ctypes.byref(o) if o else None, None)

    assert q(x=None) == nv.ERR_INVALID_ARG
    assert q(xt=3) == nv.ERR_INVALID_ARG
    assert q(ld=32) == nv.ERR_INVALID_ARG
    assert q(o=None) == nv.ERR_INVALID_ARG
    assert q(o=_mx(rows=5)) == nv.ERR_INVALID_ARG
    assert q(c=48, ld=48, o=_mx(cols=48)) == nv.ERR_UNSUPPORTED_SHAPE            # cols % 32
    assert q(x=24) == nv.ERR_MISALIGNED
    assert q(o=_mx(scales=24)) == nv.ERR_MISALIGNED

    a, b = _mx(rows=8, cols=128), _mx(rows=32, cols=128)

    def g(a_=a, b_=b, y=16, yt=nv.BF16, ldy=32, ws=4096, wb=1 << 20):
        return lib.nvfp4_mx_gemm(ctypes.byref(a_), ctypes.byref(b_), y, yt, ldy, ws, wb, None)

    assert g(y=None) == nv.ERR_INVALID_ARG
    assert g(b_=_mx(rows=32, cols=64)) == nv.ERR_INVALID_ARG                        # K mismatch
    assert g(a_=_mx(rows=8, cols=96), b_=_mx(rows=32, cols=96)) == nv.ERR_UNSUPPORTED_SHAPE   # K % 64
    assert g(ldy=16) == nv.ERR_INVALID_ARG
    assert g(ldy=36) == nv.ERR_MISALIGNED
    assert g(wb=8) == nv.ERR_WORKSPACE
    assert g(yt=4) == nv.ERR_INVALID_ARG


def test_w4a8_argument_checks_without_launch():
    """MXFP8 quantizer and W4A8 GEMM / linear layer: each call below breaks
    exactly one rule (K a multiple of 128 and 32-byte aligned weight codes,
    which the unpacking copy of the weights needs)."""
    lib = nv.lib()

    def mx8(elems=16, scales=16, rows=4, cols=128):
        return nv.CMX8Tensor(elems, scales, rows, cols)

    def q(x=16, xt=nv.BF16, r=4, c=128, ld=128, o=mx8()):
        return lib.nvfp4_mx8_quantize(x, xt, r, c, ld, ctypes.byref(o) if o else None, None)

    assert q(x=None) == nv.ERR_INVALID_ARG
    assert q(xt=3) == nv.ERR_INVALID_ARG
    assert q(ld=64) == nv.ERR_INVALID_ARG
    assert q(o=mx8(rows=5)) == nv.ERR_INVALID_ARG
    assert q(c=48, ld=48, o=mx8(cols=48)) == nv.ERR_UNSUPPORTED_SHAPE          # cols % 32
    assert q(x=24) == nv.ERR_MISALIGNED
    assert q(o=mx8(elems=24)) == nv.ERR_MISALIGNED

    def g(a_=mx8(rows=8), b_=_mx(codes=32, rows=32, cols=128), y=16, yt=nv.BF16, ldy=32, ws=4096, wb=1 << 20):
        return lib.nvfp4_w4a8_gemm(ctypes.byref(a_), ctypes.byref(b_), y, yt, ldy, ws, wb, None)

    assert g(y=None) == nv.ERR_INVALID_ARG
    assert g(b_=_mx(codes=32, rows=32, cols=256)) == nv.ERR_INVALID_ARG                       # K mismatch
    assert g(a_=mx8(rows=8, cols=192), b_=_mx(codes=32, rows=32, cols=192)) == nv.ERR_UNSUPPORTED_SHAPE
    assert g(b_=_mx(codes=48, rows=32, cols=128)) == nv.ERR_MISALIGNED                        # codes % 32
    assert g(ldy=36) == nv.ERR_MISALIGNED
    assert g(wb=8) == nv.ERR_WORKSPACE

    def lin(x=16, K=128, w=_mx(codes=32, rows=32, cols=128), ldy=32, xq=None, wb=1 << 20):
        return lib.nvfp4_w4a8_linear(x, nv.BF16, 8, K, K, ctypes.byref(w), 16, nv.BF16, ldy,
                                     ctypes.byref(xq) if xq else None, 4096, wb, None)

    assert lin(x=None) == nv.ERR_INVALID_ARG
    assert lin(K=192, w=_mx(codes=32, rows=32, cols=192)) == nv.ERR_UNSUPPORTED_SHAPE          # K % 128
    assert lin(w=_mx(codes=48, rows=32, cols=128)) == nv.ERR_MISALIGNED
    assert lin(xq=mx8(rows=7)) == nv.ERR_INVALID_ARG
    assert lin(wb=8) == nv.ERR_WORKSPACE
