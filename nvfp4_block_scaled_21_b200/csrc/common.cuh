// common.cuh -- shapes, the tiled scale layout and small helpers shared by the
// CUDA kernels of the library (never by the CPU oracle).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace nvfp4 {

constexpr int kBlock = 16;           // values per microblock (NVFP4 wiki page, "技術原理")

// Operand formats of the GEMM kernels.
constexpr int kFmtNV = 0;     // NVFP4: E2M1 (packed), UE4M3 per 16, kind::mxf4nvf4 4X, K = 64 per MMA
constexpr int kFmtMX = 1;     // MXFP4: E2M1 (packed), UE8M0 per 32, kind::mxf4 2X, K = 64 per MMA
constexpr int kFmtW4A8 = 2;   // MXFP4 weights x MXFP8 activations (8-bit containers in shared memory),
                              // UE8M0 per 32, kind::mxf8f6f4 1X, K = 32 per MMA
constexpr float kTensorScaleDiv = 2688.0f;   // 6 (E2M1 max) * 448 (E4M3 max)

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

// Number of 16-element blocks per row, padded to a multiple of 4 (one 32-bit
// scale word per 64 columns).
__host__ __device__ __forceinline__ int64_t kb4_of(int64_t cols) { return round_up(cols / kBlock, 4); }

// Byte offset of the scale of block kb of row r in the tiled layout: 128-row x
// 4-block atoms of 512 bytes, row r%32 at 16*(r%32), row quarter (r/32)%4 at
// 4*((r/32)%4), block kb%4 at kb%4.  Lane l of every TMEM lane quarter
// receives the atom's 16 bytes at 16*l (the GEMMs' scale warps copy them with
// tcgen05.st), which is where the block-scaled MMA reads the scales: lane
// r%32 of every quarter, column (r/32)%4, byte kb%4.
__host__ __device__ __forceinline__ int64_t scale_offset(int64_t r, int64_t kb, int64_t kb4) {
    int64_t tile = (r >> 7) * (kb4 >> 2) + (kb >> 2);
    return tile * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (kb & 3);
}

// Largest GEMM sizes the kernels index in 32 bits: rows of either operand (and
// sums of two row indices), and K (the TMA x coordinate reaches K/2 bytes).
constexpr int64_t kMaxGemmRows = 0x3fffffff;            // INT32_MAX / 2
constexpr int64_t kMaxGemmK = int64_t(1) << 31;

// An fp32 result in the output type: bf16 by round-to-nearest-even.
template <typename OutT> __device__ __forceinline__ OutT to_out(float v);
template <> __device__ __forceinline__ float to_out<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 to_out<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// Running max |y| over the output values one thread stores, exact: bf16
// words as two 15-bit magnitudes (non-negative floats order like their bit
// patterns), fp32 values by fmaxf.  value() gives it as an fp32 number, in the
// format of the quantizer's first pass (per-CTA partial maxima), so that a
// GEMM whose output is re-quantized needs only the encode pass afterwards.
struct YMax {
    uint32_t b = 0u;
    float f = 0.0f;
    __device__ __forceinline__ void bf16x2(uint32_t w) { b = __vmaxu2(b, w & 0x7fff7fffu); }
    __device__ __forceinline__ void bf16(__nv_bfloat16 v) {
        b = __vmaxu2(b, static_cast<uint32_t>(__bfloat16_as_ushort(v)) & 0x7fffu);
    }
    __device__ __forceinline__ void f32(float v) { f = fmaxf(f, fabsf(v)); }
    template <typename OutT> __device__ __forceinline__ void add(OutT v);
    __device__ __forceinline__ float value() const {
        return fmaxf(f, __uint_as_float(max(b & 0xffffu, b >> 16) << 16));
    }
};
template <> __device__ __forceinline__ void YMax::add<float>(float v) { f32(v); }
template <> __device__ __forceinline__ void YMax::add<__nv_bfloat16>(__nv_bfloat16 v) { bf16(v); }

// Workspace layout: [0,16) status words, [256, ...) scratch.
constexpr size_t kWsStatusBytes = 256;
constexpr size_t kGridBarOff = 128;    // grid meeting point: arrival count, generation
constexpr int kMaxAmaxPartials = 4096;

// Debug build (compiled with NVFP4_DEBUG_CHECKS): every direct global store
// of the kernels is checked against the extent of the buffer it writes; a
// store that would leave it is skipped and NVFP4_ERR_BOUNDS is recorded in
// the status word (no trap).  In the release build the check compiles away.
constexpr uint32_t kStatusBoundsBit = 1u << 8;      // bit index == NVFP4_ERR_BOUNDS
#ifdef NVFP4_DEBUG_CHECKS
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif
__device__ __forceinline__ bool store_ok(const void *p, size_t bytes, const void *base, size_t extent,
                                         uint32_t *status) {
    if constexpr (!kDebugChecks) {
        return true;
    } else {
        const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(base);
        const bool ok = a >= b && a + bytes <= b + extent;
        if (!ok && status != nullptr) atomicOr(status, kStatusBoundsBit);
        return ok;
    }
}
// Bytes of a row-major [rows][cols] matrix with row pitch ld (elements of eb bytes).
__host__ __device__ __forceinline__ size_t matrix_extent(int64_t rows, int64_t cols, int64_t ld, int64_t eb) {
    return rows <= 0 || cols <= 0 ? 0 : static_cast<size_t>(((rows - 1) * ld + cols) * eb);
}

}  // namespace nvfp4
