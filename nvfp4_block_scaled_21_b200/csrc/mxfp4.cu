// mxfp4.cu -- the MXFP4 quantizer.
//
// MXFP4 (eefocus.com article on FP4 vs INT4, section
// "FP4被视为下一代AI计算的核心标准"): 32 consecutive E2M1 elements share one
// 8-bit E8M0 scale (a power of two), about 4.25 bits per value, and there is
// no second-level tensor scale.  The page gives no rule for choosing the
// scale; the one used here is the smallest power of two X = 2^e that brings
// the block's largest magnitude into the E2M1 range, bamax <= 6 X, i.e.
// e = ceil(log2(bamax / 6)), clamped to E8M0's [-127, 127] (an all-zero block
// gets byte 0).  From bamax's fp32 bits (bamax = (1 + m/2^23) 2^k):
// bamax / 6 <= 2^(k-2) exactly when m <= 2^22 (bamax <= 1.5 * 2^k), so
// e = k - 2 then and k - 1 otherwise.  Elements are E2M1 RNE of x / X, which is
// exact (a multiply by 2^-e), with the NVFP4 rules for ties and signs.
//
// One pass (no tensor amax), one thread per 32-value block; codes packed as in
// NVFP4 (element 2j in the low nibble of byte j) and scale bytes in the same
// 512-byte tiled atoms, with kb counting 32-value blocks: an atom covers 128
// rows x 128 columns, i.e. two K steps of the block-scaled MMA.
#include "common.cuh"
#include "encode.cuh"
#include "kernels.cuh"

namespace nvfp4 {

namespace {

template <typename T> struct MxBlock;
template <> struct MxBlock<__nv_bfloat16> {
    static constexpr int W = 16;   // 32-bit words per 32-value block
    __device__ static void load(const __nv_bfloat16 *p, uint32_t (&w)[16]) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 a = load_item(p + 8 * i);
            w[4 * i] = a.x; w[4 * i + 1] = a.y; w[4 * i + 2] = a.z; w[4 * i + 3] = a.w;
        }
    }
    __device__ static uint32_t absmax_bits(const uint32_t (&w)[16]) {
        uint32_t m = 0u;
#pragma unroll
        for (int i = 0; i < 16; ++i) m = __vmaxu2(m, w[i] & 0x7fff7fffu);
        return max(m & 0xffffu, m >> 16) << 16;
    }
    __device__ static float val(const uint32_t (&w)[16], int k) {
        return __uint_as_float((k & 1) ? (w[k >> 1] & 0xffff0000u) : (w[k >> 1] << 16));
    }
};
template <> struct MxBlock<float> {
    static constexpr int W = 32;
    __device__ static void load(const float *p, uint32_t (&w)[32]) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint4 a = load_item(p + 4 * i);
            w[4 * i] = a.x; w[4 * i + 1] = a.y; w[4 * i + 2] = a.z; w[4 * i + 3] = a.w;
        }
    }
    __device__ static uint32_t absmax_bits(const uint32_t (&w)[32]) {
        uint32_t m = 0u;
#pragma unroll
        for (int i = 0; i < 32; ++i) m = max(m, w[i] & 0x7fffffffu);
        return m;
    }
    __device__ static float val(const uint32_t (&w)[32], int k) { return __uint_as_float(w[k]); }
};

// E8M0 byte of a block whose largest magnitude has fp32 bits b (finite).
__device__ __forceinline__ uint32_t e8m0_of(uint32_t b) {
    if (b == 0u) return 0u;
    const int k = static_cast<int>(b >> 23) - 127;    // subnormal bamax: k = -127
    int e = ((b & 0x7fffffu) <= 0x400000u) ? k - 2 : k - 1;
    e = max(e, -127);                                 // finite fp32 keeps e <= 126
    return static_cast<uint32_t>(e + 127);
}

// one code byte from two values: lo in the low nibble
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
    uint32_t out;
    asm("{\n\t.reg .b8 b;\n\tcvt.rn.satfinite.e2m1x2.f32 b, %2, %1;\n\tcvt.u32.u8 %0, b;\n\t}"
        : "=r"(out)
        : "f"(lo), "f"(hi));
    return out;
}

template <typename T>
__global__ void __launch_bounds__(256) mx_quantize_kernel(const T *__restrict__ x, int64_t rows, int64_t cols,
                                                          int64_t ld, uint8_t *__restrict__ codes,
                                                          uint8_t *__restrict__ scales) {
    constexpr int W = MxBlock<T>::W;
    const int64_t bpr = cols / 32, total = rows * bpr, kb4 = round_up(bpr, 4);
    const int64_t S = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int lane = threadIdx.x & 31;
    const bool word_scales = (bpr & 3) == 0;
    const int64_t nwin = ceil_div(total, S);          // the same for every thread: full-mask shuffles
    for (int64_t w = 0; w < nwin; ++w) {
        const int64_t b = t + w * S;
        const bool valid = b < total;
        const int64_t r = valid ? b / bpr : 0, j = valid ? b - r * bpr : 0;
        uint32_t v[W];
        if (valid) {
            MxBlock<T>::load(x + r * ld + j * 32, v);
        } else {
#pragma unroll
            for (int k = 0; k < W; ++k) v[k] = 0u;
        }
        const uint32_t sb = e8m0_of(MxBlock<T>::absmax_bits(v));
        const float mul = __uint_as_float((254u - sb) << 23);   // 2^-e, e = sb - 127 in [-127, 126]
        uint32_t c[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t word = 0u;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int e0 = 8 * q + 2 * k;
                word |= e2m1x2(__fmul_rn(MxBlock<T>::val(v, e0), mul), __fmul_rn(MxBlock<T>::val(v, e0 + 1), mul))
                        << (8 * k);
            }
            c[q] = word;
        }
        uint32_t sw = sb;
        sw |= __shfl_down_sync(0xffffffffu, sb, 1) << 8;
        sw |= __shfl_down_sync(0xffffffffu, sb, 2) << 16;
        sw |= __shfl_down_sync(0xffffffffu, sb, 3) << 24;
        if (valid) {
            *reinterpret_cast<uint4 *>(codes + r * (cols / 2) + j * 16) = make_uint4(c[0], c[1], c[2], c[3]);
            if (word_scales) {
                if ((lane & 3) == 0) *reinterpret_cast<uint32_t *>(scales + scale_offset(r, j, kb4)) = sw;
            } else {
                scales[scale_offset(r, j, kb4)] = static_cast<uint8_t>(sb);
            }
        }
    }
    // Zero the layout's padding: blocks [bpr, kb4) of real rows, and every
    // block of rows [rows, roundup(rows, 128)).
    const int64_t pad_a = rows * (kb4 - bpr);
    for (int64_t i = t; i < pad_a; i += S) {
        const int64_t r = i / (kb4 - bpr), q = bpr + (i - r * (kb4 - bpr));
        scales[scale_offset(r, q, kb4)] = 0;
    }
    const int64_t pad_b = (round_up(rows, 128) - rows) * kb4;
    for (int64_t i = t; i < pad_b; i += S) {
        const int64_t r = rows + i / kb4, q = i - (i / kb4) * kb4;
        scales[scale_offset(r, q, kb4)] = 0;
    }
}

// ---------------------------------------------------------------------------
// MXFP8 (the activations of the W4A8 product): the same 32-value blocks and
// E8M0 scales, with E4M3 elements.  FP4 weights with FP8 activations is the
// eefocus.com article's W4A8 (the Zhouyi X3 passage); with MX scales on both
// operands it is the tensor cores' native mixed FP4 x FP8 product.  Scale:
// the smallest power of two X with bamax <= 448 X (e = ceil(log2(bamax /
// 448)), clamped to [-127, 127]): with bamax = f 2^j (f = 1 + m/2^23 in
// [1, 2)) and 448 = 1.75 * 2^8, bamax <= 448 * 2^(j-8) exactly when f <= 1.75
// (m <= 0x600000), and 2^(j-9) is always too small, so e = j - 8 then and
// j - 7 otherwise.
// Elements: E4M3 RNE satfinite of x * 2^-e (exact).
// ---------------------------------------------------------------------------

// E8M0 byte of a block whose largest magnitude has fp32 bits b (finite).
__device__ __forceinline__ uint32_t e8m0_of_mx8(uint32_t b) {
    if (b == 0u) return 0u;
    const int j = static_cast<int>(b >> 23) - 127;    // subnormal bamax: j = -127
    int e = ((b & 0x7fffffu) <= 0x600000u) ? j - 8 : j - 7;
    e = max(e, -127);
    return static_cast<uint32_t>(e + 127);
}

template <typename T>
__global__ void __launch_bounds__(256) mx8_quantize_kernel(const T *__restrict__ x, int64_t rows, int64_t cols,
                                                           int64_t ld, uint8_t *__restrict__ elems,
                                                           uint8_t *__restrict__ scales) {
    constexpr int W = MxBlock<T>::W;
    const int64_t bpr = cols / 32, total = rows * bpr, kb4 = round_up(bpr, 4);
    const int64_t S = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int lane = threadIdx.x & 31;
    const bool word_scales = (bpr & 3) == 0;
    const int64_t nwin = ceil_div(total, S);          // the same for every thread: full-mask shuffles
    for (int64_t w = 0; w < nwin; ++w) {
        const int64_t b = t + w * S;
        const bool valid = b < total;
        const int64_t r = valid ? b / bpr : 0, j = valid ? b - r * bpr : 0;
        uint32_t v[W];
        if (valid) {
            MxBlock<T>::load(x + r * ld + j * 32, v);
        } else {
#pragma unroll
            for (int k = 0; k < W; ++k) v[k] = 0u;
        }
        const uint32_t sb = e8m0_of_mx8(MxBlock<T>::absmax_bits(v));
        const float mul = __uint_as_float((254u - sb) << 23);   // 2^-e, e = sb - 127 in [-127, 126]
        uint32_t out[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            uint16_t lo, hi;
            const int e0 = 4 * q;
            asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
                : "=h"(lo)
                : "f"(__fmul_rn(MxBlock<T>::val(v, e0 + 1), mul)), "f"(__fmul_rn(MxBlock<T>::val(v, e0), mul)));
            asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
                : "=h"(hi)
                : "f"(__fmul_rn(MxBlock<T>::val(v, e0 + 3), mul)), "f"(__fmul_rn(MxBlock<T>::val(v, e0 + 2), mul)));
            out[q] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
        }
        uint32_t sw = sb;
        sw |= __shfl_down_sync(0xffffffffu, sb, 1) << 8;
        sw |= __shfl_down_sync(0xffffffffu, sb, 2) << 16;
        sw |= __shfl_down_sync(0xffffffffu, sb, 3) << 24;
        if (valid) {
            uint4 *dst = reinterpret_cast<uint4 *>(elems + r * cols + j * 32);
            dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
            dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
            if (word_scales) {
                if ((lane & 3) == 0) *reinterpret_cast<uint32_t *>(scales + scale_offset(r, j, kb4)) = sw;
            } else {
                scales[scale_offset(r, j, kb4)] = static_cast<uint8_t>(sb);
            }
        }
    }
    const int64_t pad_a = rows * (kb4 - bpr);
    for (int64_t i = t; i < pad_a; i += S) {
        const int64_t r = i / (kb4 - bpr), q = bpr + (i - r * (kb4 - bpr));
        scales[scale_offset(r, q, kb4)] = 0;
    }
    const int64_t pad_b = (round_up(rows, 128) - rows) * kb4;
    for (int64_t i = t; i < pad_b; i += S) {
        const int64_t r = rows + i / kb4, q = i - (i / kb4) * kb4;
        scales[scale_offset(r, q, kb4)] = 0;
    }
}

}  // namespace

cudaError_t launch_mx8_quantize(const void *x, bool bf16, int64_t rows, int64_t cols, int64_t ld, uint8_t *elems,
                                uint8_t *scales, int num_sms, cudaStream_t stream) {
    if (rows == 0 || cols == 0) return cudaSuccess;
    int64_t blocks = ceil_div(rows * (cols / 32), 256);
    const int64_t cap = static_cast<int64_t>(num_sms) * 4;
    blocks = blocks < 1 ? 1 : (blocks < cap ? blocks : cap);
    if (bf16)
        mx8_quantize_kernel<__nv_bfloat16><<<static_cast<int>(blocks), 256, 0, stream>>>(
            static_cast<const __nv_bfloat16 *>(x), rows, cols, ld, elems, scales);
    else
        mx8_quantize_kernel<float><<<static_cast<int>(blocks), 256, 0, stream>>>(static_cast<const float *>(x), rows,
                                                                                cols, ld, elems, scales);
    return cudaGetLastError();
}

cudaError_t launch_mx_quantize(const void *x, bool bf16, int64_t rows, int64_t cols, int64_t ld, uint8_t *codes,
                               uint8_t *scales, int num_sms, cudaStream_t stream) {
    if (rows == 0 || cols == 0) return cudaSuccess;
    static const int occ[2] = {[]() {
                                   int n = 0;
                                   if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, mx_quantize_kernel<float>, 256,
                                                                                     0) != cudaSuccess || n < 1)
                                       n = 1;
                                   return n;
                               }(),
                               []() {
                                   int n = 0;
                                   if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                                           &n, mx_quantize_kernel<__nv_bfloat16>, 256, 0) != cudaSuccess || n < 1)
                                       n = 1;
                                   return n;
                               }()};
    int64_t blocks = ceil_div(rows * (cols / 32), 256);
    const int64_t cap = static_cast<int64_t>(num_sms) * occ[bf16];
    blocks = blocks < 1 ? 1 : (blocks < cap ? blocks : cap);
    if (bf16)
        mx_quantize_kernel<__nv_bfloat16><<<static_cast<int>(blocks), 256, 0, stream>>>(
            static_cast<const __nv_bfloat16 *>(x), rows, cols, ld, codes, scales);
    else
        mx_quantize_kernel<float><<<static_cast<int>(blocks), 256, 0, stream>>>(static_cast<const float *>(x), rows,
                                                                               cols, ld, codes, scales);
    return cudaGetLastError();
}

}  // namespace nvfp4
