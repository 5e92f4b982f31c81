// quantize.cu -- the two-pass NVFP4 quantizer and the dequantizer.
//
// Format: NVFP4 wiki page (newton.com.tw), section "技術原理": E2M1 elements,
// one E4M3 scale per 16-element microblock, one FP32 scale per tensor.
//
// Pass 1 (amax_partials_kernel): every thread streams 16-byte vectors of x,
//   keeps the running max of |x| on the bit patterns (exact), reduces through
//   warp shuffles and shared memory, and writes one partial max per CTA to the
//   workspace (no atomics, nothing to reset between calls).
// Pass 2 (encode_kernel): every CTA reduces the partial maxima (a few KB from
//   L2), derives g = amax/2688 on the device, and encodes the tensor, walking
//   the windows in the same order as pass 1 (on B200 a second forward sweep
//   finds part of x in L2).  One thread owns one 16-element block; the E4M3
//   scale and the E2M1 codes come from the hardware RNE-satfinite
//   conversions; codes go out as one 8-byte store per block and scales as one
//   32-bit word per four blocks in the tiled layout the tensor cores read.
#include "common.cuh"
#include "kernels.cuh"

namespace nvfp4 {

template <typename T> struct Elem;
template <> struct Elem<__nv_bfloat16> {
    static constexpr int kPerItem = 8;   // 16 bytes
};
template <> struct Elem<float> {
    static constexpr int kPerItem = 4;
};

// |x| max of one 16-byte item as fp32 (exact: max is taken on the bit
// patterns of |x|, which order like the values for non-negative floats).
__device__ __forceinline__ float item_absmax(const uint4 &v, __nv_bfloat16 *) {
    uint32_t a = __vmaxu2(v.x & 0x7fff7fffu, v.y & 0x7fff7fffu);
    uint32_t b = __vmaxu2(v.z & 0x7fff7fffu, v.w & 0x7fff7fffu);
    uint32_t m = __vmaxu2(a, b);
    uint32_t h = max(m & 0xffffu, m >> 16);
    return __uint_as_float(h << 16);
}
__device__ __forceinline__ float item_absmax(const uint4 &v, float *) {
    uint32_t m = max(max(v.x & 0x7fffffffu, v.y & 0x7fffffffu),
                     max(v.z & 0x7fffffffu, v.w & 0x7fffffffu));
    return __uint_as_float(m);
}

__device__ __forceinline__ uint4 load_item(const void *p) {
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

// Walks the items (16-byte vectors) of a [rows][cols] matrix with pitch ld:
// item i is row i / ipr, vector i % ipr.  Tracks (row, vector) incrementally
// so the loop needs no division.
struct ItemCursor {
    int64_t r, j;
    __device__ __forceinline__ void set(int64_t i, int64_t ipr) { r = i / ipr; j = i - r * ipr; }
    __device__ __forceinline__ void advance(int64_t dr, int64_t dj, int64_t ipr) {
        r += dr; j += dj;
        if (j >= ipr) { j -= ipr; r += 1; }
    }
    __device__ __forceinline__ void retreat(int64_t dr, int64_t dj, int64_t ipr) {
        r -= dr; j -= dj;
        if (j < 0) { j += ipr; r -= 1; }
    }
};

// ---------------------------------------------------------------------------
// Pass 1: per-CTA partial maxima of |x|.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) amax_partials_kernel(const T *__restrict__ x, int64_t rows,
                                                            int64_t cols, int64_t ld,
                                                            float *__restrict__ partials) {
    constexpr int EPI = Elem<T>::kPerItem;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");   // let the encode pass queue up
    float m = 0.0f;
    if (ld == cols && rows * cols / EPI < (int64_t(1) << 31)) {
        // contiguous: one flat stream of 16-byte vectors, 32-bit indices,
        // 8 loads in flight per thread
        const uint32_t total = static_cast<uint32_t>(rows * cols / EPI);
        const uint32_t S = gridDim.x * blockDim.x;
        const uint4 *v16 = reinterpret_cast<const uint4 *>(x);
        constexpr int U = 8;
        uint32_t i = blockIdx.x * blockDim.x + threadIdx.x;
        for (; i + (U - 1) * S < total; i += U * S) {
            uint4 v[U];
#pragma unroll
            for (int u = 0; u < U; ++u) v[u] = __ldg(v16 + i + u * S);
#pragma unroll
            for (int u = 0; u < U; ++u) m = fmaxf(m, item_absmax(v[u], static_cast<T *>(nullptr)));
        }
        for (; i < total; i += S) m = fmaxf(m, item_absmax(__ldg(v16 + i), static_cast<T *>(nullptr)));
    } else {
        const int64_t ipr = cols / EPI;
        const int64_t total = rows * ipr;
        const int64_t S = static_cast<int64_t>(gridDim.x) * blockDim.x;
        const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
        const int64_t dr = S / ipr, dj = S - dr * ipr;
        ItemCursor c;
        c.set(t, ipr);
        constexpr int U = 4;
        for (int64_t i = t; i < total; i += U * S) {
            uint4 v[U];
            ItemCursor cu = c;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (i + u * S < total)
                    v[u] = load_item(x + cu.r * ld + cu.j * EPI);
                else
                    v[u] = make_uint4(0, 0, 0, 0);
                cu.advance(dr, dj, ipr);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) m = fmaxf(m, item_absmax(v[u], static_cast<T *>(nullptr)));
            c = cu;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float wmax[32];
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        float v = threadIdx.x < (blockDim.x >> 5) ? wmax[threadIdx.x] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (threadIdx.x == 0) partials[blockIdx.x] = v;
    }
}

// ---------------------------------------------------------------------------
// Conversions (hardware RNE with saturation to the largest finite value).
// ---------------------------------------------------------------------------

// E4M3 byte of a non-negative fp32 t.
__device__ __forceinline__ uint32_t e4m3_of(float t) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(t));
    return r & 0xffu;
}

// fp32 value of an E4M3 byte (exact through f16).
__device__ __forceinline__ float e4m3_value(uint32_t s) {
    uint32_t h2;
    uint16_t in = static_cast<uint16_t>(s);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xffffu)));
}

// Reduce the pass-1 partial maxima (every CTA does it; it is a few KB of L2).
__device__ __forceinline__ float reduce_partials(const float *__restrict__ partials, int n) {
    float m = 0.0f;
    for (int i = threadIdx.x; i < n; i += blockDim.x) m = fmaxf(m, partials[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float wmax[32];
    __shared__ float result;
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        float v = threadIdx.x < (blockDim.x >> 5) ? wmax[threadIdx.x] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (threadIdx.x == 0) result = v;
    }
    __syncthreads();
    return result;
}

// ---------------------------------------------------------------------------
// Pass 2: encode.  One thread owns one 16-value block: its amax needs no
// shuffle, the scale arithmetic runs once per block, the 16 products are 8
// packed f32x2 multiplies (per-lane IEEE round-to-nearest, identical to 16
// scalar ones), and the 8 code bytes leave as one 8-byte store.  Four
// neighbouring lanes hold the four blocks of a 64-column group; their scale
// bytes are gathered into one 32-bit word in the tiled layout.
// ---------------------------------------------------------------------------

// 16 values of one block as fp32 pairs, from 2 (bf16) or 4 (fp32) 16-byte loads.
__device__ __forceinline__ void load_block(const __nv_bfloat16 *p, uint32_t (&w)[8]) {
    const uint4 a = load_item(p), b = load_item(p + 8);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
}
__device__ __forceinline__ float block_absmax(const uint32_t (&w)[8], __nv_bfloat16 *) {
    uint32_t m = __vmaxu2(__vmaxu2(w[0] & 0x7fff7fffu, w[1] & 0x7fff7fffu),
                          __vmaxu2(w[2] & 0x7fff7fffu, w[3] & 0x7fff7fffu));
    m = __vmaxu2(m, __vmaxu2(__vmaxu2(w[4] & 0x7fff7fffu, w[5] & 0x7fff7fffu),
                             __vmaxu2(w[6] & 0x7fff7fffu, w[7] & 0x7fff7fffu)));
    return __uint_as_float(max(m & 0xffffu, m >> 16) << 16);
}
// element pair k of a bf16 block as a packed (lo, hi) fp32 pair
__device__ __forceinline__ uint64_t pair_f32(const uint32_t (&w)[8], int k, __nv_bfloat16 *) {
    return static_cast<uint64_t>(w[k] << 16) | (static_cast<uint64_t>(w[k] & 0xffff0000u) << 32);
}

__device__ __forceinline__ void load_block(const float *p, uint32_t (&w)[16]) {
    const uint4 a = load_item(p), b = load_item(p + 4), c = load_item(p + 8), d = load_item(p + 12);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    w[8] = c.x; w[9] = c.y; w[10] = c.z; w[11] = c.w;
    w[12] = d.x; w[13] = d.y; w[14] = d.z; w[15] = d.w;
}
__device__ __forceinline__ float block_absmax(const uint32_t (&w)[16], float *) {
    uint32_t m = 0;
#pragma unroll
    for (int k = 0; k < 16; ++k) m = max(m, w[k] & 0x7fffffffu);
    return __uint_as_float(m);
}
__device__ __forceinline__ uint64_t pair_f32(const uint32_t (&w)[16], int k, float *) {
    return static_cast<uint64_t>(w[2 * k]) | (static_cast<uint64_t>(w[2 * k + 1]) << 32);
}

// (lo, hi) * (r, r), each lane rounded to nearest even.
__device__ __forceinline__ uint64_t mul_pair(uint64_t v, uint64_t rr) {
    uint64_t o;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(o) : "l"(v), "l"(rr));
    return o;
}

// four code bytes from four packed (lo, hi) pairs: pair k -> byte k, lo in
// the low nibble, hi in the high nibble
__device__ __forceinline__ uint32_t e2m1_x8(uint64_t p0, uint64_t p1, uint64_t p2, uint64_t p3) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(__uint_as_float(static_cast<uint32_t>(p0))), "f"(__uint_as_float(static_cast<uint32_t>(p0 >> 32))),
          "f"(__uint_as_float(static_cast<uint32_t>(p1))), "f"(__uint_as_float(static_cast<uint32_t>(p1 >> 32))),
          "f"(__uint_as_float(static_cast<uint32_t>(p2))), "f"(__uint_as_float(static_cast<uint32_t>(p2 >> 32))),
          "f"(__uint_as_float(static_cast<uint32_t>(p3))), "f"(__uint_as_float(static_cast<uint32_t>(p3 >> 32))));
    return out;
}

// E4M3 scale byte of one block: s = RNE_E4M3(fl32(bamax / six_g)).
// The quotient only feeds the E4M3 rounding, so it is first formed as
// tq = fl32(bamax * fl32(1 / six_g)), which is within 1.5 ulp of the correctly
// rounded quotient.  If rounding tq scaled by (1 - 2^-20) and by (1 + 2^-20)
// gives the same E4M3 byte, no E4M3 rounding boundary (and no tie) lies within
// that interval, which contains the exact quotient's rounding, so the byte is
// the one the correctly rounded division would give.  Otherwise (a boundary
// is near, probability about 3e-5) the division is done exactly.
__device__ __forceinline__ uint32_t block_scale_byte(float bamax, float six_g, float inv6g,
                                                     bool exact_only) {
    if (!exact_only) {
        const float tq = __fmul_rn(bamax, inv6g);
        const uint32_t lo = e4m3_of(__fmul_rn(tq, 0.99999904632568359375f));   // 1 - 2^-20
        const uint32_t hi = e4m3_of(__fmul_rn(tq, 1.00000095367431640625f));   // 1 + 2^-20
        if (lo == hi) return lo;
    }
    return e4m3_of(six_g > 0.0f ? __fdiv_rn(bamax, six_g) : 0.0f);
}

// Codes of one block: 8 bytes, element 2k in the low nibble of byte k.
template <typename T, int W>
__device__ __forceinline__ uint2 block_codes(const uint32_t (&v)[W], float rcp) {
    const uint64_t rr = static_cast<uint64_t>(__float_as_uint(rcp)) * 0x100000001ull;
    T *tag = nullptr;
    const uint32_t lo = e2m1_x8(mul_pair(pair_f32(v, 0, tag), rr), mul_pair(pair_f32(v, 1, tag), rr),
                                mul_pair(pair_f32(v, 2, tag), rr), mul_pair(pair_f32(v, 3, tag), rr));
    const uint32_t hi = e2m1_x8(mul_pair(pair_f32(v, 4, tag), rr), mul_pair(pair_f32(v, 5, tag), rr),
                                mul_pair(pair_f32(v, 6, tag), rr), mul_pair(pair_f32(v, 7, tag), rr));
    // rcp == 0 marks a zero-scale block: all of its codes are 0
    return rcp == 0.0f ? make_uint2(0u, 0u) : make_uint2(lo, hi);
}

template <typename T>
__global__ void __launch_bounds__(256) encode_kernel(const T *__restrict__ x, int64_t rows,
                                                     int64_t cols, int64_t ld,
                                                     const float *__restrict__ partials,
                                                     int num_partials, uint8_t *__restrict__ codes,
                                                     uint8_t *__restrict__ scales,
                                                     float *__restrict__ g_out) {
    constexpr int W = sizeof(T) == 2 ? 8 : 16;        // 32-bit words per block
    const int64_t bpr = cols / kBlock;                  // blocks per row
    const int64_t total = rows * bpr;
    const int64_t kb4 = kb4_of(cols);
    const int64_t S = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int lane = threadIdx.x & 31;
    const bool word_scales = (cols % 64) == 0;

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");   // let the GEMM queue up
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const float amax = reduce_partials(partials, num_partials);
    const float g = __fdiv_rn(amax, kTensorScaleDiv);
    const float six_g = __fmul_rn(6.0f, g);
    if (blockIdx.x == 0 && threadIdx.x == 0) *g_out = g;
    // Reciprocal of every possible block scale: fl32(1 / fl32(dec(s) * g)),
    // 0 marking a zero-scale block (d == 0 or 1/d overflows).
    __shared__ float rcp_table[128];
    if (threadIdx.x < 128) {
        const float d = __fmul_rn(e4m3_value(threadIdx.x), g);
        const float r = __frcp_rn(d);
        rcp_table[threadIdx.x] = (d == 0.0f || isinf(r)) ? 0.0f : r;
    }
    const float inv6g = __frcp_rn(six_g);
    const bool exact_only = !(six_g > 0.0f) || isinf(inv6g);
    __syncthreads();

    constexpr int U = 2;
    const bool flat32 = (ld == cols) && total < (int64_t(1) << 31) &&
                        round_up(rows, 128) * kb4 < (int64_t(1) << 31);
    if (flat32) {
        // contiguous tensor: block b at element 16 b, codes at byte 8 b;
        // (row, block-in-row) tracked incrementally in 32 bits
        const uint32_t total32 = static_cast<uint32_t>(total), S32 = static_cast<uint32_t>(S);
        const uint32_t bpr32 = static_cast<uint32_t>(bpr), kb4q = static_cast<uint32_t>(kb4 >> 2);
        const uint32_t dr = S32 / bpr32, dj = S32 - dr * bpr32;
        uint32_t r = static_cast<uint32_t>(t) / bpr32, kb = static_cast<uint32_t>(t) - r * bpr32;
        for (uint32_t b0 = static_cast<uint32_t>(t); b0 < total32; b0 += U * S32) {
            uint32_t v[U][W];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint32_t b = b0 + u * S32;
                if (b < total32) {
                    load_block(x + static_cast<size_t>(b) * kBlock, v[u]);
                } else {
#pragma unroll
                    for (int k = 0; k < W; ++k) v[u][k] = 0u;
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint32_t b = b0 + u * S32;
                const float bamax = block_absmax(v[u], static_cast<T *>(nullptr));
                const uint32_t sb = block_scale_byte(bamax, six_g, inv6g, exact_only);
                const uint2 cw = block_codes<T, W>(v[u], rcp_table[sb]);
                uint32_t word = sb;
                word |= __shfl_down_sync(0xffffffffu, sb, 1) << 8;
                word |= __shfl_down_sync(0xffffffffu, sb, 2) << 16;
                word |= __shfl_down_sync(0xffffffffu, sb, 3) << 24;
                if (b < total32) {
                    *reinterpret_cast<uint2 *>(codes + static_cast<size_t>(b) * 8) = cw;
                    const uint32_t off = ((r >> 7) * kb4q + (kb >> 2)) * 512u + (r & 31u) * 16u +
                                         ((r >> 5) & 3u) * 4u + (kb & 3u);
                    if (word_scales) {
                        if ((lane & 3) == 0) *reinterpret_cast<uint32_t *>(scales + off) = word;
                    } else {
                        scales[off] = static_cast<uint8_t>(sb);
                    }
                }
                r += dr;
                kb += dj;
                if (kb >= bpr32) { kb -= bpr32; ++r; }
            }
        }
    } else {
        const int64_t nwin = ceil_div(total, S);
        const int64_t dr = S / bpr, dj = S - dr * bpr;
        ItemCursor c;
        c.set(t, bpr);
        for (int64_t w = 0; w < nwin; ++w) {
            uint32_t v[W];
            const bool valid = w * S + t < total;
            if (valid) {
                load_block(x + c.r * ld + c.j * kBlock, v);
            } else {
#pragma unroll
                for (int k = 0; k < W; ++k) v[k] = 0u;
            }
            const float bamax = block_absmax(v, static_cast<T *>(nullptr));
            const uint32_t sb = block_scale_byte(bamax, six_g, inv6g, exact_only);
            const uint2 cw = block_codes<T, W>(v, rcp_table[sb]);
            uint32_t word = sb;
            word |= __shfl_down_sync(0xffffffffu, sb, 1) << 8;
            word |= __shfl_down_sync(0xffffffffu, sb, 2) << 16;
            word |= __shfl_down_sync(0xffffffffu, sb, 3) << 24;
            if (valid) {
                *reinterpret_cast<uint2 *>(codes + c.r * (cols / 2) + c.j * 8) = cw;
                if (word_scales) {
                    if ((lane & 3) == 0)
                        *reinterpret_cast<uint32_t *>(scales + scale_offset(c.r, c.j, kb4)) = word;
                } else {
                    scales[scale_offset(c.r, c.j, kb4)] = static_cast<uint8_t>(sb);
                }
            }
            c.advance(dr, dj, bpr);
        }
    }

    // Zero the padding of the scale layout: blocks kb in [cols/16, kb4) of
    // real rows, and every block of rows in [rows, roundup(rows, 128)).
    const int64_t pad_a = rows * (kb4 - bpr);
    const int64_t r128 = round_up(rows, 128);
    const int64_t pad_b_words = (r128 - rows) * (kb4 / 4);
    for (int64_t i = t; i < pad_a; i += S) {
        const int64_t r = i / (kb4 - bpr), q = bpr + (i - r * (kb4 - bpr));
        scales[scale_offset(r, q, kb4)] = 0;
    }
    for (int64_t i = t; i < pad_b_words; i += S) {
        const int64_t r = rows + i / (kb4 / 4), q = 4 * (i % (kb4 / 4));
        *reinterpret_cast<uint32_t *>(scales + scale_offset(r, q, kb4)) = 0u;
    }
}

// ---------------------------------------------------------------------------
// Dequantize: y = fl32(fl32(e * dec(s)) * g), eight values per thread.
// ---------------------------------------------------------------------------
template <typename OutT>
__global__ void __launch_bounds__(256) dequantize_kernel(const uint8_t *__restrict__ codes,
                                                         const uint8_t *__restrict__ scales,
                                                         const float *__restrict__ g_ptr,
                                                         int64_t rows, int64_t cols,
                                                         OutT *__restrict__ y, int64_t ldy) {
    const int64_t ipr = cols / 8;
    const int64_t total = rows * ipr;
    const int64_t kb4 = kb4_of(cols);
    const float g = *g_ptr;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t r = i / ipr, j = i - r * ipr;
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t *>(codes + r * (cols / 2) + j * 4));
        const float s = e4m3_value(__ldg(scales + scale_offset(r, j / 2, kb4)));
        uint32_t h[4];
        asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
            "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
            "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
            "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
            "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
            "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
            : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
            : "r"(w));
        float out[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float e0 = __half2float(__ushort_as_half(static_cast<unsigned short>(h[k] & 0xffffu)));
            const float e1 = __half2float(__ushort_as_half(static_cast<unsigned short>(h[k] >> 16)));
            out[2 * k] = __fmul_rn(__fmul_rn(e0, s), g);
            out[2 * k + 1] = __fmul_rn(__fmul_rn(e1, s), g);
        }
        OutT *dst = y + r * ldy + j * 8;
        if constexpr (sizeof(OutT) == 2) {
            uint4 pk;
            uint32_t *p = reinterpret_cast<uint32_t *>(&pk);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                __nv_bfloat162 b2 = __floats2bfloat162_rn(out[2 * k], out[2 * k + 1]);
                p[k] = *reinterpret_cast<uint32_t *>(&b2);
            }
            *reinterpret_cast<uint4 *>(dst) = pk;
        } else {
            reinterpret_cast<float4 *>(dst)[0] = make_float4(out[0], out[1], out[2], out[3]);
            reinterpret_cast<float4 *>(dst)[1] = make_float4(out[4], out[5], out[6], out[7]);
        }
    }
}

// ---------------------------------------------------------------------------
// Host launchers.
// ---------------------------------------------------------------------------

int quantize_grid(int64_t rows, int64_t cols, int elem_bytes, int num_sms, int per_sm) {
    const int64_t items = rows * (cols * elem_bytes / 16);
    int64_t blocks = ceil_div(items, 256);
    blocks = blocks < 1 ? 1 : blocks;
    const int64_t cap = static_cast<int64_t>(num_sms) * per_sm;
    return static_cast<int>(blocks < cap ? blocks : cap);
}

// Resident 256-thread CTAs per SM of a kernel (looked up once).
template <typename K>
static int resident_ctas(K kernel) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, 256, 0) != cudaSuccess || n < 1)
        n = 1;
    return n;
}

cudaError_t launch_quantize(const void *x, bool bf16, int64_t rows, int64_t cols, int64_t ld,
                            uint8_t *codes, uint8_t *scales, float *g_out, float *partials,
                            int num_sms, cudaStream_t stream) {
    // An empty tensor has no codes and no scale bytes; its amax is 0, so g = 0.
    if (rows == 0 || cols == 0) return cudaMemsetAsync(g_out, 0, sizeof(float), stream);
    const int eb = bf16 ? 2 : 4;
    static const int occ_amax[2] = {resident_ctas(amax_partials_kernel<float>),
                                    resident_ctas(amax_partials_kernel<__nv_bfloat16>)};
    static const int occ_encode[2] = {resident_ctas(encode_kernel<float>),
                                      resident_ctas(encode_kernel<__nv_bfloat16>)};
    int g1 = quantize_grid(rows, cols, eb, num_sms, occ_amax[bf16]);
    // pass 2 runs one thread per 16-value block
    const int g2 = quantize_grid(rows, cols, 1, num_sms, occ_encode[bf16]);
    if (g1 > kMaxAmaxPartials) g1 = kMaxAmaxPartials;
    if (bf16)
        amax_partials_kernel<__nv_bfloat16><<<g1, 256, 0, stream>>>(
            static_cast<const __nv_bfloat16 *>(x), rows, cols, ld, partials);
    else
        amax_partials_kernel<float><<<g1, 256, 0, stream>>>(static_cast<const float *>(x), rows,
                                                             cols, ld, partials);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(g2);
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (bf16)
        return cudaLaunchKernelEx(&cfg, encode_kernel<__nv_bfloat16>,
                                  static_cast<const __nv_bfloat16 *>(x), rows, cols, ld,
                                  static_cast<const float *>(partials), g1, codes, scales, g_out);
    return cudaLaunchKernelEx(&cfg, encode_kernel<float>, static_cast<const float *>(x), rows,
                              cols, ld, static_cast<const float *>(partials), g1, codes, scales,
                              g_out);
}

cudaError_t launch_encode_f32(const float *x, int64_t rows, int64_t cols, int64_t ld, const float *partials,
                              int num_partials, uint8_t *codes, uint8_t *scales, float *g_out, int num_sms,
                              cudaStream_t stream) {
    static const int occ_encode = resident_ctas(encode_kernel<float>);
    const int g2 = quantize_grid(rows, cols, 1, num_sms, occ_encode);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(g2);
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, encode_kernel<float>, x, rows, cols, ld, partials, num_partials, codes,
                              scales, g_out);
}

cudaError_t launch_dequantize(const uint8_t *codes, const uint8_t *scales, const float *g,
                              int64_t rows, int64_t cols, void *y, bool bf16, int64_t ldy,
                              int num_sms, cudaStream_t stream) {
    const int64_t items = rows * (cols / 8);
    int64_t blocks = ceil_div(items, 256);
    const int64_t cap = static_cast<int64_t>(num_sms) * 8;
    blocks = blocks < 1 ? 1 : (blocks < cap ? blocks : cap);
    if (bf16)
        dequantize_kernel<__nv_bfloat16><<<static_cast<int>(blocks), 256, 0, stream>>>(
            codes, scales, g, rows, cols, static_cast<__nv_bfloat16 *>(y), ldy);
    else
        dequantize_kernel<float><<<static_cast<int>(blocks), 256, 0, stream>>>(
            codes, scales, g, rows, cols, static_cast<float *>(y), ldy);
    return cudaGetLastError();
}

}  // namespace nvfp4
