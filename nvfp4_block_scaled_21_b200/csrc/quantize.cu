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
//   the windows in the reverse order of pass 1 so that the tail pass 1 read
//   last is still in L2.  A 16-element block is held by 2 (bf16) or 4 (fp32)
//   adjacent lanes; its amax is one or two shuffles; the E4M3 scale and the
//   E2M1 codes come from the hardware RNE-satfinite conversions; codes go out
//   as coalesced 32-bit (bf16) or 16-bit (fp32) stores and scales as one
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
    const int64_t ipr = cols / EPI;
    const int64_t total = rows * ipr;
    const int64_t S = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t dr = S / ipr, dj = S - dr * ipr;
    float m = 0.0f;
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
    // Let a dependent launch (the encode pass) start its prologue.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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

// Four bytes of packed E2M1 codes from eight values: element 2k in the low
// nibble of byte k, element 2k+1 in the high nibble.
__device__ __forceinline__ uint32_t e2m1x8(const float (&v)[8]) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return out;
}
__device__ __forceinline__ uint32_t e2m1x4(const float (&v)[4]) {
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1;\n\t.reg .b16 h;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "mov.b16 h, {b0, b1};\n\t"
        "cvt.u32.u16 %0, h;\n\t}"
        : "=r"(out)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]));
    return out;
}

__device__ __forceinline__ void unpack(const uint4 &v, float (&x)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        x[2 * k] = __uint_as_float(w[k] << 16);
        x[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
}
__device__ __forceinline__ void unpack(const uint4 &v, float (&x)[4]) {
    x[0] = __uint_as_float(v.x);
    x[1] = __uint_as_float(v.y);
    x[2] = __uint_as_float(v.z);
    x[3] = __uint_as_float(v.w);
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
// Pass 2: encode.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) encode_kernel(const T *__restrict__ x, int64_t rows,
                                                     int64_t cols, int64_t ld,
                                                     const float *__restrict__ partials,
                                                     int num_partials, uint8_t *__restrict__ codes,
                                                     uint8_t *__restrict__ scales,
                                                     float *__restrict__ g_out) {
    constexpr int EPI = Elem<T>::kPerItem;      // values per item
    constexpr int IPB = kBlock / EPI;           // items (lanes) per 16-value block
    constexpr int GROUP = 4 * IPB;              // lanes per 32-bit scale word
    const int64_t ipr = cols / EPI;
    const int64_t total = rows * ipr;
    const int64_t kb4 = kb4_of(cols);
    const int64_t S = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int lane = threadIdx.x & 31;
    const bool word_scales = (cols % 64) == 0;

    asm volatile("griddepcontrol.wait;" ::: "memory");
    const float amax = reduce_partials(partials, num_partials);
    const float g = __fdiv_rn(amax, kTensorScaleDiv);
    const float six_g = __fmul_rn(6.0f, g);
    if (blockIdx.x == 0 && threadIdx.x == 0) *g_out = g;

    const int64_t nwin = ceil_div(total, S);
    const int64_t dr = S / ipr, dj = S - dr * ipr;
    ItemCursor c;
    c.set((nwin - 1) * S + t, ipr);
    constexpr int U = 2;
    for (int64_t w = nwin - 1; w >= 0; w -= U) {
        uint4 v[U];
        ItemCursor cu[U];
        bool valid[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            cu[u] = c;
            const int64_t i = (w - u) * S + t;
            valid[u] = (w - u) >= 0 && i < total;
            v[u] = valid[u] ? load_item(x + c.r * ld + c.j * EPI) : make_uint4(0, 0, 0, 0);
            c.retreat(dr, dj, ipr);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float bamax = item_absmax(v[u], static_cast<T *>(nullptr));
#pragma unroll
            for (int o = 1; o < IPB; o <<= 1) bamax = fmaxf(bamax, __shfl_xor_sync(0xffffffffu, bamax, o));
            const float tb = g > 0.0f ? __fdiv_rn(bamax, six_g) : 0.0f;
            const uint32_t s = e4m3_of(tb);
            const float d = __fmul_rn(e4m3_value(s), g);
            const float rcp = __frcp_rn(d);
            const bool zero_block = (d == 0.0f) || isinf(rcp);
            float xv[EPI];
            unpack(v[u], xv);
#pragma unroll
            for (int k = 0; k < EPI; ++k) xv[k] = __fmul_rn(xv[k], rcp);
            uint32_t packed = (EPI == 8) ? e2m1x8(reinterpret_cast<float(&)[8]>(xv))
                                         : e2m1x4(reinterpret_cast<float(&)[4]>(xv));
            if (zero_block) packed = 0;
            // gather the four block scales of a 64-column group into one word
            uint32_t word = s;
            word |= __shfl_down_sync(0xffffffffu, s, IPB) << 8;
            word |= __shfl_down_sync(0xffffffffu, s, 2 * IPB) << 16;
            word |= __shfl_down_sync(0xffffffffu, s, 3 * IPB) << 24;
            if (valid[u]) {
                const int64_t r = cu[u].r, j = cu[u].j;
                if (EPI == 8)
                    *reinterpret_cast<uint32_t *>(codes + r * (cols / 2) + j * 4) = packed;
                else
                    *reinterpret_cast<uint16_t *>(codes + r * (cols / 2) + j * 2) =
                        static_cast<uint16_t>(packed);
                const int64_t kb = j / IPB;
                if (word_scales) {
                    if ((lane % GROUP) == 0)
                        *reinterpret_cast<uint32_t *>(scales + scale_offset(r, kb, kb4)) = word;
                } else if ((lane % IPB) == 0) {
                    scales[scale_offset(r, kb, kb4)] = static_cast<uint8_t>(s);
                }
            }
        }
    }

    // Zero the padding of the scale layout: blocks kb in [cols/16, kb4) of
    // real rows, and every block of rows in [rows, roundup(rows, 128)).
    const int64_t kb = cols / kBlock;
    const int64_t pad_a = rows * (kb4 - kb);
    const int64_t r128 = round_up(rows, 128);
    const int64_t pad_b_words = (r128 - rows) * (kb4 / 4);
    for (int64_t i = t; i < pad_a; i += S) {
        const int64_t r = i / (kb4 - kb), q = kb + (i - r * (kb4 - kb));
        scales[scale_offset(r, q, kb4)] = 0;
    }
    for (int64_t i = t; i < pad_b_words; i += S) {
        const int64_t r = rows + i / (kb4 / 4), q = 4 * (i % (kb4 / 4));
        *reinterpret_cast<uint32_t *>(scales + scale_offset(r, q, kb4)) = 0u;
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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

cudaError_t launch_quantize(const void *x, bool bf16, int64_t rows, int64_t cols, int64_t ld,
                            uint8_t *codes, uint8_t *scales, float *g_out, float *partials,
                            int num_sms, cudaStream_t stream) {
    const int eb = bf16 ? 2 : 4;
    int g1 = quantize_grid(rows, cols, eb, num_sms, 4);
    int g2 = quantize_grid(rows, cols, eb, num_sms, 8);
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
