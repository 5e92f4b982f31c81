// encode.cuh -- the arithmetic of NVFP4 encoding shared by the quantizer's
// encode pass and the decode GEMM that quantizes its activations itself:
// |x| maxima on bit patterns, the E4M3 block scale, the E2M1 codes.
// Format: NVFP4 wiki page (newton.com.tw), section "技術原理".
#pragma once

#include "common.cuh"

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

// Reciprocal of a decoded block scale, fl32(1 / fl32(dec(s) * g)); 0 marks a
// zero-scale block (d == 0, or 1/d overflows), whose codes are all 0.
__device__ __forceinline__ float block_rcp(uint32_t s, float g) {
    const float d = __fmul_rn(e4m3_value(s), g);
    const float r = __frcp_rn(d);
    return (d == 0.0f || isinf(r)) ? 0.0f : r;
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

}  // namespace nvfp4
