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
#include <atomic>
#include <cstdlib>
#include "common.cuh"
#include "encode.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace nvfp4 {

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
    // Launched as a programmatic dependent of the previous kernel in the
    // stream (which may have written x or still read the partials): resident
    // early, it starts work the moment that kernel completes.
    asm volatile("griddepcontrol.wait;" ::: "memory");
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
// Pass 2 helpers.
// ---------------------------------------------------------------------------

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
// Zero the padding of the tiled scale layout: blocks kb in [bpr, kb4) of the
// real rows (bytes) and every block of the rows [rows, roundup(rows, 128))
// (32-bit words), as thread tid of nthr.  Each thread divides once and then
// steps its (row, column) position incrementally.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void zero_scale_padding(uint8_t *scales, int64_t rows, int64_t bpr, int64_t kb4,
                                                   int64_t tid, int64_t nthr, size_t scales_bytes,
                                                   uint32_t *status) {
    const int64_t npad = kb4 - bpr;                     // padded blocks per real row (0..3)
    if (npad > 0) {
        const int64_t total = rows * npad;
        int64_t r = tid / npad, q = tid - r * npad;
        const int64_t dr = nthr / npad, dq = nthr - dr * npad;
        for (int64_t i = tid; i < total; i += nthr) {
            uint8_t *sp = scales + scale_offset(r, bpr + q, kb4);
            if (store_ok(sp, 1, scales, scales_bytes, status)) *sp = 0;
            r += dr;
            q += dq;
            if (q >= npad) { q -= npad; ++r; }
        }
    }
    const int64_t wpr = kb4 / 4;                        // scale words per row
    const int64_t total_w = (round_up(rows, 128) - rows) * wpr;
    if (total_w > 0) {
        int64_t r = rows + tid / wpr, q = tid % wpr;
        const int64_t dr = nthr / wpr, dq = nthr % wpr;
        for (int64_t i = tid; i < total_w; i += nthr) {
            uint8_t *sp = scales + ((r >> 7) * wpr + q) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4;
            if (store_ok(sp, 4, scales, scales_bytes, status)) *reinterpret_cast<uint32_t *>(sp) = 0u;
            r += dr;
            q += dq;
            if (q >= wpr) { q -= wpr; ++r; }
        }
    }
}

// ---------------------------------------------------------------------------
// Pass 2: encode.  One thread owns one 16-value block: its amax needs no
// shuffle, the scale arithmetic runs once per block, the 16 products are 8
// packed f32x2 multiplies (per-lane IEEE round-to-nearest, identical to 16
// scalar ones), and the 8 code bytes leave as one 8-byte store.  Four
// neighbouring lanes hold the four blocks of a 64-column group; their scale
// bytes are gathered into one 32-bit word in the tiled layout.
// ---------------------------------------------------------------------------

template <typename T>
__global__ void __launch_bounds__(256) encode_kernel(const T *__restrict__ x, int64_t rows,
                                                     int64_t cols, int64_t ld,
                                                     const float *__restrict__ partials,
                                                     int num_partials, uint8_t *__restrict__ codes,
                                                     uint8_t *__restrict__ scales,
                                                     float *__restrict__ g_out, uint32_t *status) {
    constexpr int W = sizeof(T) == 2 ? 8 : 16;        // 32-bit words per block
    const int64_t bpr = cols / kBlock;                  // blocks per row
    const int64_t total = rows * bpr;
    const int64_t kb4 = kb4_of(cols);
    const int64_t S = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int lane = threadIdx.x & 31;
    const bool word_scales = (cols % 64) == 0;
    const size_t codes_bytes = static_cast<size_t>(rows * cols / 2);           // debug-build store checks
    const size_t scales_bytes = static_cast<size_t>(round_up(rows, 128) * kb4);

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
        // The trip count is the warp's first lane's, so that every lane of
        // the warp runs the full-mask shuffles below; lanes whose block lies
        // past the end load nothing and store nothing.
        const uint32_t t0 = static_cast<uint32_t>(t) - static_cast<uint32_t>(lane);
        const uint32_t nstr = t0 < total32 ? (total32 - 1u - t0) / S32 + 1u : 0u;
        for (uint32_t s0 = 0; s0 < nstr; s0 += U) {
            const uint32_t b0 = static_cast<uint32_t>(t) + s0 * S32;
            uint32_t v[U][W];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint32_t b = b0 + u * S32;
                if (s0 + u < nstr && b < total32) {
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
                if (s0 + u < nstr && b < total32) {
                    uint8_t *cp = codes + static_cast<size_t>(b) * 8;
                    if (store_ok(cp, 8, codes, codes_bytes, status)) *reinterpret_cast<uint2 *>(cp) = cw;
                    const uint32_t off = ((r >> 7) * kb4q + (kb >> 2)) * 512u + (r & 31u) * 16u +
                                         ((r >> 5) & 3u) * 4u + (kb & 3u);
                    if (word_scales) {
                        if ((lane & 3) == 0 && store_ok(scales + off, 4, scales, scales_bytes, status))
                            *reinterpret_cast<uint32_t *>(scales + off) = word;
                    } else if (store_ok(scales + off, 1, scales, scales_bytes, status)) {
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
                uint8_t *cp = codes + c.r * (cols / 2) + c.j * 8;
                if (store_ok(cp, 8, codes, codes_bytes, status)) *reinterpret_cast<uint2 *>(cp) = cw;
                uint8_t *sp = scales + scale_offset(c.r, c.j, kb4);
                if (word_scales) {
                    if ((lane & 3) == 0 && store_ok(sp, 4, scales, scales_bytes, status))
                        *reinterpret_cast<uint32_t *>(sp) = word;
                } else if (store_ok(sp, 1, scales, scales_bytes, status)) {
                    *sp = static_cast<uint8_t>(sb);
                }
            }
            c.advance(dr, dj, bpr);
        }
    }

    zero_scale_padding(scales, rows, bpr, kb4, t, S, scales_bytes, status);
}

// ---------------------------------------------------------------------------
// Small tensors (at most kMeetMaxCtas * 256 blocks of 16, e.g. the few
// activation rows of a decode step): both passes in one cooperative launch
// of a few CTAs.  Each thread holds one block in registers; each CTA
// publishes its max |x|, the CTAs meet once (grid_meet), and every thread
// encodes its block with the same arithmetic as encode_kernel.  One launch
// instead of two dependent ones, and x is read once.
// ---------------------------------------------------------------------------
constexpr int kMeetThreads = 256;
constexpr int kMeetMaxCtas = 32;

template <typename T>
__global__ void __launch_bounds__(kMeetThreads) quantize_meet_kernel(
        const T *__restrict__ x, int64_t rows, int64_t cols, int64_t ld, uint8_t *__restrict__ codes,
        uint8_t *__restrict__ scales, float *__restrict__ g_out, float *partials, uint32_t *grid_bar,
        uint32_t *status, uint64_t timeout_ns) {
    constexpr int W = sizeof(T) == 2 ? 8 : 16;          // 32-bit words per block
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int bpr = static_cast<int>(cols / kBlock);
    const int total = static_cast<int>(rows) * bpr;
    const int b = static_cast<int>(blockIdx.x) * kMeetThreads + t;
    const int64_t kb4 = kb4_of(cols);
    const bool word_scales = (cols % 64) == 0;
    const size_t codes_bytes = static_cast<size_t>(rows * cols / 2);           // debug-build store checks
    const size_t scales_bytes = static_cast<size_t>(round_up(rows, 128) * kb4);
    __shared__ float wmax[kMeetThreads / 32];
    __shared__ float s_amax;
    __shared__ uint32_t s_go;
    __shared__ float rcp_table[128];
    __shared__ uint32_t abort_word;
    volatile uint32_t *abort_flag = &abort_word;
    if (t == 0) abort_word = 0u;
    // x may be the previous kernel's output, and that kernel may still read
    // the codes this one writes
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // the meeting point's generation, read early (see grid_meet_generation)
    const uint32_t meet_gen = threadIdx.x == 0 ? grid_meet_generation(grid_bar) : 0u;

    uint32_t v[W];
    int r = 0, kb = 0;
    if (b < total) {
        r = b / bpr;
        kb = b - r * bpr;
        load_block(x + static_cast<int64_t>(r) * ld + static_cast<int64_t>(kb) * kBlock, v);
    } else {
#pragma unroll
        for (int i = 0; i < W; ++i) v[i] = 0u;
    }
    float m = block_absmax(v, static_cast<T *>(nullptr));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) wmax[warp] = m;
    __syncthreads();
    // x is in registers: the next kernel (the GEMM) may launch and start
    // streaming its weights (earlier, that stream would queue ahead of x)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (warp == 0) {
        uint32_t go = 0u;
        if (lane == 0) {
            float cm = 0.0f;
            for (int k = 0; k < kMeetThreads / 32; ++k) cm = fmaxf(cm, wmax[k]);
            partials[blockIdx.x] = cm;
            // every CTA of the cooperative launch is resident and arrives
            // exactly once; bounded
            go = grid_meet(grid_bar, meet_gen, timeout_ns, abort_flag, status) ? 1u : 0u;
        }
        go = __shfl_sync(0xffffffffu, go, 0);
        float gm = 0.0f;
        if (go)
            for (int k = lane; k < static_cast<int>(gridDim.x); k += 32) gm = fmaxf(gm, __ldcg(partials + k));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, o));
        if (lane == 0) {
            s_amax = gm;
            s_go = go;
        }
    }
    __syncthreads();
    if (!s_go) return;
    const float g = __fdiv_rn(s_amax, kTensorScaleDiv);
    const float six_g = __fmul_rn(6.0f, g);
    const float inv6g = __frcp_rn(six_g);
    const bool exact_only = !(six_g > 0.0f) || isinf(inv6g);
    if (blockIdx.x == 0 && t == 0) *g_out = g;
    if (t < 128) rcp_table[t] = block_rcp(static_cast<uint32_t>(t), g);
    __syncthreads();

    // the 4 blocks of a scale word sit in 4 neighbouring lanes (b % 4 == lane % 4)
    const uint32_t sb = block_scale_byte(block_absmax(v, static_cast<T *>(nullptr)), six_g, inv6g, exact_only);
    const uint2 cw = block_codes<T, W>(v, rcp_table[sb]);
    uint32_t word = sb;
    word |= __shfl_down_sync(0xffffffffu, sb, 1) << 8;
    word |= __shfl_down_sync(0xffffffffu, sb, 2) << 16;
    word |= __shfl_down_sync(0xffffffffu, sb, 3) << 24;
    if (b < total) {
        uint8_t *cp = codes + static_cast<int64_t>(r) * (cols / 2) + kb * 8;
        if (store_ok(cp, 8, codes, codes_bytes, status)) *reinterpret_cast<uint2 *>(cp) = cw;
        uint8_t *sp = scales + scale_offset(r, kb, kb4);
        if (word_scales) {
            if ((lane & 3) == 0 && store_ok(sp, 4, scales, scales_bytes, status))
                *reinterpret_cast<uint32_t *>(sp) = word;
        } else if (store_ok(sp, 1, scales, scales_bytes, status)) {
            *sp = static_cast<uint8_t>(sb);
        }
    }
    zero_scale_padding(scales, rows, bpr, kb4, b, static_cast<int64_t>(gridDim.x) * kMeetThreads, scales_bytes,
                       status);
}

template <typename T>
static cudaError_t launch_meet_t(const T *x, int64_t rows, int64_t cols, int64_t ld, uint8_t *codes, uint8_t *scales,
                                 float *g_out, float *partials, uint32_t *grid_bar, uint32_t *status,
                                 uint64_t timeout_ns, int grid, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kMeetThreads);
    cfg.stream = stream;
    // cooperative (the CTAs meet once), and a programmatic dependent of the
    // kernel before it if the driver takes both; cooperative alone otherwise
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    static std::atomic<int> coop_pdl{1};
    if (coop_pdl.load()) {
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        const cudaError_t e = cudaLaunchKernelEx(&cfg, quantize_meet_kernel<T>, x, rows, cols, ld, codes, scales,
                                                 g_out, partials, grid_bar, status, timeout_ns);
        if (e == cudaSuccess) return e;
        if (e != cudaErrorInvalidValue && e != cudaErrorNotSupported) return e;
        (void)cudaGetLastError();      // a refused configuration, not a failed launch
        coop_pdl.store(0);
    }
    cfg.attrs = attr + 1;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, quantize_meet_kernel<T>, x, rows, cols, ld, codes, scales, g_out, partials,
                              grid_bar, status, timeout_ns);
}

// ---------------------------------------------------------------------------
// Dequantize: y = fl32(fl32(e * dec(s)) * g), eight values per thread.
// ---------------------------------------------------------------------------
template <typename OutT>
__global__ void __launch_bounds__(256) dequantize_kernel(const uint8_t *__restrict__ codes,
                                                         const uint8_t *__restrict__ scales,
                                                         const float *__restrict__ g_ptr,
                                                         int64_t rows, int64_t cols,
                                                         OutT *__restrict__ y, int64_t ldy, uint32_t *status) {
    const int64_t ipr = cols / 8;
    const size_t y_bytes = matrix_extent(rows, cols, ldy, sizeof(OutT));       // debug-build store checks
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
        if (!store_ok(dst, 8 * sizeof(OutT), y, y_bytes, status)) continue;
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
                            int num_sms, cudaStream_t stream, uint32_t *grid_bar, uint32_t *status,
                            uint64_t timeout_ns) {
    // An empty tensor has no codes and no scale bytes; its amax is 0, so g = 0.
    if (rows == 0 || cols == 0) return cudaMemsetAsync(g_out, 0, sizeof(float), stream);
    // Small tensors: one cooperative launch of a few CTAs (NVFP4_QUANTIZE_MEET=0:
    // the two passes).
    const char *meet_opt = getenv("NVFP4_QUANTIZE_MEET");
    const int64_t nblocks = rows * (cols / kBlock);
    if (grid_bar != nullptr && status != nullptr && (meet_opt == nullptr || meet_opt[0] != '0') &&
        nblocks <= int64_t(kMeetMaxCtas) * kMeetThreads) {
        const int grid = static_cast<int>(ceil_div(nblocks, kMeetThreads));
        return bf16 ? launch_meet_t(static_cast<const __nv_bfloat16 *>(x), rows, cols, ld, codes, scales, g_out,
                                    partials, grid_bar, status, timeout_ns, grid, stream)
                    : launch_meet_t(static_cast<const float *>(x), rows, cols, ld, codes, scales, g_out, partials,
                                    grid_bar, status, timeout_ns, grid, stream);
    }
    // Large contiguous tensors: one cooperative pass that reads x once.
    if (grid_bar != nullptr && status != nullptr && quantize_onepass_usable(rows, cols, ld, bf16)) {
        const cudaError_t e = launch_quantize_onepass(x, bf16, rows, cols, codes, scales, g_out, partials, grid_bar,
                                                      status, timeout_ns, num_sms, stream);
        if (e != cudaErrorCooperativeLaunchTooLarge) return e;
        (void)cudaGetLastError();      // fewer SMs than the grid (a shared device): the two passes
    }
    const int eb = bf16 ? 2 : 4;
    static const int occ_amax[2] = {resident_ctas(amax_partials_kernel<float>),
                                    resident_ctas(amax_partials_kernel<__nv_bfloat16>)};
    static const int occ_encode[2] = {resident_ctas(encode_kernel<float>),
                                      resident_ctas(encode_kernel<__nv_bfloat16>)};
    int g1 = quantize_grid(rows, cols, eb, num_sms, occ_amax[bf16]);
    // pass 2 runs one thread per 16-value block
    const int g2 = quantize_grid(rows, cols, 1, num_sms, occ_encode[bf16]);
    if (g1 > kMaxAmaxPartials) g1 = kMaxAmaxPartials;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg1 = {};
    cfg1.gridDim = dim3(g1);
    cfg1.blockDim = dim3(256);
    cfg1.stream = stream;
    cfg1.attrs = attr;
    cfg1.numAttrs = 1;
    cudaError_t e = bf16 ? cudaLaunchKernelEx(&cfg1, amax_partials_kernel<__nv_bfloat16>,
                                              static_cast<const __nv_bfloat16 *>(x), rows, cols, ld, partials)
                         : cudaLaunchKernelEx(&cfg1, amax_partials_kernel<float>, static_cast<const float *>(x), rows,
                                              cols, ld, partials);
    if (e != cudaSuccess) return e;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(g2);
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (bf16)
        return cudaLaunchKernelEx(&cfg, encode_kernel<__nv_bfloat16>,
                                  static_cast<const __nv_bfloat16 *>(x), rows, cols, ld,
                                  static_cast<const float *>(partials), g1, codes, scales, g_out, status);
    return cudaLaunchKernelEx(&cfg, encode_kernel<float>, static_cast<const float *>(x), rows,
                              cols, ld, static_cast<const float *>(partials), g1, codes, scales,
                              g_out, status);
}

// One CTA: *amax = the largest of n partial maxima (the reduction the encode
// pass starts with, as a value of its own).
__global__ void __launch_bounds__(256) reduce_amax_kernel(const float *__restrict__ partials, int n,
                                                         float *__restrict__ amax) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const float m = reduce_partials(partials, n);
    if (threadIdx.x == 0) *amax = m;
}

cudaError_t launch_amax(const void *x, bool bf16, int64_t rows, int64_t cols, int64_t ld, float *partials,
                        float *amax, int num_sms, cudaStream_t stream) {
    if (rows == 0 || cols == 0) return cudaMemsetAsync(amax, 0, sizeof(float), stream);
    const int eb = bf16 ? 2 : 4;
    static const int occ_amax[2] = {resident_ctas(amax_partials_kernel<float>),
                                    resident_ctas(amax_partials_kernel<__nv_bfloat16>)};
    int g1 = quantize_grid(rows, cols, eb, num_sms, occ_amax[bf16]);
    if (g1 > kMaxAmaxPartials) g1 = kMaxAmaxPartials;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(g1);
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = bf16 ? cudaLaunchKernelEx(&cfg, amax_partials_kernel<__nv_bfloat16>,
                                              static_cast<const __nv_bfloat16 *>(x), rows, cols, ld, partials)
                         : cudaLaunchKernelEx(&cfg, amax_partials_kernel<float>, static_cast<const float *>(x), rows,
                                              cols, ld, partials);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(1);
    return cudaLaunchKernelEx(&cfg, reduce_amax_kernel, static_cast<const float *>(partials), g1, amax);
}

cudaError_t launch_encode(const void *x, bool bf16, int64_t rows, int64_t cols, int64_t ld, const float *partials,
                          int num_partials, uint8_t *codes, uint8_t *scales, float *g_out, int num_sms,
                          cudaStream_t stream, uint32_t *status) {
    static const int occ_encode[2] = {resident_ctas(encode_kernel<float>),
                                      resident_ctas(encode_kernel<__nv_bfloat16>)};
    const int g2 = quantize_grid(rows, cols, 1, num_sms, occ_encode[bf16]);
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
        return cudaLaunchKernelEx(&cfg, encode_kernel<__nv_bfloat16>, static_cast<const __nv_bfloat16 *>(x), rows,
                                  cols, ld, partials, num_partials, codes, scales, g_out, status);
    return cudaLaunchKernelEx(&cfg, encode_kernel<float>, static_cast<const float *>(x), rows, cols, ld, partials,
                              num_partials, codes, scales, g_out, status);
}

cudaError_t launch_encode_f32(const float *x, int64_t rows, int64_t cols, int64_t ld, const float *partials,
                              int num_partials, uint8_t *codes, uint8_t *scales, float *g_out, int num_sms,
                              cudaStream_t stream, uint32_t *status) {
    return launch_encode(x, false, rows, cols, ld, partials, num_partials, codes, scales, g_out, num_sms, stream,
                         status);
}

cudaError_t launch_dequantize(const uint8_t *codes, const uint8_t *scales, const float *g,
                              int64_t rows, int64_t cols, void *y, bool bf16, int64_t ldy,
                              int num_sms, cudaStream_t stream, uint32_t *status) {
    const int64_t items = rows * (cols / 8);
    int64_t blocks = ceil_div(items, 256);
    const int64_t cap = static_cast<int64_t>(num_sms) * 8;
    blocks = blocks < 1 ? 1 : (blocks < cap ? blocks : cap);
    if (bf16)
        dequantize_kernel<__nv_bfloat16><<<static_cast<int>(blocks), 256, 0, stream>>>(
            codes, scales, g, rows, cols, static_cast<__nv_bfloat16 *>(y), ldy, status);
    else
        dequantize_kernel<float><<<static_cast<int>(blocks), 256, 0, stream>>>(
            codes, scales, g, rows, cols, static_cast<float *>(y), ldy, status);
    return cudaGetLastError();
}

}  // namespace nvfp4
