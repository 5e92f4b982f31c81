// quantize_onepass.cu -- the NVFP4 quantizer that reads x from memory once.
//
// The two-level NVFP4 scaling (NVFP4 wiki page, section "技術原理") needs the
// tensor's largest magnitude before the first block can be encoded, which is
// why the two-pass quantizer (quantize.cu) reads x twice.  Here a cooperative
// grid of one CTA per SM keeps its slice of x on chip across the one point
// where the whole grid must agree on that maximum:
//   pass A  each CTA brings its contiguous range of 16-value blocks in: the
//           first part into shared memory (bulk copies), the next part into
//           registers, and reads whatever is left once more only for its
//           maximum (with an L2 evict-last hint, so that the second read of
//           that tail finds it in L2); then the CTA's max |x| is published
//           and the CTAs meet (grid_meet);
//   pass B  every CTA takes the tensor amax from the published maxima and
//           encodes its range with the quantizer's arithmetic (encode.cuh):
//           g = amax / 2688, per block the E4M3 scale and the E2M1 codes,
//           the same bytes as the two-pass quantizer.
// With 148 SMs about 50 MB of bf16 x stay on chip, so a 4096 x 5120 bf16
// activation (42 MB) is read from DRAM once.
//
// Opt-in (quantize_onepass_usable), for contiguous x with cols % 64 == 0
// (every 4-block scale word lies in one row and one CTA) and at least 8 MB;
// otherwise the two-pass quantizer runs.
#include <atomic>
#include <cstdlib>
#include "common.cuh"
#include "encode.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace nvfp4 {

namespace {

constexpr int kOpThreads = 512;
constexpr int kOpSmemData = 200 * 1024;                   // shared memory for x, bytes
constexpr int kOpChunk = 16 * 1024;                       // bytes per bulk copy
constexpr int kSpillBatch = 4;                            // tail blocks per thread in flight

template <typename T> struct OpCfg {
    static constexpr int kBlockBytes = 16 * static_cast<int>(sizeof(T));
    static constexpr int kItems = kBlockBytes / 16;         // 16-byte items per block
    static constexpr int kWords = kBlockBytes / 4;          // 32-bit words per block
    static constexpr int kRegBlocks = sizeof(T) == 2 ? 8 : 4;   // blocks per thread in registers (16 items)
    static constexpr int kSmemBlocks = kOpSmemData / kBlockBytes;
    static_assert(kSmemBlocks % 4 == 0, "whole 4-block groups in shared memory");
};

struct OpArgs {
    const void *x;
    int64_t rows, cols;
    float *partials;          // one max |x| per CTA
    uint32_t *grid_bar;       // grid meeting point
    uint8_t *codes, *scales;
    float *g_out;
    uint32_t *status;
    uint64_t timeout_ns;
};

template <typename T>
__device__ __forceinline__ void words_of(const uint4 (&it)[OpCfg<T>::kItems], uint32_t (&w)[OpCfg<T>::kWords]) {
#pragma unroll
    for (int i = 0; i < OpCfg<T>::kItems; ++i) {
        w[4 * i] = it[i].x; w[4 * i + 1] = it[i].y; w[4 * i + 2] = it[i].z; w[4 * i + 3] = it[i].w;
    }
}

template <typename T>
__device__ __forceinline__ float items_absmax(const uint4 (&it)[OpCfg<T>::kItems]) {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < OpCfg<T>::kItems; ++i) m = fmaxf(m, item_absmax(it[i], static_cast<T *>(nullptr)));
    return m;
}

template <typename T>
__global__ void __launch_bounds__(kOpThreads, 1) quantize_onepass_kernel(const __grid_constant__ OpArgs a) {
    using C = OpCfg<T>;
    constexpr int T_ = kOpThreads;
    constexpr int IT = C::kItems, W = C::kWords, RB = C::kRegBlocks;
    extern __shared__ __align__(128) uint8_t sx[];             // C::kSmemBlocks blocks of x
    __shared__ uint64_t bar;
    __shared__ float wmax[kOpThreads / 32];
    __shared__ float s_amax;
    __shared__ uint32_t s_go;
    __shared__ float rcp_table[128];
    __shared__ uint32_t abort_word;
    volatile uint32_t *abort_flag = &abort_word;

    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int64_t bpr = a.cols / kBlock;                      // blocks per row (a multiple of 4)
    const int64_t kb4 = bpr;
    const int64_t groups = a.rows * bpr / 4;
    const int64_t g_lo = groups * blockIdx.x / gridDim.x, g_hi = groups * (blockIdx.x + 1) / gridDim.x;
    const int64_t b0 = 4 * g_lo;                               // this CTA's blocks [b0, b0 + nb)
    const int nb = static_cast<int>(4 * (g_hi - g_lo));
    const int S = min(nb, C::kSmemBlocks);                     // in shared memory
    const int R = min(nb - S, RB * T_);                        // in registers
    const int spill_lo = S + R;                                // read again in pass B
    const uint8_t *xb = static_cast<const uint8_t *>(a.x) + b0 * C::kBlockBytes;
    const size_t codes_bytes = static_cast<size_t>(a.rows * a.cols / 2);          // debug-build store checks
    const size_t scales_bytes = static_cast<size_t>(round_up(a.rows, 128) * kb4);

    if (t == 0) {
        mbar_init(&bar, 1);
        abort_word = 0u;
        fence_mbar_init();
    }
    __syncthreads();
    // x may be the output of the kernel before this one
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const uint32_t meet_gen = threadIdx.x == 0 ? grid_meet_generation(a.grid_bar) : 0u;   // read early

    // ---- pass A
    if (t == 0 && S > 0) {
        const uint32_t bytes = static_cast<uint32_t>(S) * C::kBlockBytes;
        mbar_arrive_expect_tx(&bar, bytes);
        const uint64_t pol = policy_evict_first();
        for (uint32_t off = 0; off < bytes; off += kOpChunk)
            bulk_load(sx + off, xb + off, min(static_cast<uint32_t>(kOpChunk), bytes - off), &bar, pol);
    }
    uint4 rv[RB][IT];
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < RB; ++j) {
        const int i = S + j * T_ + t;
        if (i < spill_lo) {
#pragma unroll
            for (int k = 0; k < IT; ++k) rv[j][k] = load_item(xb + static_cast<int64_t>(i) * C::kBlockBytes + 16 * k);
        } else {
#pragma unroll
            for (int k = 0; k < IT; ++k) rv[j][k] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    {
        // the tail: kSpillBatch blocks per thread in flight at a time
        const uint64_t pol = policy_evict_last();
        for (int i0 = spill_lo + t; i0 < nb; i0 += kSpillBatch * T_) {
            uint4 v[kSpillBatch][IT];
#pragma unroll
            for (int u = 0; u < kSpillBatch; ++u) {
                const int i = i0 + u * T_;
                const uint4 *p = reinterpret_cast<const uint4 *>(xb + static_cast<int64_t>(i) * C::kBlockBytes);
#pragma unroll
                for (int k = 0; k < IT; ++k) {
                    if (i < nb)
                        asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                                     : "=r"(v[u][k].x), "=r"(v[u][k].y), "=r"(v[u][k].z), "=r"(v[u][k].w)
                                     : "l"(p + k), "l"(pol));
                    else
                        v[u][k] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
#pragma unroll
            for (int u = 0; u < kSpillBatch; ++u) m = fmaxf(m, items_absmax<T>(v[u]));
        }
    }
#pragma unroll
    for (int j = 0; j < RB; ++j) m = fmaxf(m, items_absmax<T>(rv[j]));
    bool ok = true;
    if (S > 0) {
        ok = mbar_wait(&bar, 0, a.timeout_ns, abort_flag, a.status);
        for (int i = t; ok && i < S * IT; i += T_) {
            const uint4 v = ld_shared_v4(sx + static_cast<int64_t>(i) * 16);
            m = fmaxf(m, item_absmax(v, static_cast<T *>(nullptr)));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) wmax[warp] = m;
    __syncthreads();
    if (warp == 0) {
        uint32_t go = 0u;
        if (lane == 0) {
            float cm = 0.0f;
            for (int k = 0; k < kOpThreads / 32; ++k) cm = fmaxf(cm, wmax[k]);
            a.partials[blockIdx.x] = cm;
            // every CTA of the cooperative launch is resident and arrives
            // exactly once, also after a give-up of its own; bounded
            go = grid_meet(a.grid_bar, meet_gen, a.timeout_ns, abort_flag, a.status) ? 1u : 0u;
        }
        go = __shfl_sync(0xffffffffu, go, 0);
        float gm = 0.0f;
        if (go)
            for (int k = lane; k < static_cast<int>(gridDim.x); k += 32) gm = fmaxf(gm, __ldcg(a.partials + k));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, o));
        if (lane == 0) {
            s_amax = gm;
            s_go = go && !*abort_flag;
        }
    }
    __syncthreads();
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // CTA-uniform: a give-up anywhere in the CTA (the bulk-copy wait) raised
    // the abort flag before the barrier above.  On that path no bulk copy may
    // still be landing when the CTA exits: wait for them (bounded).
    if (!s_go) {
        if (t == 0 && S > 0) {
            volatile uint32_t keep_waiting = 0u;
            mbar_wait(&bar, 0, a.timeout_ns, &keep_waiting, a.status);
        }
        return;
    }

    // ---- pass B: the quantizer's arithmetic on the blocks held on chip,
    // then on the tail read again
    const float g = __fdiv_rn(s_amax, kTensorScaleDiv);
    const float six_g = __fmul_rn(6.0f, g);
    const float inv6g = __frcp_rn(six_g);
    const bool exact_only = !(six_g > 0.0f) || isinf(inv6g);
    if (blockIdx.x == 0 && t == 0) *a.g_out = g;
    if (t < 128) rcp_table[t] = block_rcp(static_cast<uint32_t>(t), g);
    __syncthreads();

    // Block i of the range (all lanes of a warp run the scale-word shuffles;
    // a 4-block group sits in 4 neighbouring lanes and is valid as a whole).
    auto encode = [&](int i, bool valid, const uint32_t (&w)[W]) {
        const uint32_t sb = block_scale_byte(block_absmax(w, static_cast<T *>(nullptr)), six_g, inv6g, exact_only);
        const uint2 cw = block_codes<T, W>(w, rcp_table[sb]);
        uint32_t word = sb;
        word |= __shfl_down_sync(0xffffffffu, sb, 1) << 8;
        word |= __shfl_down_sync(0xffffffffu, sb, 2) << 16;
        word |= __shfl_down_sync(0xffffffffu, sb, 3) << 24;
        if (valid) {
            const int64_t b = b0 + i;
            if (store_ok(a.codes + b * 8, 8, a.codes, codes_bytes, a.status)) *reinterpret_cast<uint2 *>(a.codes + b * 8) = cw;
            if ((lane & 3) == 0) {
                const int64_t r = b / bpr, kb = b - r * bpr;
                const int64_t off = ((r >> 7) * (kb4 >> 2) + (kb >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4;
                if (store_ok(a.scales + off, 4, a.scales, scales_bytes, a.status))
                    *reinterpret_cast<uint32_t *>(a.scales + off) = word;
            }
        }
    };
    // shared-memory part: warp-uniform trip count
    for (int base = warp * 32; base < S; base += T_) {
        const int i = base + lane;
        const bool valid = i < S;
        uint4 it[IT];
#pragma unroll
        for (int k = 0; k < IT; ++k)
            it[k] = valid ? ld_shared_v4(sx + static_cast<int64_t>(i) * C::kBlockBytes + 16 * k) : make_uint4(0u, 0u, 0u, 0u);
        uint32_t w[W];
        words_of<T>(it, w);
        encode(i, valid, w);
    }
    // register part
#pragma unroll
    for (int j = 0; j < RB; ++j) {
        if (S + j * T_ + (t - lane) >= spill_lo) break;          // warp-uniform: the warp's first lane
        const int i = S + j * T_ + t;
        uint32_t w[W];
        words_of<T>(rv[j], w);
        encode(i, i < spill_lo, w);
    }
    // the tail, read again (from L2 where the evict-last hint kept it),
    // kSpillBatch blocks per thread in flight at a time
    for (int base = spill_lo + warp * 32; base < nb; base += kSpillBatch * T_) {
        uint4 it[kSpillBatch][IT];
#pragma unroll
        for (int u = 0; u < kSpillBatch; ++u) {
            const int i = base + u * T_ + lane;
#pragma unroll
            for (int k = 0; k < IT; ++k)
                it[u][k] = i < nb ? load_item(xb + static_cast<int64_t>(i) * C::kBlockBytes + 16 * k)
                                  : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kSpillBatch; ++u) {
            const int i = base + u * T_ + lane;
            uint32_t w[W];
            words_of<T>(it[u], w);
            encode(i, i < nb, w);
        }
    }
    // zero scale words of the padding rows [rows, roundup(rows, 128)), split over the CTAs
    const int64_t pad_words = (round_up(a.rows, 128) - a.rows) * (kb4 / 4);
    const int64_t p_lo = pad_words * blockIdx.x / gridDim.x, p_hi = pad_words * (blockIdx.x + 1) / gridDim.x;
    for (int64_t i = p_lo + t; i < p_hi; i += T_) {
        const int64_t r = a.rows + i / (kb4 / 4), q = 4 * (i % (kb4 / 4));
        uint8_t *sp = a.scales + ((r >> 7) * (kb4 >> 2) + (q >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4;
        if (store_ok(sp, 4, a.scales, scales_bytes, a.status)) *reinterpret_cast<uint32_t *>(sp) = 0u;
    }
}

template <typename T>
cudaError_t launch_onepass_t(const OpArgs &a, int grid, cudaStream_t stream) {
    auto kern = quantize_onepass_kernel<T>;
    const int smem = kOpSmemData;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kOpThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    // Cooperative (its CTAs meet once), and a programmatic dependent of the
    // kernel before it if the driver takes both; cooperative alone otherwise.
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    static std::atomic<int> coop_pdl{1};
    if (coop_pdl.load()) {
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        e = cudaLaunchKernelEx(&cfg, kern, a);
        if (e == cudaSuccess) return e;
        if (e != cudaErrorInvalidValue && e != cudaErrorNotSupported) return e;
        (void)cudaGetLastError();      // a refused configuration, not a failed launch
        coop_pdl.store(0);
    }
    cfg.attrs = attr + 1;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace

bool quantize_onepass_usable(int64_t rows, int64_t cols, int64_t ld, bool bf16) {
    // Opt-in (NVFP4_QUANTIZE_ONEPASS=1).  Measured on B200, bf16 8192 x 5120:
    // 43.5 us against 37.0 us for the two passes (it does read x from DRAM
    // once, 84.0 MB, but with one 512-thread CTA per SM the encode arithmetic
    // runs at a quarter of the two-pass encode kernel's occupancy and the
    // kernel is issue-bound, not DRAM-bound: 23% of DRAM peak); bf16
    // 4096 x 5120 inside the prefill step: the same step time either way.
    const char *opt = getenv("NVFP4_QUANTIZE_ONEPASS");
    if (opt == nullptr || opt[0] != '1') return false;
    const int64_t bytes = rows * cols * (bf16 ? 2 : 4);
    return ld == cols && cols % 64 == 0 && bytes >= (int64_t(8) << 20) && rows * cols / kBlock < (int64_t(1) << 40);
}

cudaError_t launch_quantize_onepass(const void *x, bool bf16, int64_t rows, int64_t cols, uint8_t *codes,
                                    uint8_t *scales, float *g_out, float *partials, uint32_t *grid_bar,
                                    uint32_t *status, uint64_t timeout_ns, int num_sms, cudaStream_t stream) {
    OpArgs a;
    a.x = x;
    a.rows = rows;
    a.cols = cols;
    a.partials = partials;
    a.grid_bar = grid_bar;
    a.codes = codes;
    a.scales = scales;
    a.g_out = g_out;
    a.status = status;
    a.timeout_ns = timeout_ns;
    const int grid = num_sms < kMaxAmaxPartials ? num_sms : kMaxAmaxPartials;
    return bf16 ? launch_onepass_t<__nv_bfloat16>(a, grid, stream) : launch_onepass_t<float>(a, grid, stream);
}

}  // namespace nvfp4
