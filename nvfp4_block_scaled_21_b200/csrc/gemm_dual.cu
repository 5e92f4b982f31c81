// gemm_dual.cu -- the MLP's gate and up projections in one W4A4 block-scaled
// GEMM with the SiLU(gate) * up epilogue.
//
// The fused MLP step of the W4A4 path (aixq.cc article on Unsloth Dynamic
// NVFP4, section "核心差异：W4A4 vs W4A16": activations and weights both NVFP4
// into the FP4 tensor cores) computes h = SiLU(x Wg^T) * (x Wu^T) and
// re-quantizes h to NVFP4 for the down projection.  This kernel computes both
// products for one 128 x 128 output tile from the same activation slabs (the
// gate and up weight tiles as one 256-row B operand, so the fp32 accumulator
// in tensor memory holds gate in columns [0,128) and up in [128,256)) and its
// epilogue writes
//     gate = fl32(acc_g * fl32(gx * gwg)),  up = fl32(acc_u * fl32(gx * gwu)),
//     h = fl32(fl32(gate / fl32(1 + exp(-gate))) * up)
// with the hardware exponential and the fast division (__expf, __fdividef:
// a few ulp of fp32, far inside the tolerance the GEMM's own accumulation
// needs), plus, per CTA, max |h| in the format of the quantizer's first pass.
//
// Re-quantizing h (each NVFP4 tensor carries its own two-level scaling:
// NVFP4 wiki page, section "技術原理") needs max |h| over the whole tensor
// before the first block can be encoded.  When every CTA holds exactly one
// tile (a cooperative launch, tiles <= SMs: dual_fused_requant_usable), the
// epilogue does it in place:
// each CTA publishes its max |h|, meets the others at a bounded grid-wide
// meeting point (grid_meet), and encodes the tile it still holds in
// registers with the quantizer's own arithmetic (encode.cuh), so h never
// goes to memory unless asked for.
// Otherwise h is written and the quantizer's encode pass runs on it.
//
// Roles (one persistent CTA per SM, 14 warps), as in gemm.cu:
//   warp 0      TMA producer: per 256-deep K slab the A tile (128 activation
//               rows), both 128-row weight tiles, and the three 512-byte
//               scale atoms per K step, into a 4-stage ring.
//   warp 1      TMEM allocation and MMA issue: per K step one MMA
//               (M=128, N=256, K=64) whose B operand is the gate tile with
//               the up tile after it in shared memory, so gate lands in
//               columns [0,128) and up in [128,256); one accumulator stage.
//   warps 2..5  scale warps: scale atoms from shared memory to their TMEM
//               lane quarter (tcgen05.st), two stages per handshake.
//   warps 6..13 epilogue: two warps per lane quarter, 64 columns each.
// Every wait is bounded; a timeout sets the status word and winds down.
#include <atomic>
#include <cmath>
#include <cstdlib>
#include "common.cuh"
#include "encode.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace nvfp4 {

namespace {

struct DualArgs {
    const uint8_t *sfa;       // tiled scales of the activations (M rows)
    const uint8_t *sfbg;      // tiled scales of Wg (N rows)
    const uint8_t *sfbu;      // tiled scales of Wu
    const float *gx, *gwg, *gwu;
    float *h;                 // [M][ldh] fp32, or null (fused re-quantization only)
    int64_t ldh;
    float *partials;          // max |h| per CTA (gridDim.x values)
    uint8_t *hq_codes;        // fused re-quantization (null: off): h_q codes [M][N/2],
    uint8_t *hq_scales;       // tiled scales,
    float *hq_g;              // tensor scale,
    uint32_t *grid_bar;       // grid meeting point: arrival count, generation
    int32_t kb4;              // h_q scale blocks per row, rounded up to 4
    int32_t M, N;
    int32_t num_k_steps;      // K / 64
    int32_t num_p_tiles, num_q_tiles;
    int32_t preload;          // weight stages loaded before the dependent-launch wait
    uint32_t *status;
    uint64_t timeout_ns;
};

struct DualCfg {
    static constexpr int kAStage = 128 * 128;
    static constexpr int kBStage = 128 * 128;                 // each of the two weight tiles
    static constexpr int kSfStage = 4 * 512;                  // per operand: 4 K-steps x one atom
    static constexpr int kStageBytes = kAStage + 2 * kBStage + 3 * kSfStage;
    static constexpr int kStages = 4;
    static constexpr int kSfCols = 48;                        // SFA 16 | SFB 32 (gate, up per K step)
    static constexpr int kSfBase = 256;                       // after the accumulator (gate | up)
    static constexpr int kTmemCols = 512;
    static constexpr int kThreads = 448;
    static constexpr int kBarBytes = 8 * (3 * kStages + 3) + 16;
    static constexpr int kSmemBytes = kStages * kStageBytes + kBarBytes + 1024;
    static_assert(kSfBase + kStages * kSfCols <= kTmemCols, "tensor memory budget");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

__device__ __forceinline__ float silu_mul(float gate, float up) {
    return __fmul_rn(__fdividef(gate, __fadd_rn(1.0f, __expf(-gate))), up);
}

__global__ void __launch_bounds__(448, 1)
gemm_nvf4_dual_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmBg,
                      const __grid_constant__ CUtensorMap tmBu, const __grid_constant__ DualArgs args) {
    using C = DualCfg;
    constexpr int STAGES = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = sA + STAGES * C::kAStage;                  // per stage: gate tile, then up tile
    uint8_t *sSf = sB + STAGES * 2 * C::kBStage;            // per stage: SFA | SFBg | SFBu atoms
    uint64_t *full = reinterpret_cast<uint64_t *>(sSf + STAGES * 3 * C::kSfStage);
    uint64_t *sf_full = full + STAGES;
    uint64_t *empty = sf_full + STAGES;
    uint64_t *tfull = empty + STAGES;
    uint64_t *tempty = tfull + 1;
    uint64_t *mma_done = tempty + 1;                         // every MMA of this CTA has completed
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile uint32_t *abort_flag = tmem_holder + 1;
    __shared__ float warp_max[8];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmBg);
        prefetch_tensormap(&tmBu);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&sf_full[s], 4);
            mbar_init(&empty[s], 1);
        }
        mbar_init(tfull, 1);
        mbar_init(tempty, 8);
        mbar_init(mma_done, 1);
        *abort_flag = 0u;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_holder, C::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    const int num_tiles = args.num_p_tiles * args.num_q_tiles;
    const int num_kstages = (args.num_k_steps + 3) / 4;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------------ producer
            const uint64_t pol = policy_evict_normal();
            auto load_w = [&](uint32_t st, int qt, int ks, int nk) {
                tma_load_2d(sB + st * 2 * C::kBStage, &tmBg, &full[st], ks * 128, qt * 128, pol);
                tma_load_2d(sB + st * 2 * C::kBStage + C::kBStage, &tmBu, &full[st], ks * 128, qt * 128, pol);
                const int64_t off = (static_cast<int64_t>(qt) * args.num_k_steps + 4 * ks) * 512;
                bulk_load(sSf + (st * 3 + 1) * C::kSfStage, args.sfbg + off, nk * 512, &full[st], pol);
                bulk_load(sSf + (st * 3 + 2) * C::kSfStage, args.sfbu + off, nk * 512, &full[st], pol);
            };
            auto load_a = [&](uint32_t st, int pt, int ks, int nk) {
                tma_load_2d(sA + st * C::kAStage, &tmA, &full[st], ks * 128, pt * 128, pol);
                bulk_load(sSf + (st * 3) * C::kSfStage,
                          args.sfa + (static_cast<int64_t>(pt) * args.num_k_steps + 4 * ks) * 512,
                          nk * 512, &full[st], pol);
            };
            // The weights do not depend on the kernel launched before this one:
            // the first `pre` stages of weights are requested before the wait.
            const bool has_tile = static_cast<int>(blockIdx.x) < num_tiles;
            const int pre = has_tile ? min(args.preload, min(STAGES, num_kstages)) : 0;
            const int pt0 = static_cast<int>(blockIdx.x) % args.num_p_tiles;
            const int qt0 = static_cast<int>(blockIdx.x) / args.num_p_tiles;
            for (int p = 0; p < pre; ++p) {
                const int nk = min(4, args.num_k_steps - 4 * p);
                mbar_arrive_expect_tx(&full[p], C::kAStage + 2 * C::kBStage + 3 * nk * 512);
                load_w(static_cast<uint32_t>(p), qt0, p, nk);
            }
            asm volatile("griddepcontrol.wait;" ::: "memory");
            for (int p = 0; p < pre; ++p) load_a(static_cast<uint32_t>(p), pt0, p, min(4, args.num_k_steps - 4 * p));
            uint32_t stage = 0, phase = 0;
            int it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
                const int pt = tile % args.num_p_tiles;
                const int qt = tile / args.num_p_tiles;
                for (int ks = 0; ks < num_kstages; ++ks, ++it) {
                    if (it >= pre) {
                        const int nk = min(4, args.num_k_steps - 4 * ks);
                        if (!mbar_wait(&empty[stage], phase ^ 1u, args.timeout_ns, abort_flag, args.status)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&full[stage], C::kAStage + 2 * C::kBStage + 3 * nk * 512);
                        load_a(stage, pt, ks, nk);
                        load_w(stage, qt, ks, nk);
                    }
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            // No copy may still be landing when the CTA exits: wait (bounded,
            // also after an abort) for the last load issued into every stage.
            // On the normal path the MMA thread has consumed them all already.
            // (Stages counted before a failed empty wait were issued; the
            // preloaded ones always are.)
            const int issued = it > pre ? it : pre;
            volatile uint32_t keep_waiting = 0u;
            for (int j = issued > STAGES ? issued - STAGES : 0; j < issued; ++j)
                mbar_wait(&full[j % STAGES], static_cast<uint32_t>(j / STAGES) & 1u, args.timeout_ns,
                          &keep_waiting, args.status);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------------------ MMA issuer
            constexpr uint32_t idesc = make_idesc_nvf4(256);
            const uint32_t a_base = smem_addr(sA), b_base = smem_addr(sB);
            uint32_t stage = 0, phase = 0, acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
                if (!mbar_wait(tempty, acc_phase ^ 1u, args.timeout_ns, abort_flag, args.status)) break;
                tc_fence_after();
                for (int ks = 0; ks < num_kstages; ++ks) {
                    if (!mbar_wait(&full[stage], phase, args.timeout_ns, abort_flag, args.status) ||
                        !mbar_wait(&sf_full[stage], phase, args.timeout_ns, abort_flag, args.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nk = min(4, args.num_k_steps - 4 * ks);
                    const uint32_t sf = tmem_base + C::kSfBase + stage * C::kSfCols;
                    // K-step j: +32 bytes = +2 in the descriptors' address field
                    const uint64_t adesc = make_operand_desc(a_base + stage * C::kAStage);
                    // the 256 B rows: 128 of Wg, then 128 of Wu (1024-byte atoms, contiguous)
                    const uint64_t bdesc = make_operand_desc(b_base + stage * 2 * C::kBStage);
                    auto kstep = [&](int j) {
                        const uint32_t acc = (ks | j) != 0 ? 1u : 0u;
                        mma_nvf4(tmem_base, adesc + 2 * j, bdesc + 2 * j, idesc, sf + 4 * j, sf + 16 + 8 * j, acc);
                    };
                    if (nk == 4) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) kstep(j);
                    } else {
                        for (int j = 0; j < nk; ++j) kstep(j);
                    }
                    tc_commit(&empty[stage]);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit(tfull);
                acc_phase ^= 1u;
            }
            // Tensor memory is freed below: first let every MMA this thread
            // issued complete (bounded, also after an abort).
            tc_commit(mma_done);
            volatile uint32_t keep_waiting = 0u;
            mbar_wait(mma_done, 0, args.timeout_ns, &keep_waiting, args.status);
        }
    } else if (warp < 6) {
        // ------------------------------------------------------------ scale warps
        // Lane l of every quarter receives the 16 bytes at l*16 of each atom
        // (the replicated scale layout the block-scaled MMA reads).
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        uint32_t stage = 0, phase = 0;
        uint32_t pend[2];
        int npend = 0;
        auto flush = [&]() {
            if (npend == 0) return;
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                for (int i = 0; i < npend; ++i) mbar_arrive(&sf_full[pend[i]]);
            npend = 0;
        };
        bool ok = true;
        for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
            for (int ks = 0; ks < num_kstages; ++ks) {
                const bool got = mbar_wait(&full[stage], phase, args.timeout_ns, abort_flag, args.status);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                const uint8_t *src = sSf + stage * 3 * C::kSfStage + lane * 16;
                uint32_t av[16], bv[32];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 a = ld_shared_v4(src + j * 512);
                    const uint4 g = ld_shared_v4(src + C::kSfStage + j * 512);
                    const uint4 u = ld_shared_v4(src + 2 * C::kSfStage + j * 512);
                    av[4 * j] = a.x; av[4 * j + 1] = a.y; av[4 * j + 2] = a.z; av[4 * j + 3] = a.w;
                    // B scales of K step j: the gate rows' 4 columns, then the up rows'
                    bv[8 * j] = g.x; bv[8 * j + 1] = g.y; bv[8 * j + 2] = g.z; bv[8 * j + 3] = g.w;
                    bv[8 * j + 4] = u.x; bv[8 * j + 5] = u.y; bv[8 * j + 6] = u.z; bv[8 * j + 7] = u.w;
                }
                const uint32_t sf = tmem_base + lane_off + C::kSfBase + stage * C::kSfCols;
                tmem_st_32x32b_x16(sf, av);
                tmem_st_32x32b_x32(sf + 16, bv);
                pend[npend++] = stage;
                if (npend == 2) flush();
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
        }
        flush();
    } else {
        // ------------------------------------------------------------ epilogue
        asm volatile("griddepcontrol.wait;" ::: "memory");   // tensor scales may be fresh
        // the meeting point's generation, read early (see grid_meet_generation)
        const uint32_t meet_gen = (warp == 6 && lane == 0 && args.hq_codes != nullptr)
                                      ? grid_meet_generation(args.grid_bar) : 0u;
        const int quarter = warp & 3;
        const int half = (warp - 6) >> 2;
        const int row = quarter * 32 + lane;
        const float ag = __fmul_rn(*args.gx, *args.gwg);
        const float au = __fmul_rn(*args.gx, *args.gwu);
        const bool fuse = args.hq_codes != nullptr;    // then this CTA has exactly one tile
        float hv[2][32];                               // that tile's h for this thread
        int tile_pt = 0, tile_qt = 0;
        bool have_tile = false;
        float amax = 0.0f;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            const int pt = tile % args.num_p_tiles;
            const int qt = tile / args.num_p_tiles;
            const bool ok = mbar_wait(tfull, acc_phase, args.timeout_ns, abort_flag, args.status);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const int p = pt * 128 + row;
            const uint32_t tb = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + half * 64;
            float *hrow = args.h + static_cast<int64_t>(p) * args.ldh;
            tile_pt = pt;
            tile_qt = qt;
            have_tile = true;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t g[32], u[32];
                tmem_ld_32x32b_x32(tb + c * 32, g);
                tmem_ld_32x32b_x32(tb + 128 + c * 32, u);
                tmem_ld_wait();
                float *h = hv[c];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    h[i] = silu_mul(__fmul_rn(__uint_as_float(g[i]), ag), __fmul_rn(__uint_as_float(u[i]), au));
                    amax = fmaxf(amax, fabsf(h[i]));
                }
                const int q0 = qt * 128 + half * 64 + c * 32;
                if (args.h != nullptr && p < args.M) {
                    const size_t h_bytes = matrix_extent(args.M, args.N, args.ldh, 4);   // debug-build checks
                    if (q0 + 32 <= args.N) {
                        if (store_ok(hrow + q0, 128, args.h, h_bytes, args.status)) {
#pragma unroll
                            for (int i = 0; i < 32; i += 4)
                                *reinterpret_cast<float4 *>(hrow + q0 + i) = make_float4(h[i], h[i + 1], h[i + 2], h[i + 3]);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (q0 + i < args.N && store_ok(hrow + q0 + i, 4, args.h, h_bytes, args.status))
                                hrow[q0 + i] = h[i];
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty);
            acc_phase ^= 1u;
        }
        // this CTA's max |h| (rows past M and columns past N hold exact zeros)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (lane == 0) warp_max[warp - 6] = amax;

        if (fuse) {
            // ---- grid-wide max |h|, then encode this thread's 4 blocks of 16
            __shared__ float s_amax;
            __shared__ uint32_t s_go;
            asm volatile("bar.sync 1, 256;" ::: "memory");        // the 8 epilogue warps
            if (warp == 6) {
                uint32_t go = 0u;
                if (lane == 0) {
                    float m = 0.0f;
                    for (int i = 0; i < 8; ++i) m = fmaxf(m, warp_max[i]);
                    args.partials[blockIdx.x] = m;
                    // every CTA of the cooperative launch is resident and
                    // arrives exactly once (also after a give-up of its own),
                    // so the wait ends unless one of them gave up; bounded
                    go = grid_meet(args.grid_bar, meet_gen, args.timeout_ns, abort_flag, args.status) ? 1u : 0u;
                }
                go = __shfl_sync(0xffffffffu, go, 0);
                // the grid's maxima, read by the whole warp at once
                float gmax = 0.0f;
                if (go)
                    for (int i = lane; i < static_cast<int>(gridDim.x); i += 32)
                        gmax = fmaxf(gmax, __ldcg(args.partials + i));
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, o));
                if (lane == 0) {
                    s_amax = gmax;
                    s_go = go && have_tile && !*abort_flag;
                }
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (s_go) {
                // the quantizer's arithmetic: g, 6g, its reciprocal, per block
                // the E4M3 scale byte and the E2M1 codes
                const float g = __fdiv_rn(s_amax, kTensorScaleDiv);
                const float six_g = __fmul_rn(6.0f, g);
                const float inv6g = __frcp_rn(six_g);
                const bool exact_only = !(six_g > 0.0f) || isinf(inv6g);
                if (blockIdx.x == 0 && warp == 6 && lane == 0) *args.hq_g = g;
                const int p = tile_pt * 128 + row;
                const int kb0 = (tile_qt * 128 + half * 64) / kBlock;   // first of this thread's 4 blocks
                const int nblk = args.N / kBlock;
                uint32_t word = 0;
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) w[i] = __float_as_uint(hv[b >> 1][(b & 1) * 16 + i]);
                    const uint32_t sb = block_scale_byte(block_absmax(w, static_cast<float *>(nullptr)), six_g, inv6g,
                                                         exact_only);
                    const uint2 cw = block_codes<float, 16>(w, block_rcp(sb, g));
                    word |= sb << (8 * b);
                    uint8_t *cp = args.hq_codes + static_cast<int64_t>(p) * (args.N / 2) + (kb0 + b) * 8;
                    if (p < args.M && kb0 + b < nblk &&
                        store_ok(cp, 8, args.hq_codes, static_cast<size_t>(args.M) * (args.N / 2), args.status))
                        *reinterpret_cast<uint2 *>(cp) = cw;
                }
                // rows past M and blocks past N/16 are zero blocks: byte 0, the
                // layout's padding value; blocks past kb4 are outside it
                if (kb0 < args.kb4) {
                    const int64_t off = (static_cast<int64_t>(p >> 7) * (args.kb4 / 4) + (kb0 >> 2)) * 512 +
                                        (p & 31) * 16 + ((p >> 5) & 3) * 4;
                    if (store_ok(args.hq_scales + off, 4, args.hq_scales,
                                 static_cast<size_t>(round_up(args.M, 128)) * args.kb4, args.status))
                        *reinterpret_cast<uint32_t *>(args.hq_scales + off) = word;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = 0.0f;
        for (int i = 0; i < 8; ++i) m = fmaxf(m, warp_max[i]);
        args.partials[blockIdx.x] = m;
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

}  // namespace

bool dual_fused_requant_usable(int64_t M, int64_t N, int num_sms, int max_partials) {
    // NVFP4_MLP_FUSED_REQUANT=0 keeps the separate encode pass on h.  Measured
    // on B200 at M = 128, K = 5120, N = 17408: the gate/up call takes 37.9 us
    // this way against 40.0 us with the encode pass.
    const char *opt = getenv("NVFP4_MLP_FUSED_REQUANT");
    if (opt != nullptr && opt[0] == '0') return false;
    const int64_t tiles = ceil_div(M, 128) * ceil_div(N, 128);
    return tiles >= 1 && tiles <= num_sms && tiles <= max_partials;
}

cudaError_t launch_gemm_dual_silu(const Operand &act, const Operand &wg, const Operand &wu, int64_t K,
                                  float *h, int64_t ldh, float *partials, int max_partials, int *num_partials,
                                  uint32_t *status, uint64_t timeout_ns, int num_sms, cudaStream_t stream,
                                  bool weights_ready, uint8_t *hq_codes, uint8_t *hq_scales, float *hq_g,
                                  uint32_t *grid_bar) {
    using C = DualCfg;
    CUtensorMap tmA, tmBg, tmBu;
    if (encode_tensor_map_u8(&tmA, act.codes, K / 2, act.rows, 128, 128) != CUDA_SUCCESS ||
        encode_tensor_map_u8(&tmBg, wg.codes, K / 2, wg.rows, 128, 128) != CUDA_SUCCESS ||
        encode_tensor_map_u8(&tmBu, wu.codes, K / 2, wu.rows, 128, 128) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    DualArgs a;
    a.sfa = act.scales;
    a.sfbg = wg.scales;
    a.sfbu = wu.scales;
    a.gx = act.g;
    a.gwg = wg.g;
    a.gwu = wu.g;
    a.h = h;
    a.ldh = ldh;
    a.partials = partials;
    a.hq_codes = hq_codes;
    a.hq_scales = hq_scales;
    a.hq_g = hq_g;
    a.grid_bar = grid_bar;
    a.kb4 = static_cast<int32_t>(kb4_of(wg.rows));
    a.M = static_cast<int32_t>(act.rows);
    a.N = static_cast<int32_t>(wg.rows);
    a.num_k_steps = static_cast<int32_t>(K / 64);
    a.num_p_tiles = static_cast<int32_t>(ceil_div(act.rows, 128));
    a.num_q_tiles = static_cast<int32_t>(ceil_div(wg.rows, 128));
    a.preload = weights_ready ? C::kStages : 0;
    a.status = status;
    a.timeout_ns = timeout_ns;
    const int tiles = a.num_p_tiles * a.num_q_tiles;
    int grid = tiles < num_sms ? tiles : num_sms;
    if (grid > max_partials) grid = max_partials;
    if (grid < 1) grid = 1;
    *num_partials = grid;
    // the in-epilogue re-quantization: one tile per CTA and a meeting point
    if (hq_codes != nullptr && (grid != tiles || grid_bar == nullptr)) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(gemm_nvf4_dual_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeCooperative;        // the fused form's CTAs wait for one another
    attr[1].val.cooperative = 1;
    cfg.attrs = attr;
    if (hq_codes == nullptr) {
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, gemm_nvf4_dual_kernel, tmA, tmBg, tmBu, a);
    }
    // Cooperative, and a programmatic dependent of the quantizer if the
    // driver takes both; cooperative alone otherwise (remembered).
    static std::atomic<int> coop_pdl{1};
    if (coop_pdl.load()) {
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        e = cudaLaunchKernelEx(&cfg, gemm_nvf4_dual_kernel, tmA, tmBg, tmBu, a);
        if (e == cudaSuccess) return e;
        if (e != cudaErrorInvalidValue && e != cudaErrorNotSupported) return e;
        (void)cudaGetLastError();      // a refused configuration, not a failed launch
        coop_pdl.store(0);
    }
    cfg.attrs = attr + 1;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemm_nvf4_dual_kernel, tmA, tmBg, tmBu, a);
}

}  // namespace nvfp4
