// gemm2sm.cu -- W4A4 block-scaled FP4 GEMM with two-CTA (cta_group::2) MMAs
// for large M (prefill-shaped calls).
//
// Same operation as gemm.cu (NVFP4 activations x NVFP4 weights on the FP4
// tensor cores, fp32 accumulation, tensor scales in the epilogue; aixq.cc
// article on Unsloth Dynamic NVFP4, section "核心差异：W4A4 vs W4A16").  Why a
// second kernel: a one-CTA 128x256 tile moves more bytes through each SM's
// shared memory (TMA fill plus tensor-core operand reads) per MMA than shared
// memory can deliver in the MMA's time.  A CTA pair computes a 256x256 tile
// with one M=256 MMA: each CTA loads and feeds only its own 128 A rows and its
// own 128-row half of B, so shared-memory traffic per FLOP drops by a third.
//
// Pair protocol (cluster of 2, leader = rank 0):
//   producer (each CTA)  TMA of its A and B halves, completion counted on the
//                        leader's `full` barrier (cta_group::2 load form; the
//                        leader posts the expected bytes of both CTAs); its
//                        scale atoms by bulk copy onto its own `sfdata` barrier.
//   scale warps (each)   own TMEM scale slot via tcgen05.st, then arrive on the
//                        leader's `sf_full` barrier (remote arrive for rank 1).
//   MMA (leader only)    tcgen05.mma.cta_group::2 M=256 N=256 K=64 into both
//                        CTAs' TMEM; commits multicast to both CTAs' `empty`
//                        and `tfull` barriers.
//   epilogue (each)      drains its own 128 accumulator rows, then arrives on
//                        the leader's `tempty` barrier.
// No load uses cluster multicast.  Every wait is bounded.
#include <cstdlib>
#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace nvfp4 {

struct PairArgs {
    const uint8_t *sfa;      // tiled scales of A (M rows)
    const uint8_t *sfb;      // tiled scales of B (N rows)
    const float *ga;
    const float *gb;
    void *y;
    int64_t ldy;
    int32_t M, N;
    int32_t num_k_steps;     // K / 64
    int32_t num_pm, num_qn;  // 256-row / 256-column pair tiles
    int32_t a_row_tiles;     // ceil(M / 128)
    int32_t b_row_tiles;     // ceil(N / 128)
    uint32_t *status;
    uint64_t timeout_ns;
};

struct PairCfg {
    static constexpr int kAStage = 128 * 128;     // own 128 A rows x 128 bytes
    static constexpr int kBStage = 128 * 128;     // own 128-row half of B
    static constexpr int kSfaStage = 4 * 512;     // own rows' atoms, 4 K-steps
    static constexpr int kSfbStage = 2 * 4 * 512; // all 256 N rows' atoms, 4 K-steps
    static constexpr int kStageBytes = kAStage + kBStage + kSfaStage + kSfbStage;
    static constexpr int kStages = 5;
    static constexpr int kSfCols = 16 + 32;       // TMEM scale columns per stage
    static constexpr int kAccCols = 256;
    static constexpr int kSfBase = kAccCols;
    static constexpr int kTmemCols = 512;
    static constexpr int kBarBytes = 8 * (4 * kStages + 4) + 16;
    static constexpr int kSmemBytes = kStages * kStageBytes + kBarBytes + 1024;
    static constexpr int kThreads = 448;
    static_assert(kSfBase + kStages * kSfCols <= kTmemCols, "tensor memory budget");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

template <typename OutT>
__global__ void __launch_bounds__(448, 1)
gemm_nvf4_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ PairArgs args) {
    using C = PairCfg;
    constexpr int STAGES = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = sA + STAGES * C::kAStage;
    uint8_t *sSfa = sB + STAGES * C::kBStage;
    uint8_t *sSfb = sSfa + STAGES * C::kSfaStage;
    uint64_t *full = reinterpret_cast<uint64_t *>(sSfb + STAGES * C::kSfbStage);   // leader's
    uint64_t *sfdata = full + STAGES;                                                // each CTA's
    uint64_t *sf_full = sfdata + STAGES;                                             // leader's
    uint64_t *empty = sf_full + STAGES;                                              // each CTA's
    uint64_t *tfull = empty + STAGES;                                                // each CTA's
    uint64_t *tempty = tfull + 2;                                                    // leader's
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(tempty + 2);
    volatile uint32_t *abort_flag = tmem_holder + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&sfdata[s], 1);
            mbar_init(&sf_full[s], 8);     // one arrive per scale warp, both CTAs
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&tfull[s], 1);
            mbar_init(&tempty[s], 16);     // one arrive per epilogue warp, both CTAs
        }
        *abort_flag = 0u;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc_pair(tmem_holder, C::kTmemCols);
    tc_fence_before();
    cluster_sync();       // both CTAs' barriers initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    const int cid = static_cast<int>(blockIdx.x >> 1);
    const int ncl = static_cast<int>(gridDim.x >> 1);
    const int num_tiles = args.num_pm * args.num_qn;
    const int num_kstages = (args.num_k_steps + 3) / 4;

    if (warp == 0) {
        if (lane == 0) {
            // -------------------------------------------------------- producer
            asm volatile("griddepcontrol.wait;" ::: "memory");
            const uint64_t pol = policy_evict_normal();
            uint32_t stage = 0, phase = 0;
            for (int tile = cid; tile < num_tiles; tile += ncl) {
                const int pm = tile % args.num_pm;
                const int qn = tile / args.num_pm;
                const int a_rt = 2 * pm + static_cast<int>(rank);   // this CTA's A row tile
                bool ok = true;
                for (int ks = 0; ks < num_kstages; ++ks) {
                    if (!mbar_wait_cluster(&empty[stage], phase ^ 1u, args.timeout_ns, abort_flag, args.status)) {
                        ok = false;
                        break;
                    }
                    const int nk = min(4, args.num_k_steps - 4 * ks);
                    const uint32_t leader_full = mapa_shared(smem_addr(&full[stage]), 0);
                    if (leader) mbar_arrive_expect_tx(&full[stage], 2 * (C::kAStage + C::kBStage));
                    tma_load_2d_pair(sA + stage * C::kAStage, &tmA, leader_full, ks * 128, a_rt * 128, pol);
                    tma_load_2d_pair(sB + stage * C::kBStage, &tmB, leader_full, ks * 128,
                                     (2 * qn + static_cast<int>(rank)) * 128, pol);
                    uint32_t sf_bytes = 0;
                    const bool have_a = a_rt < args.a_row_tiles;
                    sf_bytes += have_a ? nk * 512 : 0;
                    for (int q = 0; q < 2; ++q) sf_bytes += (2 * qn + q < args.b_row_tiles) ? nk * 512 : 0;
                    mbar_arrive_expect_tx(&sfdata[stage], sf_bytes);
                    if (have_a)
                        bulk_load(sSfa + stage * C::kSfaStage,
                                  args.sfa + (static_cast<int64_t>(a_rt) * args.num_k_steps + 4 * ks) * 512,
                                  nk * 512, &sfdata[stage], pol);
                    for (int q = 0; q < 2; ++q) {
                        const int rt = 2 * qn + q;
                        if (rt < args.b_row_tiles)
                            bulk_load(sSfb + stage * C::kSfbStage + q * 2048,
                                      args.sfb + (static_cast<int64_t>(rt) * args.num_k_steps + 4 * ks) * 512,
                                      nk * 512, &sfdata[stage], pol);
                    }
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // -------------------------------------------------------- MMA issuer
            constexpr uint32_t idesc = make_idesc_nvf4_pair(256);
            const uint32_t a_base = smem_addr(sA), b_base = smem_addr(sB);
            uint32_t stage = 0, phase = 0, acc_phase = 0;
            for (int tile = cid; tile < num_tiles; tile += ncl) {
                if (!mbar_wait_cluster(&tempty[0], acc_phase ^ 1u, args.timeout_ns, abort_flag, args.status)) break;
                tc_fence_after();
                bool ok = true;
                for (int ks = 0; ks < num_kstages; ++ks) {
                    if (!mbar_wait_cluster(&full[stage], phase, args.timeout_ns, abort_flag, args.status) ||
                        !mbar_wait_cluster(&sf_full[stage], phase, args.timeout_ns, abort_flag, args.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nk = min(4, args.num_k_steps - 4 * ks);
                    const uint32_t sf = tmem_base + C::kSfBase + stage * C::kSfCols;
                    for (int j = 0; j < nk; ++j) {
                        const uint64_t adesc = make_operand_desc(a_base + stage * C::kAStage + 32 * j);
                        const uint64_t bdesc = make_operand_desc(b_base + stage * C::kBStage + 32 * j);
                        mma_nvf4_pair(tmem_base, adesc, bdesc, idesc, sf + 4 * j, sf + 16 + 8 * j,
                                      (ks | j) != 0 ? 1u : 0u);
                    }
                    tc_commit_pair(&empty[stage], 0x3);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit_pair(&tfull[0], 0x3);
                acc_phase ^= 1u;
            }
        }
    } else if (warp < 6) {
        // ------------------------------------------------------------ scale warps
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        uint32_t stage = 0, phase = 0;
        for (int tile = cid; tile < num_tiles; tile += ncl) {
            bool ok = true;
            for (int ks = 0; ks < num_kstages; ++ks) {
                const bool got = mbar_wait(&sfdata[stage], phase, args.timeout_ns, abort_flag, args.status);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                const int nk = min(4, args.num_k_steps - 4 * ks);
                const uint32_t sf = tmem_base + lane_off + C::kSfBase + stage * C::kSfCols;
                const uint8_t *a_src = sSfa + stage * C::kSfaStage + lane * 16;
                const uint8_t *b_src = sSfb + stage * C::kSfbStage + lane * 16;
                // one 16-column and one 32-column TMEM store per stage (columns
                // of K-steps a partial last stage does not have are never read)
                uint32_t av[16], bv[32];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 a = ld_shared_v4(a_src + j * 512);
                    const uint4 b0 = ld_shared_v4(b_src + j * 512);
                    const uint4 b1 = ld_shared_v4(b_src + 2048 + j * 512);
                    av[4 * j] = a.x; av[4 * j + 1] = a.y; av[4 * j + 2] = a.z; av[4 * j + 3] = a.w;
                    bv[8 * j] = b0.x; bv[8 * j + 1] = b0.y; bv[8 * j + 2] = b0.z; bv[8 * j + 3] = b0.w;
                    bv[8 * j + 4] = b1.x; bv[8 * j + 5] = b1.y; bv[8 * j + 6] = b1.z; bv[8 * j + 7] = b1.w;
                }
                (void)nk;
                tmem_st_32x32b_x16(sf, av);
                tmem_st_32x32b_x32(sf + 16, bv);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_addr(&sf_full[stage]), 0));
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
        }
    } else {
        // ------------------------------------------------------------ epilogue
        asm volatile("griddepcontrol.wait;" ::: "memory");
        const int quarter = warp & 3;
        const int half = (warp - 6) >> 2;
        const int row = quarter * 32 + lane;
        const float alpha = __fmul_rn(*args.ga, *args.gb);
        const uint32_t leader_tempty = mapa_shared(smem_addr(&tempty[0]), 0);
        uint32_t acc_phase = 0;
        for (int tile = cid; tile < num_tiles; tile += ncl) {
            const int pm = tile % args.num_pm;
            const int qn = tile / args.num_pm;
            const bool ok = mbar_wait_cluster(&tfull[0], acc_phase, args.timeout_ns, abort_flag, args.status);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const int p = pm * 256 + static_cast<int>(rank) * 128 + row;
            const uint32_t tb = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + half * 128;
            OutT *yrow = static_cast<OutT *>(args.y) + static_cast<int64_t>(p) * args.ldy;
            uint32_t r[2][32];
            tmem_ld_32x32b_x32(tb, r[0]);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (c + 1 < 4) tmem_ld_32x32b_x32(tb + (c + 1) * 32, r[(c + 1) & 1]);
                const int q0 = qn * 256 + half * 128 + c * 32;
                if (p < args.M) {
                    if constexpr (sizeof(OutT) == 2) {
                        uint32_t pk[16];
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            __nv_bfloat162 b2 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(r[c & 1][2 * k]), alpha),
                                                                      __fmul_rn(__uint_as_float(r[c & 1][2 * k + 1]), alpha));
                            pk[k] = *reinterpret_cast<uint32_t *>(&b2);
                        }
                        if (q0 + 32 <= args.N) {
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                *reinterpret_cast<uint4 *>(yrow + q0 + 8 * i) =
                                    make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                        } else {
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                if (q0 + 2 * i < args.N)
                                    reinterpret_cast<unsigned short *>(yrow)[q0 + 2 * i] = static_cast<unsigned short>(pk[i] & 0xffffu);
                                if (q0 + 2 * i + 1 < args.N)
                                    reinterpret_cast<unsigned short *>(yrow)[q0 + 2 * i + 1] = static_cast<unsigned short>(pk[i] >> 16);
                            }
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (q0 + i < args.N) yrow[q0 + i] = __fmul_rn(__uint_as_float(r[c & 1][i]), alpha);
                    }
                }
                if (c + 1 < 4) tmem_ld_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_tempty);
            acc_phase ^= 1u;
        }
    }

    tc_fence_before();
    cluster_sync();       // no CTA leaves while its peer may still touch its memory
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

template <typename OutT>
static cudaError_t run_pair(const Operand &act, const Operand &wgt, int64_t K, void *y, int64_t ldy,
                            uint32_t *status, uint64_t timeout_ns, int max_clusters, cudaStream_t stream) {
    using C = PairCfg;
    CUtensorMap tmA, tmB;
    if (encode_tensor_map_u8(&tmA, act.codes, K / 2, act.rows, 128, 128) != CUDA_SUCCESS ||
        encode_tensor_map_u8(&tmB, wgt.codes, K / 2, wgt.rows, 128, 128) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    PairArgs a;
    a.sfa = act.scales;
    a.sfb = wgt.scales;
    a.ga = act.g;
    a.gb = wgt.g;
    a.y = y;
    a.ldy = ldy;
    a.M = static_cast<int32_t>(act.rows);
    a.N = static_cast<int32_t>(wgt.rows);
    a.num_k_steps = static_cast<int32_t>(K / 64);
    a.num_pm = static_cast<int32_t>(ceil_div(act.rows, 256));
    a.num_qn = static_cast<int32_t>(ceil_div(wgt.rows, 256));
    a.a_row_tiles = static_cast<int32_t>(ceil_div(act.rows, 128));
    a.b_row_tiles = static_cast<int32_t>(ceil_div(wgt.rows, 128));
    a.status = status;
    a.timeout_ns = timeout_ns;
    const int tiles = a.num_pm * a.num_qn;
    const int clusters = tiles < max_clusters ? tiles : max_clusters;
    cudaError_t e = cudaFuncSetAttribute(gemm_nvf4_pair_kernel<OutT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * clusters);
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, gemm_nvf4_pair_kernel<OutT>, tmA, tmB, a);
}

// How many 2-CTA clusters of the pair kernel can be resident at once (0 if
// the kernel cannot be configured).
static int pair_max_clusters() {
    static int cached = -1;
    if (cached >= 0) return cached;
    int n = 0;
    bool ok = true;
    auto kb = gemm_nvf4_pair_kernel<__nv_bfloat16>;
    auto kf = gemm_nvf4_pair_kernel<float>;
    ok = ok && cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, PairCfg::kSmemBytes) == cudaSuccess;
    ok = ok && cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, PairCfg::kSmemBytes) == cudaSuccess;
    if (ok) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2);
        cfg.blockDim = dim3(PairCfg::kThreads);
        cfg.dynamicSmemBytes = PairCfg::kSmemBytes;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, kb, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();
    cached = n;
    return cached;
}

bool pair_gemm_usable(int64_t M, int64_t N, int num_sms) {
    // Opt-in (NVFP4_GEMM_CTA_PAIR=1): on the shapes measured so far the
    // one-CTA kernel is faster, so the pair kernel is not the default.
    const char *opt = getenv("NVFP4_GEMM_CTA_PAIR");
    if (opt == nullptr || opt[0] != '1') return false;
    const int maxc = pair_max_clusters();
    return maxc > 0 && M >= 256 && ceil_div(M, 256) * ceil_div(N, 256) >= 2 * maxc && num_sms > 0;
}

cudaError_t launch_gemm_pair(const Operand &act, const Operand &wgt, int64_t K, void *y, bool y_bf16,
                             int64_t ldy, uint32_t *status, uint64_t timeout_ns, cudaStream_t stream) {
    const int maxc = pair_max_clusters();
    if (maxc <= 0) return cudaErrorLaunchOutOfResources;
    return y_bf16 ? run_pair<__nv_bfloat16>(act, wgt, K, y, ldy, status, timeout_ns, maxc, stream)
                  : run_pair<float>(act, wgt, K, y, ldy, status, timeout_ns, maxc, stream);
}

}  // namespace nvfp4
