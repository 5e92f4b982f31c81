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
// Pair protocol (cluster of 2, leader = rank 0), K in slabs of 256 (4 MMA
// K-steps of 64), slabs in groups of two:
//   producer (each CTA)  TMA (cta_group::2 form) of its A rows and its half of
//                        B, completing on the leader's `full` barrier (the
//                        leader posts both CTAs' bytes); TMA of its A-scale
//                        atoms and of all 256 B rows' atoms onto its own
//                        `sfull` barrier.
//   TMEM warps (8/CTA)   scale factors: shared -> registers -> tcgen05.st into
//                        this CTA's TMEM scale slot, one slot per group of two
//                        slabs; the two slots alternate and each belongs to
//                        one half of the warps (one warp per lane quarter),
//                        which writes the group with one x64 and one x32
//                        store and then arrives remotely on the leader's
//                        `sf_ready`.  Few, wide stores per handshake keep the
//                        tensor pipe fed; one slab per handshake measured
//                        about 50% slower per slab.
//                        Epilogue: read this CTA's 128x256 accumulator into
//                        registers, release it on the leader's `tempty`, then
//                        scale, convert and store while the next tile runs.
//   MMA (leader only)    per group: wait `sf_ready`; per slab: wait `full`,
//                        4 pair MMAs M=256 N=256 K=64, commit to both CTAs'
//                        `empty`; after the group commit to both CTAs'
//                        `sf_free`; after a tile commit to both CTAs' `tfull`.
// TMEM: accumulator columns [0,256), scale slots [256,352) and [352,448).
// No load uses cluster multicast.  Every wait is bounded.
#include <cstdlib>
#include <cstring>
#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace nvfp4 {

struct PairArgs {
    const float *ga;
    const float *gb;
    void *y;
    int64_t ldy;
    int32_t M, N;
    int32_t num_k_steps;     // MMA K steps: K / 64 (FP4 kinds) or K / 32 (W4A8)
    int32_t num_pm, num_qn;  // 256-row / 256-column pair tiles
    int32_t tma_store;       // bf16 output written by TMA stores (needs N % 8 == 0)
    float *ymax_part;        // if set: this CTA's largest |y| as stored, at [blockIdx.x]
    uint32_t *status;
    uint64_t timeout_ns;
};

struct PairCfg {
    static constexpr int kAStage = 128 * 128;     // own 128 A rows x 128 bytes
    static constexpr int kBStage = 128 * 128;     // own 128-row half of B
    static constexpr int kSfaStage = 4 * 512;     // own rows' atoms, 4 K-steps
    static constexpr int kSfbStage = 2 * 4 * 512; // both B row tiles' atoms, 4 K-steps
    static constexpr int kABBytes = kAStage + kBStage;
    static constexpr int kSfBytes = kSfaStage + kSfbStage;
    static constexpr int kStageBytes = kABBytes + kSfBytes;
    static constexpr int kStages = 5;
    static constexpr int kSlabCols = 48;          // scale columns of one slab: 16 A + 32 B
    static constexpr int kSlotCols = 2 * kSlabCols;
    static constexpr int kSfCol = 256;            // first scale slot
    static constexpr int kTmemCols = 512;
    static constexpr int kTmemWarps = 8;
    static constexpr int kThreads = 32 * (2 + kTmemWarps);
    static constexpr int kStagingBytes = kTmemWarps * 32 * 128;   // per warp: 32 rows x 64 bf16
    static constexpr int kBarBytes = 8 * (3 * kStages + 4 + 3) + 16;
    static constexpr int kSmemBytes = kStages * kStageBytes + kStagingBytes + kBarBytes + 1024;
    static_assert(kSfCol + 2 * kSlotCols <= kTmemCols, "tensor memory budget");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// (columns past N are exact zeros: folding them into ym cannot raise it)
// (y_base, y_bytes, status: the debug build's store checks)
template <typename OutT>
__device__ __forceinline__ void pair_store_chunk(const uint32_t (&r)[32], float alpha, OutT *yrow,
                                                 int q0, int N, YMax &ym, const void *y_base, size_t y_bytes,
                                                 uint32_t *status) {
    if constexpr (sizeof(OutT) == 2) {
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(r[2 * k]), alpha),
                                                      __fmul_rn(__uint_as_float(r[2 * k + 1]), alpha));
            pk[k] = *reinterpret_cast<uint32_t *>(&b2);
            ym.bf16x2(pk[k]);
        }
        if (q0 + 32 <= N) {
            if (store_ok(yrow + q0, 64, y_base, y_bytes, status)) {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    *reinterpret_cast<uint4 *>(yrow + q0 + 8 * i) =
                        make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                if (q0 + 2 * i < N && store_ok(yrow + q0 + 2 * i, 2, y_base, y_bytes, status))
                    reinterpret_cast<unsigned short *>(yrow)[q0 + 2 * i] = static_cast<unsigned short>(pk[i] & 0xffffu);
                if (q0 + 2 * i + 1 < N && store_ok(yrow + q0 + 2 * i + 1, 2, y_base, y_bytes, status))
                    reinterpret_cast<unsigned short *>(yrow)[q0 + 2 * i + 1] = static_cast<unsigned short>(pk[i] >> 16);
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float v = __fmul_rn(__uint_as_float(r[i]), alpha);
            if (q0 + i < N && store_ok(yrow + q0 + i, 4, y_base, y_bytes, status)) yrow[q0 + i] = v;
            ym.f32(v);
        }
    }
}

template <typename OutT, int FMT>
__global__ void __launch_bounds__(PairCfg::kThreads, 1)
gemm_nvf4_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                      const __grid_constant__ CUtensorMap tmY, const __grid_constant__ PairArgs args) {
    using C = PairCfg;
    constexpr int STAGES = C::kStages;
    constexpr bool MX = FMT == kFmtMX;
    constexpr bool W8 = FMT == kFmtW4A8;          // MXFP8 A (activations) x MXFP4 B (weights, unpacked)
    // scale atoms per stage and 128-row tile: one per K step (NVFP4, K = 64),
    // one per two (MXFP4), one per stage (W4A8: four K steps of 32)
    constexpr int kAtoms = MX ? 2 : (W8 ? 1 : 4);
    // operand bytes both CTAs' copies signal on the leader's barrier: the
    // unpacking copy of the W4A8 weights counts the packed bytes it reads
    constexpr uint32_t kFullTx = 2u * (W8 ? C::kAStage + C::kBStage / 2 : C::kABBytes);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = sA + STAGES * C::kAStage;
    uint8_t *sSfa = sB + STAGES * C::kBStage;
    uint8_t *sSfb = sSfa + STAGES * C::kSfaStage;
    uint8_t *staging = sSfb + STAGES * C::kSfbStage;                                 // 1024-aligned
    uint64_t *full = reinterpret_cast<uint64_t *>(staging + C::kStagingBytes);       // leader's
    uint64_t *sfull = full + STAGES;                                                 // each CTA's
    uint64_t *empty = sfull + STAGES;                                                // each CTA's
    uint64_t *sf_ready = empty + STAGES;                                             // leader's [2]
    uint64_t *sf_free = sf_ready + 2;                                                // each CTA's [2]
    uint64_t *tfull = sf_free + 2;                                                   // each CTA's
    uint64_t *tempty = tfull + 1;                                                    // leader's
    uint64_t *mma_done = tempty + 1;                                                 // leader's
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile uint32_t *abort_flag = tmem_holder + 1;
    __shared__ float s_ymax[C::kTmemWarps];               // TMEM warps' largest |stored y|

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;

    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmSA);
        prefetch_tensormap(&tmSB);
        if (args.tma_store) prefetch_tensormap(&tmY);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&sfull[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sf_ready[s], C::kTmemWarps);       // the slot's 4 warps in both CTAs
            mbar_init(&sf_free[s], 1);
        }
        mbar_init(tfull, 1);
        mbar_init(tempty, 2 * C::kTmemWarps);
        mbar_init(mma_done, 1);
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
    const int num_groups = (num_kstages + 1) / 2;

    if (warp == 0) {
        {
            // -------------------------------------------------------- producer
            // The whole warp walks the loop (its waits are warp-uniform); one
            // elected lane issues the copies.
            const bool issue = elect_one_sync();
            asm volatile("griddepcontrol.wait;" ::: "memory");
            const uint64_t pol = policy_evict_normal();
            const uint32_t leader_full0 = mapa_shared(smem_addr(&full[0]), 0);
            uint32_t stage = 0, phase = 0;
            int issued = 0;
            for (int tile = cid; tile < num_tiles; tile += ncl) {
                const int pm = tile % args.num_pm;
                const int qn = tile / args.num_pm;
                const int a_rt = 2 * pm + static_cast<int>(rank);   // this CTA's A row tile
                const int b_rt = 2 * qn + static_cast<int>(rank);   // this CTA's half of B
                bool ok = true;
                for (int ks = 0; ks < num_kstages; ++ks) {
                    if (!__all_sync(0xffffffffu, mbar_wait(&empty[stage], phase ^ 1u, args.timeout_ns, abort_flag,
                                                           args.status))) {
                        ok = false;
                        break;
                    }
                    const uint32_t bar = leader_full0 + 8u * stage;
                    if (issue) {
                        if (leader) mbar_arrive_expect_tx(&full[stage], kFullTx);
                        tma_load_2d_pair(sA + stage * C::kAStage, &tmA, bar, ks * 128, a_rt * 128, pol);
                        tma_load_2d_pair(sB + stage * C::kBStage, &tmB, bar, ks * 128, b_rt * 128, pol);
                        // scale atoms of this stage: kAtoms per 128-row tile
                        mbar_arrive_expect_tx(&sfull[stage], C::kSfBytes / (4 / kAtoms));
                        tma_load_3d(sSfa + stage * C::kSfaStage, &tmSA, &sfull[stage], 0, kAtoms * ks, a_rt, pol);
                        tma_load_3d(sSfb + stage * C::kSfbStage, &tmSB, &sfull[stage], 0, kAtoms * ks, 2 * qn, pol);
                    }
                    __syncwarp();
                    ++issued;
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
            }
            // No copy may still be landing when the pair exits: wait (bounded,
            // also after an abort) for the last loads issued into every stage:
            // this CTA's scale loads on its own barrier, and in the leader the
            // operand loads of both CTAs, which complete on the leader's.
            volatile uint32_t keep_waiting = 0u;
            for (int j = issued > STAGES ? issued - STAGES : 0; j < issued; ++j) {
                const uint32_t par = static_cast<uint32_t>(j / STAGES) & 1u;
                mbar_wait(&sfull[j % STAGES], par, args.timeout_ns, &keep_waiting, args.status);
                if (leader) mbar_wait(&full[j % STAGES], par, args.timeout_ns, &keep_waiting, args.status);
            }
        }
    } else if (warp == 1) {
        if (leader) {
            // -------------------------------------------------------- MMA issuer
            // The whole warp walks the loop; one elected lane issues the MMAs
            // and commits.
            const uint32_t issue = elect_one_sync() ? 1u : 0u;
            constexpr uint32_t idesc = make_idesc_nvf4_pair(256);
            constexpr uint32_t idesc_w8[4] = {make_idesc_mxf8f6f4_pair(256, 0, 5, 0), make_idesc_mxf8f6f4_pair(256, 0, 5, 1),
                                              make_idesc_mxf8f6f4_pair(256, 0, 5, 2), make_idesc_mxf8f6f4_pair(256, 0, 5, 3)};
            constexpr uint32_t idesc_mx0 = make_idesc_mxf4(256, 256, 0), idesc_mx1 = make_idesc_mxf4(256, 256, 1);
            const uint32_t a_base = smem_addr(sA), b_base = smem_addr(sB);
            uint32_t stage = 0, phase = 0;
            uint32_t gcount = 0;     // groups issued so far (slot = gcount & 1)
            int t = 0;
            bool ok = true;
            for (int tile = cid; tile < num_tiles && ok; tile += ncl, ++t) {
                // the previous tile's accumulator has been read out of TMEM
                if (t > 0 && !__all_sync(0xffffffffu, mbar_wait(tempty, static_cast<uint32_t>(t - 1) & 1u,
                                                                 args.timeout_ns, abort_flag, args.status)))
                    break;
                tc_fence_after();
                for (int g = 0; g < num_groups && ok; ++g, ++gcount) {
                    const uint32_t slot = gcount & 1u;
                    if (!__all_sync(0xffffffffu, mbar_wait(&sf_ready[slot], (gcount >> 1) & 1u, args.timeout_ns,
                                                           abort_flag, args.status))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int h = 0; h < 2; ++h) {
                        const int ks = 2 * g + h;
                        if (ks >= num_kstages) break;
                        if (!__all_sync(0xffffffffu,
                                        mbar_wait(&full[stage], phase, args.timeout_ns, abort_flag, args.status))) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const int nk = min(4, args.num_k_steps - 4 * ks);
                        const uint32_t sf = tmem_base + C::kSfCol + slot * C::kSlotCols + h * C::kSlabCols;
                        // K-step j is 32 bytes further along the swizzled rows: +2 in
                        // the descriptors' address field (units of 16 bytes)
                        const uint64_t adesc = make_operand_desc(a_base + stage * C::kAStage);
                        const uint64_t bdesc = make_operand_desc(b_base + stage * C::kBStage);
                        // MXFP4: K step j reads the columns of atom j/2 and
                        // its bytes {0,1} or {2,3} (descriptor's scale IDs)
                        auto kstep = [&](int j) {
                            if constexpr (W8)   // atom 0 of the slab, byte j (scale ID), E4M3 x E2M1
                                mma_mxf8f6f4_pair(tmem_base, adesc + 2 * j, bdesc + 2 * j, idesc_w8[j], sf, sf + 16,
                                                  (ks | j) != 0 ? 1u : 0u, issue);
                            else if constexpr (MX)
                                mma_mxf4_pair(tmem_base, adesc + 2 * j, bdesc + 2 * j, (j & 1) ? idesc_mx1 : idesc_mx0,
                                              sf + 4 * (j >> 1), sf + 16 + 8 * (j >> 1), (ks | j) != 0 ? 1u : 0u, issue);
                            else
                                mma_nvf4_pair(tmem_base, adesc + 2 * j, bdesc + 2 * j, idesc, sf + 4 * j,
                                              sf + 16 + 8 * j, (ks | j) != 0 ? 1u : 0u, issue);
                        };
                        if (nk == 4) {
#pragma unroll
                            for (int j = 0; j < 4; ++j) kstep(j);
                        } else {
                            for (int j = 0; j < nk; ++j) kstep(j);
                        }
                        tc_commit_pair(&empty[stage], 0x3, issue);
                        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                    }
                    if (ok) tc_commit_pair(&sf_free[slot], 0x3, issue);
                }
                if (ok) tc_commit_pair(tfull, 0x3, issue);
            }
            // Tensor memory is freed after the final cluster barrier: first let
            // every MMA this warp issued complete (bounded, also after an abort).
            tc_commit_pair(mma_done, 0x1, issue);
            volatile uint32_t keep_waiting = 0u;
            mbar_wait(mma_done, 0, args.timeout_ns, &keep_waiting, args.status);
        }
    } else {
        // ------------------------------------------------------------ TMEM warps
        const int quarter = warp & 3;
        const int half = (warp - 2) >> 2;         // which slab of a group this warp's scales cover
        const int row = quarter * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
        const uint32_t leader_ready0 = mapa_shared(smem_addr(&sf_ready[0]), 0);
        const uint32_t leader_tempty = mapa_shared(smem_addr(tempty), 0);
        float alpha = 0.0f;
        bool alpha_ready = false;
        // Largest |y| this thread stores; rows and columns past M and N are
        // exact zeros (zero-filled operand rows), so folding them is harmless.
        YMax ym;
        uint32_t gcount = 0;
        int t = 0;
        bool ok = true;
        // Epilogue of tile number te (this CTA's count), pair-tile index tile_e.
        auto epilogue = [&](int te, int tile_e) -> bool {
            const bool got = mbar_wait(tfull, static_cast<uint32_t>(te) & 1u, args.timeout_ns, abort_flag,
                                               args.status);
            if (!__all_sync(0xffffffffu, got)) return false;
            tc_fence_after();
            if (!alpha_ready) {
                asm volatile("griddepcontrol.wait;" ::: "memory");
                alpha = __fmul_rn(args.ga ? *args.ga : 1.0f, args.gb ? *args.gb : 1.0f);   // MXFP4: none
                alpha_ready = true;
            }
            uint32_t r[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld_32x32b_x32(lane_base + half * 128 + c * 32, r[c]);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(leader_tempty);
            const int pm = tile_e % args.num_pm;
            const int qn = tile_e / args.num_pm;
            if (sizeof(OutT) == 2 && args.tma_store) {
                // bf16: stage 32 rows x 64 columns at a time (128-byte swizzle,
                // 16-byte chunk c of row r at chunk c ^ (r % 8)) and let one
                // TMA store write it; rows and columns past M and N are clipped
                // (exactly, because rows are whole 16-byte units when N % 8 == 0).
                uint8_t *stg = staging + (warp - 2) * (32 * 128);
                const int row0 = pm * 256 + static_cast<int>(rank) * 128 + quarter * 32;
                const int col0 = qn * 256 + half * 128;
#pragma unroll
                for (int c2 = 0; c2 < 2; ++c2) {
                    if (lane == 0) bulk_wait_group_read0();   // staging buffer free again
                    __syncwarp();
#pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {
                        const uint32_t *src = r[2 * c2 + (ch >> 2)] + (ch & 3) * 8;
                        uint32_t w[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            __nv_bfloat162 b2 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(src[2 * k]), alpha),
                                                                      __fmul_rn(__uint_as_float(src[2 * k + 1]), alpha));
                            w[k] = *reinterpret_cast<uint32_t *>(&b2);
                            ym.bf16x2(w[k]);
                        }
                        st_shared_v4(stg + lane * 128 + ((ch ^ (lane & 7)) * 16), w[0], w[1], w[2], w[3]);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    // a box wholly past the last row or column is not issued
                    if (lane == 0 && row0 < args.M && col0 + 64 * c2 < args.N) {
                        tma_store_2d(&tmY, stg, col0 + 64 * c2, row0);
                        bulk_commit_group();
                    }
                }
            } else {
                const int p = pm * 256 + static_cast<int>(rank) * 128 + row;
                if (p < args.M) {
                    OutT *yrow = static_cast<OutT *>(args.y) + static_cast<int64_t>(p) * args.ldy;
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        pair_store_chunk<OutT>(r[c], alpha, yrow, qn * 256 + half * 128 + c * 32, args.N, ym, args.y,
                                               matrix_extent(args.M, args.N, args.ldy, sizeof(OutT)), args.status);
                }
            }
            return true;
        };
        uint32_t sstage = 0, sphase = 0;   // scale-ring position of the next slab
        int prev_tile = -1;
        for (int tile = cid; tile < num_tiles && ok; tile += ncl, ++t) {
            for (int g = 0; g < num_groups; ++g, ++gcount) {
                const uint32_t slot = gcount & 1u;
                const int nslab = min(2, num_kstages - 2 * g);
                // slot h belongs to the warps of half h: one x64 and one x32
                // store write both slabs' scales of the group for this lane quarter
                if (slot == static_cast<uint32_t>(half)) {
                    const bool freed = mbar_wait(&sf_free[slot], ((gcount >> 1) & 1u) ^ 1u, args.timeout_ns,
                                                         abort_flag, args.status);
                    if (!__all_sync(0xffffffffu, freed)) { ok = false; break; }
                    tc_fence_after();
                    uint32_t v[2 * C::kSlabCols];
                    uint32_t st_i = sstage, ph_i = sphase;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (h < nslab) {
                            const bool got = mbar_wait(&sfull[st_i], ph_i, args.timeout_ns, abort_flag, args.status);
                            if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                            const uint8_t *a_src = sSfa + st_i * C::kSfaStage + lane * 16;
                            const uint8_t *b_src = sSfb + st_i * C::kSfbStage + lane * 16;
                            // the B box holds both row tiles' atoms, tile after tile:
                            // kAtoms each (the atom slots past kAtoms hold bytes no
                            // MMA reads)
                            constexpr int kTile1 = kAtoms * 512;
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const uint4 a = ld_shared_v4(a_src + j * 512);
                                const uint4 b0 = ld_shared_v4(b_src + j * 512);
                                const uint4 b1 = ld_shared_v4(b_src + kTile1 + j * 512);
                                uint32_t *va = v + h * C::kSlabCols + 4 * j;
                                uint32_t *vb = v + h * C::kSlabCols + 16 + 8 * j;
                                va[0] = a.x; va[1] = a.y; va[2] = a.z; va[3] = a.w;
                                vb[0] = b0.x; vb[1] = b0.y; vb[2] = b0.z; vb[3] = b0.w;
                                vb[4] = b1.x; vb[5] = b1.y; vb[6] = b1.z; vb[7] = b1.w;
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < C::kSlabCols; ++i) v[h * C::kSlabCols + i] = 0u;   // never read
                        }
                        if (++st_i == STAGES) { st_i = 0; ph_i ^= 1u; }
                    }
                    if (!ok) break;
                    const uint32_t sf = lane_base + C::kSfCol + slot * C::kSlotCols;
                    tmem_st_32x32b_x64(sf, *reinterpret_cast<const uint32_t(*)[64]>(v));
                    tmem_st_32x32b_x32(sf + 64, *reinterpret_cast<const uint32_t(*)[32]>(v + 64));
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_remote(leader_ready0 + 8u * slot);
                }
                for (int h = 0; h < nslab; ++h)
                    if (++sstage == STAGES) { sstage = 0; sphase ^= 1u; }
                // once the first group of this tile is handed over, drain the previous tile
                if (g == 0 && prev_tile >= 0) {
                    if (!epilogue(t - 1, prev_tile)) { ok = false; break; }
                    prev_tile = -1;
                }
            }
            if (ok) prev_tile = tile;
        }
        if (ok && prev_tile >= 0) epilogue(t - 1, prev_tile);
        if (lane == 0) bulk_wait_group0();   // this warp's output stores are complete
        float m = ym.value();
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) s_ymax[warp - 2] = m;
    }

    tc_fence_before();
    cluster_sync();       // no CTA leaves while its peer may still touch its memory
    if (threadIdx.x == 0 && args.ymax_part != nullptr) {
        float m = 0.0f;
#pragma unroll
        for (int k = 0; k < C::kTmemWarps; ++k) m = fmaxf(m, s_ymax[k]);
        args.ymax_part[blockIdx.x] = m;
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

template <typename OutT, int FMT>
static cudaError_t run_pair(const Operand &act, const Operand &wgt, int64_t K, void *y, int64_t ldy,
                            uint32_t *status, uint64_t timeout_ns, int max_clusters, cudaStream_t stream,
                            float *ymax_part, int *nparts) {
    using C = PairCfg;
    constexpr bool MX = FMT == kFmtMX, W8 = FMT == kFmtW4A8;
    // MMA K steps: 64 values (FP4 kinds) or 32 (W4A8)
    const uint64_t k_steps = static_cast<uint64_t>(W8 ? K / 32 : K / 64);
    // 512-byte scale atoms per 128-row tile: one per K step (NVFP4), one per
    // two (MXFP4), one per four (W4A8)
    const uint64_t atoms_rt = W8 ? (k_steps + 3) / 4 : (MX ? (k_steps + 1) / 2 : k_steps);
    const uint32_t box_atoms = W8 ? 1 : (MX ? 2 : 4);
    CUtensorMap tmA, tmB, tmSA, tmSB;
    // A rows of 128 bytes per stage: 256 E2M1 values, or 128 E4M3 values
    // (W4A8); W4A8's E2M1 weights are unpacked by the copy into 8-bit
    // containers, 128 values per 128-byte row
    const bool maps_ok =
        encode_tensor_map_u8(&tmA, act.codes, W8 ? K : K / 2, act.rows, 128, 128) == CUDA_SUCCESS &&
        (W8 ? encode_tensor_map_fp4_unpacked(&tmB, wgt.codes, K, wgt.rows, 128)
            : encode_tensor_map_u8(&tmB, wgt.codes, K / 2, wgt.rows, 128, 128)) == CUDA_SUCCESS &&
        encode_scale_map(&tmSA, act.scales, atoms_rt, ceil_div(act.rows, 128), 1, box_atoms) == CUDA_SUCCESS &&
        encode_scale_map(&tmSB, wgt.scales, atoms_rt, ceil_div(wgt.rows, 128), 2, box_atoms) == CUDA_SUCCESS;
    if (!maps_ok) return cudaErrorInvalidValue;
    CUtensorMap tmY;
    memset(&tmY, 0, sizeof(tmY));    // unused unless tma_store
    const bool tma_store = sizeof(OutT) == 2 && wgt.rows % 8 == 0;
    if (tma_store &&
        encode_output_map_bf16(&tmY, y, static_cast<uint64_t>(act.rows), static_cast<uint64_t>(wgt.rows),
                               static_cast<uint64_t>(ldy), 64, 32) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    PairArgs a;
    a.ga = act.g;
    a.gb = wgt.g;
    a.y = y;
    a.ldy = ldy;
    a.M = static_cast<int32_t>(act.rows);
    a.N = static_cast<int32_t>(wgt.rows);
    a.num_k_steps = static_cast<int32_t>(k_steps);
    a.num_pm = static_cast<int32_t>(ceil_div(act.rows, 256));
    a.num_qn = static_cast<int32_t>(ceil_div(wgt.rows, 256));
    a.tma_store = tma_store ? 1 : 0;
    a.ymax_part = ymax_part;
    a.status = status;
    a.timeout_ns = timeout_ns;
    const int tiles = a.num_pm * a.num_qn;
    const int clusters = tiles < max_clusters ? tiles : max_clusters;
    cudaError_t e = cudaFuncSetAttribute(gemm_nvf4_pair_kernel<OutT, FMT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * clusters);
    if (nparts) *nparts = 2 * clusters;
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
    return cudaLaunchKernelEx(&cfg, gemm_nvf4_pair_kernel<OutT, FMT>, tmA, tmB, tmSA, tmSB, tmY, a);
}

// How many 2-CTA clusters of the pair kernel can be resident at once (0 if
// the kernel cannot be configured).  Computed once (a function-local static's
// initialiser runs exactly once, also under concurrent first calls).
static int pair_max_clusters_query() {
    int n = 0;
    bool ok = true;
    auto kb = gemm_nvf4_pair_kernel<__nv_bfloat16, kFmtNV>;
    ok = ok && cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, PairCfg::kSmemBytes) == cudaSuccess;
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
    return n;
}

static int pair_max_clusters() {
    static const int n = pair_max_clusters_query();
    return n;
}

bool pair_gemm_usable(int64_t M, int64_t N, int num_sms) {
    // NVFP4_GEMM_CTA_PAIR=0 keeps every shape on the one-CTA kernel.
    const char *opt = getenv("NVFP4_GEMM_CTA_PAIR");
    if (opt != nullptr && opt[0] == '0') return false;
    const int maxc = pair_max_clusters();
    // every resident pair gets at least one 256x256 tile
    return maxc > 0 && num_sms > 0 && M >= 256 && ceil_div(M, 256) * ceil_div(N, 256) >= maxc;
}

cudaError_t launch_gemm_pair(const Operand &act, const Operand &wgt, int64_t K, void *y, bool y_bf16,
                             int64_t ldy, uint32_t *status, uint64_t timeout_ns, cudaStream_t stream,
                             float *ymax_part, int *nparts, int fmt) {
    const int maxc = pair_max_clusters();
    if (maxc <= 0) return cudaErrorLaunchOutOfResources;
#define NVFP4_PAIR(F)                                                                                              \
    return y_bf16 ? run_pair<__nv_bfloat16, F>(act, wgt, K, y, ldy, status, timeout_ns, maxc, stream, ymax_part, nparts) \
                  : run_pair<float, F>(act, wgt, K, y, ldy, status, timeout_ns, maxc, stream, ymax_part, nparts);
    if (fmt == kFmtMX) { NVFP4_PAIR(kFmtMX) }
    if (fmt == kFmtW4A8) { NVFP4_PAIR(kFmtW4A8) }
    NVFP4_PAIR(kFmtNV)
#undef NVFP4_PAIR
}

}  // namespace nvfp4
