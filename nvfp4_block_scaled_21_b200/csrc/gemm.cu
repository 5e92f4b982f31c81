// gemm.cu -- W4A4 block-scaled FP4 GEMM on the sm_100a tensor cores.
//
// The linear layer consumes NVFP4 weights and NVFP4 activations directly on
// the FP4 tensor cores, with no dequantize-to-16-bit step (aixq.cc article on
// Unsloth Dynamic NVFP4, section "核心差异：W4A4 vs W4A16"); the tensor cores
// apply the per-16-element E4M3 block scales themselves, and the FP32 tensor
// scales are applied once in the epilogue (NVFP4 wiki page, section "技術原理":
// a second-level FP32 scale over the whole tensor).
//
// Design (one persistent CTA per SM, 14 warps; large M runs on the CTA-pair
// kernel of gemm2sm.cu instead):
//   warp 0      TMA producer: for every 256-element K slab, a 128-row tile of
//               the MMA's A operand and a BN-row tile of its B operand (packed
//               E2M1, 128-byte swizzle) plus their 512-byte scale atoms (bulk
//               copies) into a STAGES-deep shared-memory ring (mbarriers).
//   warp 1      TMEM allocator and MMA issuer: tcgen05.mma kind::mxf4nvf4
//               (M=128, N=BN, K=64) into an fp32 accumulator in tensor memory;
//               a stage is released by tcgen05.commit when its MMAs are done.
//   warps 2..5  scale warps: each copies the stage's scale atoms from shared
//               memory into its own 32-lane quarter of tensor memory with
//               tcgen05.st (the four quarters hold the same scales, which is the
//               replicated layout the block-scaled MMA reads), into a TMEM scale
//               slot owned by the stage, handing stages to the MMA two at a
//               time.  This keeps scale movement off the tensor pipe, where a
//               tcgen05.cp per 512-byte atom would cost about as much
//               tensor-pipe time as the MMAs themselves.
//   warps 6..13 epilogue, two warps per TMEM lane quarter, each owning half
//               of the tile's columns (bf16 output, tiles >= 64 wide):
//               tcgen05.ld of the accumulator with the next chunk in flight,
//               y = acc * (gA*gB), RNE to bf16, store; the accumulator is
//               released to the MMA warp as soon as both halves are read.
// Small M (decode) runs "swapped": the weights ride the MMA's M = 128 and the
// few activation rows ride N = BN, so the weight stream spreads over all SMs.
// When the output tiles would leave at least half of the SMs idle, CTAs take
// equal runs of (tile, K slab) units instead of whole tiles (stream-K): partial
// tiles are added in fp32 in the workspace and the CTA that completes a
// tile's K range writes it.  That launch is cooperative: the epilogue warps
// zero-fill the CTA's share of the partial-sum buffer and its counters and
// meet the grid once before the first partial sum lands, while the first
// work item's loads and MMAs run.
// When the weights are known not to come from the kernel launched just before
// (inside nvfp4_linear_fused), the producer starts streaming them before the
// programmatic-dependent-launch wait, hiding the pipeline fill behind the
// activation quantizer.
// Every wait is bounded; a timeout sets the status word and winds the CTA
// down without leaving tensor memory allocated.
#include <atomic>
#include <cstdlib>
#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace nvfp4 {

struct GemmArgs {
    const uint8_t *sfa;      // tiled scales of the MMA A operand (P rows)
    const uint8_t *sfb;      // tiled scales of the MMA B operand (Q rows)
    const float *ga;         // tensor scales (null for MXFP4 operands, which have none)
    const float *gb;
    void *y;
    int64_t ldy;
    int32_t P, Q;            // rows of the A and B operands
    int32_t num_k_steps;     // K / 64
    int32_t num_p_tiles, num_q_tiles;
    int32_t q_row_tiles;     // ceil(Q / 128): 128-row scale tiles of B
    int32_t preload;         // stages of the weight operand loaded before the PDL wait
    int32_t weights_are_a;   // 1: the weights are the MMA A operand (swapped)
    int32_t streamk;         // 1: CTAs take equal contiguous runs of (tile, K slab) units
    int32_t q_pad;           // row pitch (floats) of acc_ws: num_q_tiles * BN
    float *acc_ws;           // stream-K: fp32 partial sums [num_p_tiles*128][q_pad], zeroed in-kernel
    int32_t *tile_cnt;       // stream-K: K slabs added per tile so far (follows acc_ws), zeroed in-kernel
    int64_t zero_words;      // stream-K: 32-bit words from acc_ws that the grid zero-fills
    uint32_t *grid_bar;      // stream-K: grid meeting point (the workspace header's)
    float *ymax_part;        // if set: this CTA's largest |y| as stored, at [blockIdx.x]
    uint32_t *status;
    uint64_t timeout_ns;
};

// One CTA's work item: K slabs [ks0, ks1) of one output tile.
struct Seg {
    int tile, ks0, ks1;
};

// The sequence of work items of this CTA; every role walks the same sequence.
// Tile mode: whole tiles blockIdx.x, blockIdx.x + gridDim.x, ...  Stream-K
// mode: the CTA's equal share of the tiles x K-slabs units, in tile-major
// order, cut at tile boundaries (at most a partial first and last tile).
struct SegIter {
    int64_t u, end;
    int nks, tile, tstep, ntiles;
    bool sk;
    __device__ SegIter(const GemmArgs &a, int num_tiles, int num_kstages)
        : u(0), end(0), nks(num_kstages), tile(static_cast<int>(blockIdx.x)), tstep(static_cast<int>(gridDim.x)),
          ntiles(num_tiles), sk(a.streamk != 0) {
        if (sk) {
            const int64_t T = static_cast<int64_t>(num_tiles) * num_kstages;
            u = T * blockIdx.x / gridDim.x;
            end = T * (blockIdx.x + 1) / gridDim.x;
        }
    }
    __device__ bool next(Seg &s) {
        if (sk) {
            if (u >= end) return false;
            s.tile = static_cast<int>(u / nks);
            s.ks0 = static_cast<int>(u % nks);
            s.ks1 = static_cast<int>(min(static_cast<int64_t>(nks), s.ks0 + (end - u)));
            u += s.ks1 - s.ks0;
            return true;
        }
        if (tile >= ntiles) return false;
        s.tile = tile;
        s.ks0 = 0;
        s.ks1 = nks;
        tile += tstep;
        return true;
    }
};

// NACC accumulators per tile: K step j of a stage accumulates into
// accumulator j % NACC, so that consecutive MMAs do not wait for one another
// (with few output columns an MMA takes far less time than the latency of the
// previous one into the same accumulator); the epilogue adds them in order.
template <int BN, int NACC = 1>
struct GemmCfg {
    static constexpr int kNQT = (BN + 127) / 128;              // 128-row scale tiles per B tile
    static constexpr int kAStage = 128 * 128;                  // bytes of A per stage
    static constexpr int kBStage = BN * 128;
    static constexpr int kSfaStage = 4 * 512;                  // 4 K-steps x one 512 B atom
    static constexpr int kSfbStage = kNQT * 4 * 512;
    static constexpr int kStageBytes = kAStage + kBStage + kSfaStage + kSfbStage;
    static constexpr int kStages = (BN == 256) ? 4 : (BN == 128 ? 6 : (BN == 64 ? 7 : 8));
    static constexpr int kSfCols = 16 + 16 * kNQT;             // TMEM scale columns per stage
    static constexpr int kAccCols = NACC * BN;                 // columns of one tile's accumulators
    static constexpr int kAccStages = (2 * kAccCols + kStages * kSfCols <= 512) ? 2 : 1;
    static constexpr int kSfBase = kAccStages * kAccCols;      // first scale column
    static constexpr int kColsUsed = kSfBase + kStages * kSfCols;
    static constexpr int kTmemCols = kColsUsed <= 32 ? 32 : kColsUsed <= 64 ? 64 : kColsUsed <= 128 ? 128
                                   : kColsUsed <= 256 ? 256 : 512;
    static constexpr int kBarBytes = 8 * (3 * kStages + 7) + 16;
    static constexpr int kSmemBytes = kStages * kStageBytes + kBarBytes + 1024;   // + alignment slack
    static constexpr int kThreads = 448;                       // 14 warps
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static_assert(kColsUsed <= 512, "tensor memory budget");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
    static_assert(NACC == 1 || NACC == 4, "one accumulator, or one per K step of a stage");
};

// Swapped tiles (few activation rows on the MMA's N) use four accumulators.
template <bool SWAP> constexpr int kNumAcc = SWAP ? 4 : 1;

// Accumulator columns [taddr, taddr + CH) of a tile, the NACC accumulators
// (nvalid of them written) added in order ((a0 + a1) + a2) + a3.  Warp-uniform
// nvalid (tcgen05.ld is .sync.aligned).
template <int CH, int NACC, int STRIDE>
__device__ __forceinline__ void tmem_ld_acc(uint32_t taddr, int nvalid, uint32_t (&r)[CH]) {
    auto ld = [&](uint32_t a, uint32_t (&dst)[CH]) {
        if constexpr (CH == 32) tmem_ld_32x32b_x32(a, reinterpret_cast<uint32_t(&)[32]>(dst));
        else tmem_ld_32x32b_x16(a, reinterpret_cast<uint32_t(&)[16]>(dst));
    };
    ld(taddr, r);
    tmem_ld_wait();
#pragma unroll
    for (int s = 1; s < NACC; ++s) {
        if (s < nvalid) {
            uint32_t t[CH];
            ld(taddr + s * STRIDE, t);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < CH; ++i) r[i] = __float_as_uint(__fadd_rn(__uint_as_float(r[i]), __uint_as_float(t[i])));
        }
    }
}

// Scale atoms (512 bytes: 128 rows x 4 blocks) per ring stage and per 128-row
// tile.  A stage is four MMA K steps: 256 values of K for the FP4 kinds, 128
// for W4A8, and always 128 bytes per operand row in shared memory.  NVFP4 has
// one atom per K step (4 blocks of 16), MXFP4 one per two (4 blocks of 32),
// W4A8 one per four.
template <int FMT> struct ScaleFmt {
    static constexpr int kAtomsPerStage = FMT == kFmtNV ? 4 : (FMT == kFmtMX ? 2 : 1);
    static constexpr int kStepsPerAtom = 4 / kAtomsPerStage;              // MMA K steps one atom covers
    __host__ __device__ static int atoms_per_row_tile(int k_steps) { return (k_steps + kStepsPerAtom - 1) / kStepsPerAtom; }
    __host__ __device__ static int stage_atoms(int nk) { return (nk + kStepsPerAtom - 1) / kStepsPerAtom; }
};

// The block-scaled MMAs of K step j of a stage.  NVFP4 reads the stage's
// scale columns 4j (A) and 4*NQT*j past the A columns (B); MXFP4 reads the
// columns of atom j/2 and picks their bytes {0,1} or {2,3} by the
// descriptor; W4A8 reads atom 0's columns and picks byte j.
template <int FMT, int BN, int NQT, bool SWAP>
__device__ __forceinline__ void mma_kstep(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t sf, int j,
                                          uint32_t acc, uint32_t issue) {
    if constexpr (FMT == kFmtW4A8) {
        // the weights are E2M1 (format 5), the activations E4M3 (format 0)
        constexpr uint32_t fa = SWAP ? 5u : 0u, fb = SWAP ? 0u : 5u;
        const uint32_t idesc = make_idesc_mxf8f6f4(BN, fa, fb, static_cast<uint32_t>(j));
        mma_mxf8f6f4(d_tmem, adesc + 2 * j, bdesc + 2 * j, idesc, sf, sf + 16, acc, issue);
    } else if constexpr (FMT == kFmtMX) {
        const uint32_t idesc = (j & 1) ? make_idesc_mxf4(BN, 128, 1) : make_idesc_mxf4(BN, 128, 0);
        mma_mxf4(d_tmem, adesc + 2 * j, bdesc + 2 * j, idesc, sf + 4 * (j >> 1), sf + 16 + 4 * NQT * (j >> 1), acc,
                 issue);
    } else {
        mma_nvf4(d_tmem, adesc + 2 * j, bdesc + 2 * j, make_idesc_nvf4(BN), sf + 4 * j, sf + 16 + 4 * NQT * j, acc,
                 issue);
    }
}

template <int BN, bool SWAP, typename OutT, int FMT>
__global__ void __launch_bounds__(448, 1)
gemm_nvf4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ GemmArgs args) {
    constexpr int NACC = kNumAcc<SWAP>;
    using C = GemmCfg<BN, NACC>;
    using F = ScaleFmt<FMT>;
    constexpr int STAGES = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = sA + STAGES * C::kAStage;
    uint8_t *sSfa = sB + STAGES * C::kBStage;
    uint8_t *sSfb = sSfa + STAGES * C::kSfaStage;
    uint64_t *full = reinterpret_cast<uint64_t *>(sSfb + STAGES * C::kSfbStage);
    uint64_t *sf_full = full + STAGES;
    uint64_t *empty = sf_full + STAGES;
    uint64_t *tfull = empty + STAGES;
    uint64_t *tempty = tfull + 2;
    uint64_t *epi_done = tempty + 2;                    // stream-K: epilogue warps' partial sums added
    uint64_t *epi_flag = epi_done + 1;                  // stream-K: last_flag published
    uint64_t *mma_done = epi_flag + 1;                  // every MMA of this CTA has completed
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile uint32_t *abort_flag = tmem_holder + 1;
    volatile uint32_t *last_flag = tmem_holder + 2;     // stream-K: this CTA completes the tile
    __shared__ float s_ymax[8];                         // epilogue warps' largest |stored y|

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&sf_full[s], 4);     // one arrive per scale warp
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&tfull[s], 1);
            mbar_init(&tempty[s], 8);      // one arrive per epilogue warp
        }
        mbar_init(epi_done, 8);
        mbar_init(epi_flag, 1);
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
    // Bytes the operand copies of one stage signal on its barrier.  The
    // unpacking copy of the W4A8 weights counts the packed bytes it reads
    // (64 per row), not the 128 it writes.
    constexpr uint32_t kOperandTxBytes =
        FMT != kFmtW4A8 ? C::kAStage + C::kBStage : (SWAP ? C::kAStage / 2 + C::kBStage : C::kAStage + C::kBStage / 2);

    if (warp == 0) {
        {
            // -------------------------------------------------------- producer
            // The whole warp walks the loop (its waits are warp-uniform); one
            // elected lane issues the copies.
            const bool issue = elect_one_sync();
            const uint64_t pol_a = SWAP ? policy_evict_first() : policy_evict_normal();
            const uint64_t pol_b = SWAP ? policy_evict_last() : policy_evict_normal();
            // The weights may be streamed before the dependent-launch wait for
            // the first `pre` stages of this CTA's first work item.
            Seg first{0, 0, 0};
            const bool has_first = SegIter(args, num_tiles, num_kstages).next(first);
            const int pre = has_first ? min(args.preload, min(STAGES, first.ks1 - first.ks0)) : 0;
            const int pt0 = first.tile % args.num_p_tiles;
            const int qt0 = first.tile / args.num_p_tiles;
            const int atoms_rt = F::atoms_per_row_tile(args.num_k_steps);
            auto load_a = [&](uint32_t st, int pt, int ks, int nk) {
                tma_load_2d(sA + st * C::kAStage, &tmA, &full[st], ks * 128, pt * 128, pol_a);
                bulk_load(sSfa + st * C::kSfaStage,
                          args.sfa + (static_cast<int64_t>(pt) * atoms_rt + F::kAtomsPerStage * ks) * 512,
                          F::stage_atoms(nk) * 512, &full[st], pol_a);
            };
            auto load_b = [&](uint32_t st, int qt, int ks, int nk) {
                tma_load_2d(sB + st * C::kBStage, &tmB, &full[st], ks * 128, qt * BN, pol_b);
                for (int q = 0; q < C::kNQT; ++q) {
                    const int rt = qt * C::kNQT + q;
                    if (rt < args.q_row_tiles)
                        bulk_load(sSfb + st * C::kSfbStage + q * 2048,
                                  args.sfb + (static_cast<int64_t>(rt) * atoms_rt + F::kAtomsPerStage * ks) * 512,
                                  F::stage_atoms(nk) * 512, &full[st], pol_b);
                }
            };
            bool waited = (pre == 0);
            if (waited) asm volatile("griddepcontrol.wait;" ::: "memory");
            // after the wait: the dependent operand of the preloaded stages
            // (stages 0..pre-1 = K slabs first.ks0 .. first.ks0+pre-1)
            auto finish_preload = [&]() {
                asm volatile("griddepcontrol.wait;" ::: "memory");
                waited = true;
                for (int p = 0; p < pre && issue; ++p) {
                    const int ks = first.ks0 + p;
                    const int nk = min(4, args.num_k_steps - 4 * ks);
                    if (args.weights_are_a) load_b(static_cast<uint32_t>(p), qt0, ks, nk);
                    else load_a(static_cast<uint32_t>(p), pt0, ks, nk);
                }
                __syncwarp();
            };
            uint32_t stage = 0, phase = 0;
            int it = 0;   // stage index within this CTA's work
            SegIter segs(args, num_tiles, num_kstages);
            Seg sg;
            bool ok = true;
            while (ok && segs.next(sg)) {
                const int pt = sg.tile % args.num_p_tiles;
                const int qt = sg.tile / args.num_p_tiles;
                int nq_loaded = 0;
                for (int q = 0; q < C::kNQT; ++q) nq_loaded += (qt * C::kNQT + q < args.q_row_tiles);
                for (int ks = sg.ks0; ks < sg.ks1; ++ks, ++it) {
                    const int nk = min(4, args.num_k_steps - 4 * ks);
                    const uint32_t bytes = kOperandTxBytes + F::stage_atoms(nk) * 512 * (1 + nq_loaded);
                    if (it < pre) {
                        // fresh stage (first pass over the ring): no empty wait needed
                        if (issue) {
                            mbar_arrive_expect_tx(&full[stage], bytes);
                            if (args.weights_are_a) load_a(stage, pt, ks, nk);
                            else load_b(stage, qt, ks, nk);
                        }
                    } else {
                        if (!waited) finish_preload();
                        if (!__all_sync(0xffffffffu, mbar_wait(&empty[stage], phase ^ 1u, args.timeout_ns,
                                                               abort_flag, args.status))) {
                            ok = false;
                            break;
                        }
                        if (issue) {
                            mbar_arrive_expect_tx(&full[stage], bytes);
                            load_a(stage, pt, ks, nk);
                            load_b(stage, qt, ks, nk);
                        }
                    }
                    __syncwarp();
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!waited) finish_preload();   // everything fit in the preload
            // No copy may still be landing when the CTA exits: wait (bounded,
            // also after an abort) for the last load issued into every stage.
            // On the normal path the MMA thread has consumed them all already.
            volatile uint32_t keep_waiting = 0u;
            for (int j = it > STAGES ? it - STAGES : 0; j < it; ++j)
                mbar_wait(&full[j % STAGES], static_cast<uint32_t>(j / STAGES) & 1u, args.timeout_ns,
                          &keep_waiting, args.status);
        }
    } else if (warp == 1) {
        {
            // -------------------------------------------------------- MMA issuer
            // The whole warp walks the loop; one elected lane issues the MMAs
            // and commits.
            const uint32_t issue = elect_one_sync() ? 1u : 0u;
            const uint32_t a_base = smem_addr(sA), b_base = smem_addr(sB);
            uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
            SegIter segs(args, num_tiles, num_kstages);
            Seg sg;
            while (segs.next(sg)) {
                if (!__all_sync(0xffffffffu, mbar_wait(&tempty[acc], acc_phase ^ 1u, args.timeout_ns, abort_flag,
                                                       args.status)))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * C::kAccCols;
                bool ok = true;
                for (int ks = sg.ks0; ks < sg.ks1; ++ks) {
                    if (!__all_sync(0xffffffffu,
                                    mbar_wait(&full[stage], phase, args.timeout_ns, abort_flag, args.status) &&
                                    mbar_wait(&sf_full[stage], phase, args.timeout_ns, abort_flag, args.status))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nk = min(4, args.num_k_steps - 4 * ks);
                    const uint32_t sf = tmem_base + C::kSfBase + stage * C::kSfCols;
                    // K-step j: +32 bytes = +2 in the descriptors' address field
                    const uint64_t adesc = make_operand_desc(a_base + stage * C::kAStage);
                    const uint64_t bdesc = make_operand_desc(b_base + stage * C::kBStage);
                    const uint32_t acc0 = ks != sg.ks0 ? 1u : 0u;
                    // K step j -> accumulator j % NACC; its first MMA of the
                    // tile overwrites it
                    auto accf = [&](int j) -> uint32_t { return NACC == 1 ? ((acc0 | j) != 0 ? 1u : 0u) : acc0; };
                    if (nk == 4) {
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            mma_kstep<FMT, BN, C::kNQT, SWAP>(d_tmem + (j % NACC) * BN, adesc, bdesc, sf, j, accf(j), issue);
                    } else {
                        for (int j = 0; j < nk; ++j)
                            mma_kstep<FMT, BN, C::kNQT, SWAP>(d_tmem + (j % NACC) * BN, adesc, bdesc, sf, j, accf(j), issue);
                    }
                    tc_commit(&empty[stage], issue);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit(&tfull[acc], issue);
                if (C::kAccStages == 2) {
                    acc ^= 1u;
                    if (acc == 0) acc_phase ^= 1u;
                } else {
                    acc_phase ^= 1u;
                }
            }
            // Tensor memory is freed below: first let every MMA this warp
            // issued complete (bounded, also after an abort).
            tc_commit(mma_done, issue);
            volatile uint32_t keep_waiting = 0u;
            mbar_wait(mma_done, 0, args.timeout_ns, &keep_waiting, args.status);
        }
    } else if (warp < 6) {
        // ------------------------------------------------------------ scale warps
        // Lane l of every quarter receives the 16 bytes at l*16 of each 512-byte
        // atom: columns c = 0..3 hold rows 32c + l, bytes = the 4 K-blocks.
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
        SegIter segs(args, num_tiles, num_kstages);
        Seg sg;
        while (segs.next(sg)) {
            bool ok = true;
            for (int ks = sg.ks0; ks < sg.ks1; ++ks) {
                const bool got = mbar_wait(&full[stage], phase, args.timeout_ns, abort_flag, args.status);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                const int nk = min(4, args.num_k_steps - 4 * ks);
                const uint32_t sf = tmem_base + lane_off + C::kSfBase + stage * C::kSfCols;
                const uint8_t *a_src = sSfa + stage * C::kSfaStage + lane * 16;
                const uint8_t *b_src = sSfb + stage * C::kSfbStage + lane * 16;
                // one 16-column store for A's scales and one 16*kNQT-column
                // store for B's per stage (columns of K-steps a partial last
                // stage does not have, and for MXFP4 the two atom slots a stage
                // does not use, hold stale bytes that are never read)
                uint32_t av[16], bv[16 * C::kNQT];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 a = ld_shared_v4(a_src + j * 512);
                    av[4 * j] = a.x; av[4 * j + 1] = a.y; av[4 * j + 2] = a.z; av[4 * j + 3] = a.w;
#pragma unroll
                    for (int q = 0; q < C::kNQT; ++q) {
                        const uint4 b = ld_shared_v4(b_src + q * 2048 + j * 512);
                        const int o = 4 * (j * C::kNQT + q);
                        bv[o] = b.x; bv[o + 1] = b.y; bv[o + 2] = b.z; bv[o + 3] = b.w;
                    }
                }
                (void)nk;
                tmem_st_32x32b_x16(sf, av);
                if constexpr (C::kNQT == 1)
                    tmem_st_32x32b_x16(sf + 16, reinterpret_cast<uint32_t(&)[16]>(bv));
                else
                    tmem_st_32x32b_x32(sf + 16, reinterpret_cast<uint32_t(&)[32]>(bv));
                // Hand stages over two at a time: one store-completion wait and
                // handshake per pair keeps the MMA fed (one per stage left the
                // tensor pipe waiting on the handshake's latency).
                pend[npend++] = stage;
                if (npend == 2) flush();
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
        }
        flush();
    } else {
        // ------------------------------------------------------------ epilogue
        asm volatile("griddepcontrol.wait;" ::: "memory");   // tensor scales may be fresh
        const int quarter = warp & 3;               // TMEM lane quarter this warp may read
        const int half = (warp - 6) >> 2;           // column half of the tile (fast drain)
        const int row = quarter * 32 + lane;        // accumulator row (MMA M index)
        const float alpha = __fmul_rn(args.ga ? *args.ga : 1.0f, args.gb ? *args.gb : 1.0f);   // MXFP4: none
        constexpr bool kFastDrain = !SWAP && sizeof(OutT) == 2 && BN >= 64;
        // debug-build store checks: y is [M][N] with pitch ldy (M = Q when swapped)
        const size_t y_bytes = matrix_extent(SWAP ? args.Q : args.P, SWAP ? args.P : args.Q, args.ldy, sizeof(OutT));
        const size_t acc_bytes = static_cast<size_t>(args.num_p_tiles) * 128 * args.q_pad * sizeof(float);
        auto y_ok = [&](const void *ptr, size_t bytes) { return store_ok(ptr, bytes, args.y, y_bytes, args.status); };
        uint32_t acc = 0, acc_phase = 0;
        uint32_t npart = 0;      // partial (stream-K) work items so far: epi_done/epi_flag phase
        if (args.streamk) {
            // Zero-fill this CTA's share of the partial sums and counters (a
            // previous call may have left anything there; the dependent-launch
            // wait above covers a previous kernel still using them), then meet
            // the grid: no partial sum is added before every share is zero.
            const uint32_t meet_gen = (warp == 6 && lane == 0) ? grid_meet_generation(args.grid_bar) : 0u;
            const int64_t per = (args.zero_words / 4 + gridDim.x - 1) / gridDim.x;      // uint4 per CTA
            uint4 *zb = reinterpret_cast<uint4 *>(args.acc_ws);
            const int64_t lo = per * blockIdx.x, hi = min(per * (blockIdx.x + 1), args.zero_words / 4);
            for (int64_t i = lo + (threadIdx.x - 6 * 32); i < hi; i += 8 * 32)
                if (store_ok(zb + i, 16, args.acc_ws, static_cast<size_t>(args.zero_words) * 4, args.status))
                    zb[i] = make_uint4(0u, 0u, 0u, 0u);
            __threadfence();
            asm volatile("bar.sync 1, 256;" ::: "memory");             // the 8 epilogue warps
            if (warp == 6) {
                uint32_t go = 0u;
                if (lane == 0) go = grid_meet(args.grid_bar, meet_gen, args.timeout_ns, abort_flag, args.status) ? 1u : 0u;
                go = __shfl_sync(0xffffffffu, go, 0);
                if (lane == 0 && !go) *abort_flag = 1u;
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
        }
        // Largest |y| this thread stores.  Accumulator rows and columns past P
        // and Q are exact zeros (their operand rows are zero-filled by the
        // loads), so folding a whole computed chunk cannot raise it.
        YMax ym;
        SegIter segs(args, num_tiles, num_kstages);
        Seg sg;
        while (segs.next(sg)) {
            const int pt = sg.tile % args.num_p_tiles;
            const int qt = sg.tile / args.num_p_tiles;
            // The decision must be warp-uniform: tcgen05.ld below is .sync.aligned.
            const bool ok = mbar_wait(&tfull[acc], acc_phase, args.timeout_ns, abort_flag, args.status);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const int p = pt * 128 + row;
            const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * C::kAccCols;
            // accumulators this work item wrote: one per K step it has, at most NACC
            const int nvalid = min(NACC, min(4 * sg.ks1, args.num_k_steps) - 4 * sg.ks0);
            // (stream-K is never chosen for 256-wide tiles; keep that path out of them)
            const bool partial = BN <= 128 && (sg.ks0 != 0 || sg.ks1 != num_kstages);
            if (partial) {
                // ---- stream-K: part of the tile's K range.  Add the partial
                // sums into acc_ws (zero-filled by the launcher); the CTA that
                // brings the tile's slab count to num_kstages scales, converts
                // and stores it.
                constexpr int WC = BN >= 64 ? BN / 2 : BN;          // columns per warp
                constexpr int CH = WC < 32 ? WC : 32;
                const int c0 = BN >= 64 ? half * WC : 0;
                if (BN >= 64 || half == 0) {
                    float *accrow = args.acc_ws + static_cast<int64_t>(p) * args.q_pad + qt * BN + c0;
#pragma unroll
                    for (int c = 0; c < WC / CH; ++c) {
                        uint32_t r[CH];
                        tmem_ld_acc<CH, NACC, BN>(tbase + c0 + c * CH, nvalid, r);
#pragma unroll
                        for (int i = 0; i < CH; i += 4)
                            if (store_ok(accrow + c * CH + i, 16, args.acc_ws, acc_bytes, args.status))
                                red_add_v4_f32(accrow + c * CH + i, __uint_as_float(r[i]), __uint_as_float(r[i + 1]),
                                               __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[acc]);
                __threadfence();                                 // this thread's adds before the count
                __syncwarp();
                if (lane == 0) mbar_arrive(epi_done);
                // Warp 6 (all lanes, so that no warp spins on two barriers at
                // once) waits until the 8 epilogue warps have added, counts
                // this CTA's slabs and publishes whether it completed the tile.
                bool is_last;
                if (warp == 6) {
                    const bool done_ok = mbar_wait(epi_done, npart & 1u, args.timeout_ns, abort_flag, args.status);
                    uint32_t last = 0u;
                    if (lane == 0 && done_ok) {
                        const int add = sg.ks1 - sg.ks0;
                        const int before = atomicAdd(&args.tile_cnt[sg.tile], add);
                        last = (before + add == num_kstages) ? 1u : 0u;
                    }
                    last = __shfl_sync(0xffffffffu, last, 0);
                    if (lane == 0) {
                        *last_flag = last;
                        mbar_arrive(epi_flag);
                    }
                    is_last = last != 0u;
                } else {
                    const bool flag_ok = mbar_wait(epi_flag, npart & 1u, args.timeout_ns, abort_flag, args.status);
                    is_last = flag_ok && *last_flag != 0u;
                }
                ++npart;
                if (is_last) {
                    // Coalesced: a warp covers contiguous output, so that each
                    // store instruction writes whole sectors.
                    __threadfence();
                    const int ew = warp - 6;                       // 0..7
                    OutT *y = static_cast<OutT *>(args.y);
                    float *tile_acc = args.acc_ws + static_cast<int64_t>(pt) * 128 * args.q_pad + qt * BN;
                    if constexpr (!SWAP) {
                        // y[p][q] (BN = 128 here): warp ew takes rows ew, ew + 8, ...,
                        // lane l columns 4l..4l+3.  All loads are issued before
                        // any is used (the finalize is on the kernel's tail).
                        constexpr int RPW = 128 / 8;
                        float4 f[RPW];
#pragma unroll
                        for (int i = 0; i < RPW; ++i)
                            f[i] = __ldcg(reinterpret_cast<const float4 *>(
                                tile_acc + static_cast<int64_t>(ew + 8 * i) * args.q_pad + lane * 4));
#pragma unroll
                        for (int i = 0; i < RPW; ++i) {
                            const int rr = ew + 8 * i;
                            const int pr = pt * 128 + rr;
                            const float v0 = __fmul_rn(f[i].x, alpha), v1 = __fmul_rn(f[i].y, alpha);
                            const float v2 = __fmul_rn(f[i].z, alpha), v3 = __fmul_rn(f[i].w, alpha);
                            const int q = qt * BN + lane * 4;
                            if (pr < args.P && lane * 4 < BN) {
                                OutT *dst = y + static_cast<int64_t>(pr) * args.ldy + q;
                                if (q + 4 <= args.Q && y_ok(dst, 4 * sizeof(OutT))) {
                                    if constexpr (sizeof(OutT) == 2) {
                                        __nv_bfloat162 lo = __floats2bfloat162_rn(v0, v1);
                                        __nv_bfloat162 hi = __floats2bfloat162_rn(v2, v3);
                                        *reinterpret_cast<uint2 *>(dst) =
                                            make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
                                        ym.bf16x2(*reinterpret_cast<uint32_t *>(&lo));
                                        ym.bf16x2(*reinterpret_cast<uint32_t *>(&hi));
                                    } else {
                                        *reinterpret_cast<float4 *>(dst) = make_float4(v0, v1, v2, v3);
                                        ym.f32(v0); ym.f32(v1); ym.f32(v2); ym.f32(v3);
                                    }
                                } else if (q + 4 > args.Q) {
                                    const float vv[4] = {v0, v1, v2, v3};
#pragma unroll
                                    for (int k = 0; k < 4; ++k)
                                        if (q + k < args.Q && y_ok(dst + k, sizeof(OutT))) {
                                            const OutT o = to_out<OutT>(vv[k]);
                                            dst[k] = o;
                                            ym.add<OutT>(o);
                                        }
                                }
                            }
                        }
                    } else {
                        // y[q][p]: warp ew takes columns q = ew, ew + 8, ...; lanes
                        // run along p (rows lane, lane + 32, ...).  Loads first.
                        constexpr int QPW = BN / 8;
                        float v[QPW][4];
#pragma unroll
                        for (int j = 0; j < QPW; ++j)
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                v[j][i] = __ldcg(tile_acc + static_cast<int64_t>(lane + 32 * i) * args.q_pad + ew + 8 * j);
#pragma unroll
                        for (int j = 0; j < QPW; ++j) {
                            const int q = qt * BN + ew + 8 * j;
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int rr = lane + 32 * i;
                                const int pr = pt * 128 + rr;
                                const float o = __fmul_rn(v[j][i], alpha);
                                if (pr < args.P && q < args.Q && y_ok(y + static_cast<int64_t>(q) * args.ldy + pr, sizeof(OutT))) {
                                    const OutT oo = to_out<OutT>(o);
                                    y[static_cast<int64_t>(q) * args.ldy + pr] = oo;
                                    ym.add<OutT>(oo);
                                }
                            }
                        }
                    }
                }
            } else if constexpr (kFastDrain) {
                // each warp drains and stores its half of the columns, the next
                // 32-column chunk in flight while the current one is stored
                constexpr int HC = BN / 2;
                constexpr int NCH = HC / 32;
                uint32_t r[2][32];
                const uint32_t tb = tbase + half * HC;
                tmem_ld_32x32b_x32(tb, r[0]);
                tmem_ld_wait();
                OutT *yrow = static_cast<OutT *>(args.y) + static_cast<int64_t>(p) * args.ldy;
#pragma unroll
                for (int c = 0; c < NCH; ++c) {
                    if (c + 1 < NCH) tmem_ld_32x32b_x32(tb + (c + 1) * 32, r[(c + 1) & 1]);
                    uint32_t pk[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(r[c & 1][2 * k]), alpha),
                                                                  __fmul_rn(__uint_as_float(r[c & 1][2 * k + 1]), alpha));
                        pk[k] = *reinterpret_cast<uint32_t *>(&b2);
                        ym.bf16x2(pk[k]);
                    }
                    const int q0 = qt * BN + half * HC + c * 32;
                    if (p < args.P) {
                        if (q0 + 32 <= args.Q) {
                            if (y_ok(yrow + q0, 32 * sizeof(OutT))) {
#pragma unroll
                                for (int i = 0; i < 4; ++i)
                                    *reinterpret_cast<uint4 *>(yrow + q0 + 8 * i) =
                                        make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                if (q0 + 2 * i < args.Q && y_ok(yrow + q0 + 2 * i, 2))
                                    reinterpret_cast<unsigned short *>(yrow)[q0 + 2 * i] = static_cast<unsigned short>(pk[i] & 0xffffu);
                                if (q0 + 2 * i + 1 < args.Q && y_ok(yrow + q0 + 2 * i + 1, 2))
                                    reinterpret_cast<unsigned short *>(yrow)[q0 + 2 * i + 1] = static_cast<unsigned short>(pk[i] >> 16);
                            }
                        }
                    }
                    if (c + 1 < NCH) tmem_ld_wait();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[acc]);
            } else {
                if (half == 0) {
                    constexpr int CH = BN < 32 ? BN : 32;
                    constexpr int NCH = BN / CH;
                    uint32_t r[2][CH];
                    auto ld = [&](int c, uint32_t (&dst)[CH]) {
                        if constexpr (CH == 32)
                            tmem_ld_32x32b_x32(tbase + c * CH, reinterpret_cast<uint32_t(&)[32]>(dst));
                        else
                            tmem_ld_32x32b_x16(tbase + c * CH, reinterpret_cast<uint32_t(&)[16]>(dst));
                    };
                    if constexpr (NACC == 1) {
                        ld(0, r[0]);
                        tmem_ld_wait();
                    }
#pragma unroll
                    for (int c = 0; c < NCH; ++c) {
                        if constexpr (NACC > 1)
                            tmem_ld_acc<CH, NACC, BN>(tbase + c * CH, nvalid, r[c & 1]);   // summed, not prefetched
                        else if (c + 1 < NCH)
                            ld(c + 1, r[(c + 1) & 1]);       // next chunk in flight
                        float v[CH];
#pragma unroll
                        for (int i = 0; i < CH; ++i) v[i] = __fmul_rn(__uint_as_float(r[c & 1][i]), alpha);
#pragma unroll
                        for (int i = 0; i < CH; ++i) ym.add<OutT>(to_out<OutT>(v[i]));
                        const int q0 = qt * BN + c * CH;
                        if constexpr (SWAP) {
                            // y[q][p]: for each i the warp writes 32 consecutive p
                            if (p < args.P) {
                                OutT *y = static_cast<OutT *>(args.y);
#pragma unroll
                                for (int i = 0; i < CH; ++i) {
                                    const int q = q0 + i;
                                    if (q < args.Q && y_ok(y + static_cast<int64_t>(q) * args.ldy + p, sizeof(OutT))) {
                                        if constexpr (sizeof(OutT) == 2)
                                            y[static_cast<int64_t>(q) * args.ldy + p] = __float2bfloat16_rn(v[i]);
                                        else
                                            y[static_cast<int64_t>(q) * args.ldy + p] = v[i];
                                    }
                                }
                            }
                        } else {
                            // y[p][q0 .. q0+CH): one contiguous run per thread
                            if (p < args.P) {
                                OutT *yrow = static_cast<OutT *>(args.y) + static_cast<int64_t>(p) * args.ldy;
                                if (q0 + CH <= args.Q && y_ok(yrow + q0, CH * sizeof(OutT))) {
                                    if constexpr (sizeof(OutT) == 2) {
#pragma unroll
                                        for (int i = 0; i < CH; i += 8) {
                                            uint4 pk;
                                            uint32_t *w = reinterpret_cast<uint32_t *>(&pk);
#pragma unroll
                                            for (int k = 0; k < 4; ++k) {
                                                __nv_bfloat162 b2 = __floats2bfloat162_rn(v[i + 2 * k], v[i + 2 * k + 1]);
                                                w[k] = *reinterpret_cast<uint32_t *>(&b2);
                                            }
                                            *reinterpret_cast<uint4 *>(yrow + q0 + i) = pk;
                                        }
                                    } else {
#pragma unroll
                                        for (int i = 0; i < CH; i += 4)
                                            *reinterpret_cast<float4 *>(yrow + q0 + i) =
                                                make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
                                    }
                                } else if (q0 + CH > args.Q) {
#pragma unroll
                                    for (int i = 0; i < CH; ++i) {
                                        if (q0 + i < args.Q && y_ok(yrow + q0 + i, sizeof(OutT))) {
                                            if constexpr (sizeof(OutT) == 2)
                                                yrow[q0 + i] = __float2bfloat16_rn(v[i]);
                                            else
                                                yrow[q0 + i] = v[i];
                                        }
                                    }
                                }
                            }
                        }
                        if (NACC == 1 && c + 1 < NCH) tmem_ld_wait();
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[acc]);
            }
            if (C::kAccStages == 2) {
                acc ^= 1u;
                if (acc == 0) acc_phase ^= 1u;
            } else {
                acc_phase ^= 1u;
            }
        }
        float m = ym.value();
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) s_ymax[warp - 6] = m;
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && args.ymax_part != nullptr) {
        float m = 0.0f;
#pragma unroll
        for (int k = 0; k < 8; ++k) m = fmaxf(m, s_ymax[k]);
        args.ymax_part[blockIdx.x] = m;
    }
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Looked up once; the initialiser of a function-local static runs exactly once
// even when several host threads make their first call at the same time.
static EncodeTiledFn get_encode_fn() {
    static const EncodeTiledFn fn = []() -> EncodeTiledFn {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(p);
        return nullptr;
    }();
    return fn;
}

CUresult encode_tensor_map_u8(CUtensorMap *map, const void *base, uint64_t inner_bytes,
                              uint64_t rows, uint32_t box_inner, uint32_t box_rows) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return CUDA_ERROR_NOT_FOUND;
    cuuint64_t dims[2] = {inner_bytes, rows};
    cuuint64_t strides[1] = {inner_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

CUresult encode_tensor_map_fp4_unpacked(CUtensorMap *map, const void *base, uint64_t k_elems, uint64_t rows,
                                        uint32_t box_rows) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return CUDA_ERROR_NOT_FOUND;
    // packed E2M1 rows of k_elems values (k_elems / 2 bytes apart); each box
    // of 128 values x box_rows rows lands as 128-byte rows in shared memory,
    // 16 values per 16-byte chunk (8 bytes of values, 8 bytes of gap), the
    // operand form of the mixed FP4 x FP8 MMA
    cuuint64_t dims[2] = {k_elems, rows};
    cuuint64_t strides[1] = {k_elems / 2};
    cuuint32_t box[2] = {128, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

CUresult encode_scale_map(CUtensorMap *map, const void *scales, uint64_t k_steps, uint64_t row_tiles,
                          uint32_t box_tiles, uint32_t box_atoms) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return CUDA_ERROR_NOT_FOUND;
    // x: 128 words of one 512-byte atom; y: atom along K within a 128-row
    // tile (k_steps of them); z: 128-row tile.  A box holds box_atoms atoms
    // of box_tiles row tiles.
    cuuint64_t dims[3] = {128, k_steps, row_tiles};
    cuuint64_t strides[2] = {512, k_steps * 512};
    cuuint32_t box[3] = {128, box_atoms, box_tiles};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void *>(scales), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

CUresult encode_output_map_bf16(CUtensorMap *map, void *y, uint64_t rows, uint64_t cols, uint64_t ld,
                                uint32_t box_cols, uint32_t box_rows) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return CUDA_ERROR_NOT_FOUND;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld * 2};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, y, dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// Stream-K scratch layout for a GEMM of M activation rows and N weight rows:
// fp32 partial sums [p_rows][q_cols] over the padded tile grid, then one int32
// counter per tile.  The path is only taken for few tiles (<= kMaxStreamKTiles).
static constexpr int64_t kMaxStreamKTiles = 1024;
struct SplitKLayout {
    int64_t p_rows, q_cols, tiles;
    size_t acc_bytes, bytes;
};
static SplitKLayout splitk_layout(int64_t M, int64_t N) {
    SplitKLayout l;
    if (M <= 64) {      // swapped: weights on the MMA's M, activations on N (BN <= 64)
        l.p_rows = round_up(N, 128);
        l.q_cols = 64;
        l.tiles = ceil_div(N, 128);
    } else {            // 128x128 tiles
        l.p_rows = round_up(M, 128);
        l.q_cols = round_up(N, 128);
        l.tiles = ceil_div(M, 128) * ceil_div(N, 128);
    }
    auto a256 = [](size_t v) { return (v + 255) & ~size_t(255); };
    l.acc_bytes = a256(static_cast<size_t>(l.p_rows * l.q_cols) * sizeof(float));
    l.bytes = (l.tiles <= kMaxStreamKTiles) ? l.acc_bytes + a256(static_cast<size_t>(l.tiles) * sizeof(int32_t)) : 0;
    return l;
}

size_t splitk_ws_bytes(int64_t M, int64_t N) { return splitk_layout(M, N).bytes; }

template <int BN, bool SWAP, typename OutT, int FMT>
static cudaError_t run_gemm(const Operand &pa, const Operand &qb, int64_t K, void *y, int64_t ldy,
                            uint32_t *status, uint64_t timeout_ns, int num_sms, int preload,
                            uint8_t *splitk_ws, const SplitKLayout &skl, float *ymax_part, int *nparts,
                            cudaStream_t stream) {
    using C = GemmCfg<BN, kNumAcc<SWAP>>;
    CUtensorMap tmA, tmB;
    if constexpr (FMT == kFmtW4A8) {
        // 128 values of K per 128-byte shared-memory row: the MXFP4 weights
        // unpacked by the copy into 8-bit containers, the E4M3 activations as
        // they are
        const Operand &w = SWAP ? pa : qb, &x = SWAP ? qb : pa;
        CUtensorMap &tw = SWAP ? tmA : tmB, &tx = SWAP ? tmB : tmA;
        if (encode_tensor_map_fp4_unpacked(&tw, w.codes, K, w.rows, SWAP ? 128 : BN) != CUDA_SUCCESS ||
            encode_tensor_map_u8(&tx, x.codes, K, x.rows, 128, SWAP ? BN : 128) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    } else {
        if (encode_tensor_map_u8(&tmA, pa.codes, K / 2, pa.rows, 128, 128) != CUDA_SUCCESS ||
            encode_tensor_map_u8(&tmB, qb.codes, K / 2, qb.rows, 128, BN) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    GemmArgs a;
    a.sfa = pa.scales;
    a.sfb = qb.scales;
    a.ga = pa.g;
    a.gb = qb.g;
    a.y = y;
    a.ldy = ldy;
    a.P = static_cast<int32_t>(pa.rows);
    a.Q = static_cast<int32_t>(qb.rows);
    a.num_k_steps = static_cast<int32_t>(FMT == kFmtW4A8 ? K / 32 : K / 64);   // MMA K steps
    a.num_p_tiles = static_cast<int32_t>(ceil_div(pa.rows, 128));
    a.num_q_tiles = static_cast<int32_t>(ceil_div(qb.rows, BN));
    a.q_row_tiles = static_cast<int32_t>(ceil_div(qb.rows, 128));
    a.preload = preload;
    a.weights_are_a = SWAP ? 1 : 0;
    a.status = status;
    a.timeout_ns = timeout_ns;
    a.ymax_part = ymax_part;
    const int tiles = a.num_p_tiles * a.num_q_tiles;
    const int64_t units = static_cast<int64_t>(tiles) * ((a.num_k_steps + 3) / 4);
    // Stream-K when the tiles alone would leave at least half of the SMs idle
    // (NVFP4_GEMM_STREAMK=0 turns it off).  Its reduction tail (partial sums
    // through L2, then the finishing CTA's pass) costs a few microseconds, so
    // with about one tile per SM the plain tile loop is faster (measured: M=8
    // and M=128 at N=17408, 136 tiles); the 40-tile MLP down projection gains
    // about 30%.
    const char *sk_opt = getenv("NVFP4_GEMM_STREAMK");
    const bool sk = BN <= 128 && splitk_ws != nullptr && skl.bytes != 0 && 2 * tiles <= num_sms &&
                    !(sk_opt != nullptr && sk_opt[0] == '0') &&
                    units >= 2 * tiles && a.num_q_tiles * BN <= skl.q_cols && a.num_p_tiles * 128 <= skl.p_rows;
    a.streamk = sk ? 1 : 0;
    a.q_pad = a.num_q_tiles * BN;
    a.acc_ws = sk ? reinterpret_cast<float *>(splitk_ws) : nullptr;
    a.tile_cnt = sk ? reinterpret_cast<int32_t *>(splitk_ws + skl.acc_bytes) : nullptr;
    // The stream-K scratch is zero-filled by the kernel itself for every call
    // (so it may share a workspace with whatever other calls left there); its
    // CTAs meet at the meeting point in the workspace header, which `status`
    // starts.
    a.zero_words = sk ? static_cast<int64_t>(skl.bytes / 4) : 0;
    a.grid_bar = sk ? reinterpret_cast<uint32_t *>(reinterpret_cast<uint8_t *>(status) + kGridBarOff) : nullptr;
    auto kern = gemm_nvf4_kernel<BN, SWAP, OutT, FMT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    const int64_t work = sk ? units : tiles;
    cfg.gridDim = dim3(static_cast<unsigned>(work < num_sms ? work : num_sms));
    if (nparts) *nparts = static_cast<int>(cfg.gridDim.x);
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (!sk) return cudaLaunchKernelEx(&cfg, kern, tmA, tmB, a);
    // stream-K: cooperative (one grid-wide meeting), and a programmatic
    // dependent of the kernel before it if the driver takes both
    static std::atomic<int> coop_pdl{1};
    if (coop_pdl.load()) {
        cfg.numAttrs = 2;
        e = cudaLaunchKernelEx(&cfg, kern, tmA, tmB, a);
        if (e == cudaSuccess) return e;
        if (e != cudaErrorInvalidValue && e != cudaErrorNotSupported) return e;
        (void)cudaGetLastError();      // a refused configuration, not a failed launch
        coop_pdl.store(0);
    }
    cfg.attrs = attr + 1;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tmA, tmB, a);
}

template <int FMT>
static cudaError_t launch_gemm_fmt(const Operand &act, const Operand &wgt, int64_t K, void *y, bool y_bf16,
                                   int64_t ldy, uint32_t *status, uint64_t timeout_ns, int num_sms,
                                   cudaStream_t stream, bool weights_ready, void *splitk_ws, float *ymax_part,
                                   int *nparts) {
    // weights_ready: the weights were not written by the kernel launched just
    // before this one, so they may be streamed before the dependent-launch wait.
    const int preload = weights_ready ? 8 : 0;
    const int64_t M = act.rows, N = wgt.rows;
    const SplitKLayout skl = splitk_layout(M, N);
    uint8_t *skw = static_cast<uint8_t *>(splitk_ws);
    if (M <= 64) {
        // weights on the MMA's M side, activations on N; y[m][n] = acc[n][m]
        const int bn = M <= 16 ? 16 : (M <= 32 ? 32 : 64);
#define NVFP4_SWAPPED(BNV)                                                                          \
    return y_bf16 ? run_gemm<BNV, true, __nv_bfloat16, FMT>(wgt, act, K, y, ldy, status, timeout_ns, num_sms, preload, skw, skl, ymax_part, nparts, stream) \
                  : run_gemm<BNV, true, float, FMT>(wgt, act, K, y, ldy, status, timeout_ns, num_sms, preload, skw, skl, ymax_part, nparts, stream);
        if (bn == 16) { NVFP4_SWAPPED(16) }
        if (bn == 32) { NVFP4_SWAPPED(32) }
        NVFP4_SWAPPED(64)
#undef NVFP4_SWAPPED
    }
    if (pair_gemm_usable(M, N, num_sms))
        return launch_gemm_pair(act, wgt, K, y, y_bf16, ldy, status, timeout_ns, stream, ymax_part, nparts, FMT);
    const int64_t ptiles = ceil_div(M, 128);
    const bool wide = ptiles * ceil_div(N, 256) >= 2 * num_sms;
    if (wide)
        return y_bf16 ? run_gemm<256, false, __nv_bfloat16, FMT>(act, wgt, K, y, ldy, status, timeout_ns, num_sms, preload, skw, skl, ymax_part, nparts, stream)
                      : run_gemm<256, false, float, FMT>(act, wgt, K, y, ldy, status, timeout_ns, num_sms, preload, skw, skl, ymax_part, nparts, stream);
    return y_bf16 ? run_gemm<128, false, __nv_bfloat16, FMT>(act, wgt, K, y, ldy, status, timeout_ns, num_sms, preload, skw, skl, ymax_part, nparts, stream)
                  : run_gemm<128, false, float, FMT>(act, wgt, K, y, ldy, status, timeout_ns, num_sms, preload, skw, skl, ymax_part, nparts, stream);
}

cudaError_t launch_gemm(const Operand &act, const Operand &wgt, int64_t K, void *y, bool y_bf16,
                        int64_t ldy, uint32_t *status, uint64_t timeout_ns, int num_sms,
                        cudaStream_t stream, bool weights_ready, void *splitk_ws, float *ymax_part,
                        int *nparts) {
    return launch_gemm_fmt<kFmtNV>(act, wgt, K, y, y_bf16, ldy, status, timeout_ns, num_sms, stream, weights_ready,
                                  splitk_ws, ymax_part, nparts);
}

cudaError_t launch_gemm_mx(const Operand &act, const Operand &wgt, int64_t K, void *y, bool y_bf16,
                           int64_t ldy, uint32_t *status, uint64_t timeout_ns, int num_sms,
                           cudaStream_t stream, void *splitk_ws) {
    return launch_gemm_fmt<kFmtMX>(act, wgt, K, y, y_bf16, ldy, status, timeout_ns, num_sms, stream, false,
                                   splitk_ws, nullptr, nullptr);
}

cudaError_t launch_gemm_w4a8(const Operand &act, const Operand &wgt, int64_t K, void *y, bool y_bf16,
                             int64_t ldy, uint32_t *status, uint64_t timeout_ns, int num_sms,
                             cudaStream_t stream, bool weights_ready, void *splitk_ws) {
    return launch_gemm_fmt<kFmtW4A8>(act, wgt, K, y, y_bf16, ldy, status, timeout_ns, num_sms, stream,
                                     weights_ready, splitk_ws, nullptr, nullptr);
}

// ---------------------------------------------------------------------------
// Bounded-wait self test: one thread waits on a barrier nothing completes.
// ---------------------------------------------------------------------------
__global__ void wait_selftest_kernel(uint32_t *status, uint64_t timeout_ns) {
    __shared__ uint64_t bar;
    __shared__ uint32_t abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0u;
        fence_mbar_init();
        // Phase 0 never completes: nobody arrives on the barrier.
        mbar_wait(&bar, 0u, timeout_ns, &abort_flag, status);
    }
}

cudaError_t launch_wait_selftest(uint32_t *status, uint64_t timeout_ns, cudaStream_t stream) {
    wait_selftest_kernel<<<1, 32, 0, stream>>>(status, timeout_ns);
    return cudaGetLastError();
}

}  // namespace nvfp4
