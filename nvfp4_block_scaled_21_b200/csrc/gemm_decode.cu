// gemm_decode.cu -- the W4A4 linear layer for a few activation rows (decode),
// with the activation quantizer inside the GEMM: one launch per call.
//
// y[m][n] = (x_q . W_q^T)[m][n] * gx * gw for M <= 16 activation rows.  The
// weights ride the MMA's M = 128 and the activations its N = 16, so the weight
// stream spreads over the SMs.  Decode is bound by that stream (eefocus.com
// article on FP4 vs INT4: the decode stage is limited by memory bandwidth,
// prefill by compute), so everything else is hidden under it: instead of a
// separate two-pass quantizer whose output every CTA would then load, every
// CTA quantizes x itself (at most 16 x K values).  The arithmetic is the
// standalone quantizer's (tensor amax, g = amax/2688, E4M3 block scale, E2M1
// codes; NVFP4 wiki page, section "技術原理"), so the codes are the same
// bytes; they go straight into the 128-byte-swizzled operand layout in shared
// memory and the block scales into tensor memory.  Both operands then go to
// the FP4 tensor cores as they are (aixq.cc article, section
// "核心差异：W4A4 vs W4A16").
//
// Timeline of one CTA: x is loaded first (every load of a thread issued at
// once; with the weight stream already saturating DRAM an x load would queue
// behind megabytes of weight requests), while the producer has only the first
// kEarlyStages weight stages in flight; then the producer fills the rest of
// the ring while the quantizer warps reduce the amax, encode and write the x
// scales into tensor memory.  From then on the CTA streams weights at the
// ring's pace.
//
// Warps:
//   0     TMA producer: per 256-element K slab, a 128-row weight tile (128-byte
//         swizzle) and its four 512-byte scale atoms, S-deep ring.
//   1     TMEM allocator and MMA issuer: block-scaled MMAs (M = 128, N = 16,
//         K = 64) per slab once the slab's data and weight scales are in;
//         tcgen05.commit releases the stage.
//   2..9  quantize x (amax, scales, codes), write the x scales into tensor
//         memory (and, when asked, x_q to global memory from CTA 0); then
//         warps 2..5 copy each stage's weight scales from shared to tensor
//         memory (tcgen05.st, one warp per TMEM lane quarter, two stages per
//         handshake), and warps 6..9 run the epilogue y = acc * fl32(gx * gw).
// Every wait is bounded; a timeout sets the status word and winds the CTA
// down after its copies and MMAs in flight have landed.
#include <cstdlib>
#include "common.cuh"
#include "encode.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace nvfp4 {

struct DecodeArgs {
    const void *x;           // activations [M][K], row pitch ldx elements
    int64_t ldx;
    int32_t M, K, N;
    int32_t num_tiles;       // ceil(N / 128)
    const uint8_t *sfw;      // tiled scales of the weights
    const float *gw;         // weight tensor scale
    void *y;                 // [M][N], row pitch ldy elements
    int64_t ldy;
    uint8_t *xq_codes;       // optional x_q: codes [M][K/2], tiled scales, tensor scale
    uint8_t *xq_scales;
    float *xq_g;
    float *ymax_part;        // if set: this CTA's largest |y| as stored, at [blockIdx.x]
    uint32_t *status;
    uint64_t timeout_ns;
};

template <int S>
struct DecodeCfg {
    static constexpr int kStages = S;
    static constexpr int kAStage = 128 * 128;              // 128 weight rows x 128 B
    static constexpr int kSfaStage = 4 * 512;              // 4 K-steps x one 512-byte atom
    static constexpr int kStageBytes = kAStage + kSfaStage;
    static constexpr int kXSlab = 16 * 128;                // 16 activation rows x 128 B
    static constexpr int kN = 16;                          // MMA N
    static constexpr int kThreads = 320;                   // 10 warps
    static constexpr int kQThreads = 256;                  // quantizer warps 2..9
    static constexpr int kEarlyStages = 2;                 // weight stages in flight while x loads
    // Each K step of a slab accumulates into its own accumulator (four
    // independent chains of dependent MMAs instead of one), summed in a
    // fixed order in the epilogue; two tiles' worth, double-buffered.
    static constexpr int kAcc = 4;
    static constexpr uint32_t kAccCols = kAcc * kN;        // 64 columns per tile buffer
    static constexpr uint32_t kSlotCol = 2 * kAccCols;     // stage scale slots after the accumulators
    static constexpr uint32_t kSlotCols = 32;              // weight scales 16 | x scales 16
    static constexpr uint32_t kTmemCols = 512;
    static constexpr int kMaxSlabs = 22;                   // x codes in shared memory: K <= 5632
    static constexpr int kBarriers = 3 * kStages + 8;
    static_assert(kSlotCol + kStages * kSlotCols <= kTmemCols, "tensor memory budget");
    static_assert(kStageBytes % 1024 == 0, "stages must stay 1024-byte aligned");
    static_assert(kEarlyStages <= kStages, "early stages fit the ring");
};

// Dynamic shared memory of the kernel with S stages at this K.
template <int S>
static size_t decode_smem_bytes(int64_t K) {
    using C = DecodeCfg<S>;
    const int64_t kslabs = ceil_div(K, 256), ksteps = K / 64;
    return 1024 + static_cast<size_t>(S) * C::kStageBytes + kslabs * C::kXSlab + 16 * ksteps * 4 +
           C::kBarriers * 8 + 64;
}

template <typename T, typename OutT, int S>
__global__ void __launch_bounds__(DecodeCfg<S>::kThreads, 1)
gemm_decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ DecodeArgs args) {
    using C = DecodeCfg<S>;
    constexpr int EPI = Elem<T>::kPerItem;             // values per 16-byte item
    constexpr int W = sizeof(T) == 2 ? 8 : 16;         // 32-bit words per 16-value block
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int kslabs = (args.K + 255) / 256;
    const int ksteps = args.K / 64;
    uint8_t *ring = smem;
    uint8_t *xc = smem + S * C::kStageBytes;                             // x codes, kslabs x 2 KB
    uint32_t *sfw = reinterpret_cast<uint32_t *>(xc + kslabs * C::kXSlab);   // x scale words [ksteps][16]
    uint64_t *full = reinterpret_cast<uint64_t *>(sfw + 16 * ksteps);
    uint64_t *empty = full + S;
    uint64_t *sf_full = empty + S;     // a stage's weight scales are in tensor memory
    uint64_t *tfull = sf_full + S;
    uint64_t *tempty = tfull + 2;
    uint64_t *xready = tempty + 2;     // x codes in shared memory and x scales in TMEM
    uint64_t *red = xready + 1;        // quantizer warps: amax, reciprocal table, codes posted
    uint64_t *mma_done = red + 1;      // every MMA of the MMA thread has completed
    uint64_t *xloaded = mma_done + 1;  // the quantizer warps' x loads have returned
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(xloaded + 1);
    volatile uint32_t *abort_flag = tmem_holder + 1;
    volatile float *wmax = reinterpret_cast<volatile float *>(tmem_holder + 2);   // [8]
    __shared__ float rcp_table[128];   // fl32(1 / fl32(dec(s) * g)) for every E4M3 byte s (0: zero block)
    __shared__ float s_ymax[4];        // epilogue warps' largest |stored y|

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        prefetch_tensormap(&tmW);
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&sf_full[s], 4);     // one arrive per scale warp
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&tfull[s], 1);
            mbar_init(&tempty[s], 4);      // one arrive per epilogue warp
        }
        mbar_init(xready, 8);
        mbar_init(red, 8);
        mbar_init(mma_done, 1);
        mbar_init(xloaded, 8);
        *abort_flag = 0u;
        fence_mbar_init();
    }
    if (threadIdx.x < 4) s_ymax[threadIdx.x] = 0.0f;
    if (warp == 1) tmem_alloc(tmem_holder, C::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const int my_tiles = static_cast<int>(blockIdx.x) < args.num_tiles
                             ? (args.num_tiles - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                             : 0;
    const int total = my_tiles * kslabs;              // weight slabs of this CTA, all tiles
    // The next launch may set itself up on idle SMs now; its own dependent-
    // launch wait still waits for this whole grid to finish.  Then wait for
    // the kernel before this one: it may have written x or the weights.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------------ producer
            const uint64_t pol = policy_evict_first();
            int issued = 0;
            for (int i = 0; i < total; ++i) {
                const int t = static_cast<int>(blockIdx.x) + (i / kslabs) * static_cast<int>(gridDim.x);
                const int ks = i % kslabs;
                const int nk = min(4, ksteps - 4 * ks);
                const uint32_t st = static_cast<uint32_t>(i % S);
                // only kEarlyStages stages compete with the x loads
                if (i == C::kEarlyStages && !mbar_wait(xloaded, 0, args.timeout_ns, abort_flag, args.status)) break;
                if (i >= S &&
                    !mbar_wait(&empty[st], static_cast<uint32_t>(i / S - 1) & 1u, args.timeout_ns, abort_flag,
                               args.status))
                    break;
                uint8_t *sp = ring + st * C::kStageBytes;
                mbar_arrive_expect_tx(&full[st], C::kAStage + nk * 512);
                tma_load_2d(sp, &tmW, &full[st], ks * 128, t * 128, pol);
                bulk_load(sp + C::kAStage, args.sfw + (static_cast<int64_t>(t) * ksteps + 4 * ks) * 512, nk * 512,
                          &full[st], pol);
                ++issued;
            }
            // No copy may still be landing when the CTA exits: wait (bounded,
            // also after an abort) for the last load issued into every stage.
            // On the normal path the MMA thread has consumed them all already.
            volatile uint32_t keep_waiting = 0u;
            for (int j = issued > S ? issued - S : 0; j < issued; ++j)
                mbar_wait(&full[j % S], static_cast<uint32_t>(j / S) & 1u, args.timeout_ns, &keep_waiting,
                          args.status);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------------------ MMA issuer
            constexpr uint32_t idesc = make_idesc_nvf4(C::kN);
            const uint32_t ring_base = smem_addr(ring), x_base = smem_addr(xc);
            bool ok = mbar_wait(xready, 0, args.timeout_ns, abort_flag, args.status);
            tc_fence_after();
            uint32_t acc = 0, acc_phase = 0;
            for (int i = 0; ok && i < total; ++i) {
                const int ks = i % kslabs;
                const uint32_t st = static_cast<uint32_t>(i % S), par = static_cast<uint32_t>(i / S) & 1u;
                if (ks == 0) {
                    if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, args.timeout_ns, abort_flag, args.status)) break;
                    tc_fence_after();
                }
                if (!mbar_wait(&full[st], par, args.timeout_ns, abort_flag, args.status) ||
                    !mbar_wait(&sf_full[st], par, args.timeout_ns, abort_flag, args.status))
                    break;
                tc_fence_after();
                const int nk = min(4, ksteps - 4 * ks);
                // K step q of the slab into accumulator q (the first slab overwrites)
                const uint32_t d_tmem = tmem_base + acc * C::kAccCols;
                const uint32_t sfa = tmem_base + C::kSlotCol + C::kSlotCols * st;
                const uint32_t sfb = sfa + 16;
                // K-step q: +32 bytes = +2 in the descriptors' address field
                const uint64_t adesc = make_operand_desc(ring_base + st * C::kStageBytes);
                const uint64_t bdesc = make_operand_desc(x_base + ks * C::kXSlab);
                if (nk == 4) {
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        mma_nvf4(d_tmem + q * C::kN, adesc + 2 * q, bdesc + 2 * q, idesc, sfa + 4 * q, sfb + 4 * q,
                                 ks != 0 ? 1u : 0u);
                } else {
                    for (int q = 0; q < nk; ++q)
                        mma_nvf4(d_tmem + q * C::kN, adesc + 2 * q, bdesc + 2 * q, idesc, sfa + 4 * q, sfb + 4 * q,
                                 ks != 0 ? 1u : 0u);
                }
                tc_commit(&empty[st]);
                if (ks == kslabs - 1) {
                    tc_commit(&tfull[acc]);
                    acc ^= 1u;
                    if (acc == 0) acc_phase ^= 1u;
                }
            }
            // Tensor memory is freed below: first let every MMA this thread
            // issued complete (bounded, also after an abort).
            tc_commit(mma_done);
            volatile uint32_t keep_waiting = 0u;
            mbar_wait(mma_done, 0, args.timeout_ns, &keep_waiting, args.status);
        }
    } else {
        // ---------------------------------------------------------------- quantizer
        const int qt = static_cast<int>(threadIdx.x) - 64;  // 0..255
        const int qw = warp - 2;                            // 0..7
        const int quarter = warp & 3;                       // TMEM lane quarter this warp may access
        const int half = qw >> 2;                           // 0: scale warps (2..5), 1: epilogue (6..9)
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
        const T *x = static_cast<const T *>(args.x);
        // One thread per 16-value block: block b = j * 256 + qt (j < BPT in one
        // round; more rounds re-read x).  Consecutive threads take consecutive
        // blocks along a row, so a warp's loads are contiguous, and the four
        // blocks of a 64-value group (one MMA K step, one scale word) sit in
        // four neighbouring lanes: K/16 is a multiple of 4, so is 256, hence
        // b % 4 == lane % 4 and the group's blocks share a row.
        constexpr int BPT = sizeof(T) == 2 ? 10 : 5;        // blocks per thread per round
        constexpr int IPB = 16 / EPI;                       // 16-byte items per block
        const int bpr = args.K / 16;
        const int nblocks = args.M * bpr;
        const int per_round = C::kQThreads * BPT;
        const int rounds = (nblocks + per_round - 1) / per_round;
        uint4 v[BPT][IPB];
        auto load_round = [&](int rd) {
#pragma unroll
            for (int j = 0; j < BPT; ++j) {
                const int b = rd * per_round + j * C::kQThreads + qt;
                if (b < nblocks) {
                    const int r = b / bpr, kb = b - r * bpr;
                    const T *src = x + static_cast<int64_t>(r) * args.ldx + static_cast<int64_t>(kb) * 16;
#pragma unroll
                    for (int i = 0; i < IPB; ++i) v[j][i] = load_item(src + i * EPI);
                } else {
#pragma unroll
                    for (int i = 0; i < IPB; ++i) v[j][i] = make_uint4(0u, 0u, 0u, 0u);
                }
            }
        };
        auto block_words = [&](int j, uint32_t (&w)[W]) {
#pragma unroll
            for (int i = 0; i < IPB; ++i) {
                w[4 * i] = v[j][i].x; w[4 * i + 1] = v[j][i].y; w[4 * i + 2] = v[j][i].z; w[4 * i + 3] = v[j][i].w;
            }
        };

        // (1) tensor amax of x, exact (maxima of |x| bit patterns), over the 8 warps
        float m = 0.0f;
        for (int rd = 0; rd < rounds; ++rd) {
            load_round(rd);
#pragma unroll
            for (int j = 0; j < BPT; ++j)
#pragma unroll
                for (int i = 0; i < IPB; ++i) m = fmaxf(m, item_absmax(v[j][i], static_cast<T *>(nullptr)));
            if (rd == 0) {
                __syncwarp();
                if (lane == 0) mbar_arrive(xloaded);        // the producer may fill the rest of the ring
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) {
            wmax[qw] = m;
            mbar_arrive(red);
        }
        bool ok = __all_sync(0xffffffffu, mbar_wait(red, 0, args.timeout_ns, abort_flag, args.status));
        float amax = 0.0f;
#pragma unroll
        for (int k = 0; k < 8; ++k) amax = fmaxf(amax, wmax[k]);
        const float g = __fdiv_rn(amax, kTensorScaleDiv);
        const float six_g = __fmul_rn(6.0f, g);
        const float inv6g = __frcp_rn(six_g);
        const bool exact_only = !(six_g > 0.0f) || isinf(inv6g);
        const bool write_xq = args.xq_codes != nullptr && blockIdx.x == 0;
        // reciprocal of every possible decoded block scale, one per thread
        if (qt < 128) rcp_table[qt] = block_rcp(static_cast<uint32_t>(qt), g);
        __syncwarp();
        if (lane == 0) mbar_arrive(red);
        ok = ok && __all_sync(0xffffffffu, mbar_wait(red, 1, args.timeout_ns, abort_flag, args.status));

        // (2) codes and scale words (the last round's values are still in
        // registers): all block scales first, then all codes, so that the
        // thread's independent blocks overlap.  Block kb of row r (K step
        // gq = kb / 4) holds bytes 32*(gq%4) + 8*(kb%4) .. +7 of that row in
        // slab gq/4, i.e. 16-byte chunk 2*(gq%4) + (kb%4)/2, half kb%2, placed
        // with the 128-byte swizzle (chunk c of row r at chunk c ^ (r % 8)),
        // the layout a TMA load would give.
        if (ok) {
            for (int rd = rounds - 1; rd >= 0; --rd) {
                if (rd != rounds - 1) load_round(rd);
                uint32_t sb[BPT];
#pragma unroll
                for (int j = 0; j < BPT; ++j) {
                    uint32_t w[W];
                    block_words(j, w);
                    sb[j] = block_scale_byte(block_absmax(w, static_cast<T *>(nullptr)), six_g, inv6g, exact_only);
                }
#pragma unroll
                for (int j = 0; j < BPT; ++j) {
                    uint32_t w[W];
                    block_words(j, w);
                    const uint2 cw = block_codes<T, W>(w, rcp_table[sb[j]]);
                    uint32_t word = sb[j];
                    word |= __shfl_down_sync(0xffffffffu, sb[j], 1) << 8;
                    word |= __shfl_down_sync(0xffffffffu, sb[j], 2) << 16;
                    word |= __shfl_down_sync(0xffffffffu, sb[j], 3) << 24;
                    const int b = rd * per_round + j * C::kQThreads + qt;
                    if (b < nblocks) {
                        const int r = b / bpr, kb = b - r * bpr, gq = kb >> 2;
                        const int c = 2 * (gq & 3) + ((kb & 3) >> 1);
                        *reinterpret_cast<uint2 *>(xc + (gq >> 2) * C::kXSlab + r * 128 + ((c ^ (r & 7)) << 4) +
                                                   8 * (kb & 1)) = cw;
                        if ((lane & 3) == 0) sfw[gq * 16 + r] = word;
                        if (write_xq)
                            if (store_ok(args.xq_codes + static_cast<int64_t>(r) * (args.K / 2) + kb * 8, 8, args.xq_codes,
                                         static_cast<size_t>(args.M) * (args.K / 2), args.status))
                                *reinterpret_cast<uint2 *>(args.xq_codes + static_cast<int64_t>(r) * (args.K / 2) + kb * 8) = cw;
                    }
                }
            }
            // rows M..15 of the MMA's N = 16 are zero (codes and scales)
            for (int i = qt; i < (C::kN - args.M) * ksteps; i += C::kQThreads) {
                const int r = args.M + i / ksteps, gq = i % ksteps;
                sfw[gq * 16 + r] = 0u;
                uint8_t *row = xc + (gq >> 2) * C::kXSlab + r * 128;
                const int c0 = 2 * (gq & 3);
                st_shared_v4(row + ((c0 ^ (r & 7)) << 4), 0u, 0u, 0u, 0u);
                st_shared_v4(row + (((c0 + 1) ^ (r & 7)) << 4), 0u, 0u, 0u, 0u);
            }
            if (write_xq && qt == 0) *args.xq_g = g;
        }
        fence_proxy_async_smem();          // the codes, for the tensor cores' operand reads
        __syncwarp();
        if (lane == 0) mbar_arrive(red);
        ok = ok && __all_sync(0xffffffffu, mbar_wait(red, 0, args.timeout_ns, abort_flag, args.status));

        // The x codes are in shared memory and the x scale words in sfw: the
        // MMA may read the codes; the scale warps copy each slab's x scale words
        // into tensor memory together with its weight scales.
        __syncwarp();
        if (lane == 0) mbar_arrive(xready);
        if (ok && write_xq) {
            // x_q's tiled scales, whole 16-byte chunks: chunk l of K step gq's
            // atom holds rows l, l + 32, l + 64, l + 96; only row l < M <= 16
            // is data, the rest (and rows M .. 15 of sfw) is zero padding
            for (int i = qt; i < ksteps * 32; i += C::kQThreads) {
                const int gq = i >> 5, l = i & 31;
                const uint32_t w0 = l < C::kN ? sfw[gq * 16 + l] : 0u;
                uint8_t *sp = args.xq_scales + static_cast<int64_t>(gq) * 512 + l * 16;
                if (store_ok(sp, 16, args.xq_scales, static_cast<size_t>(ksteps) * 512, args.status))
                    *reinterpret_cast<uint4 *>(sp) = make_uint4(w0, 0u, 0u, 0u);
            }
        }

        if (half == 0) {
            // ------------------------------------------------------------ scale warps
            // Per slab, one 32-column store into the stage's TMEM slot:
            // the weight scales (lane l of every quarter receives the 16 bytes
            // at l*16 of each 512-byte atom: columns c = 0..3 hold rows 32c + l,
            // bytes = the 4 K-blocks), then the x scales (replicated in every
            // quarter: the word of row l < 16 at K step q of the slab goes to
            // lane l, column 16 + 4q; the other columns and lanes are zero).
            // Stages are handed to the MMA two at a time (one store-completion
            // wait per pair).  A partial last slab's missing atoms and K steps
            // are bytes no MMA reads.
            uint32_t pend[2];
            int npend = 0;
            auto flush = [&]() {
                if (npend == 0) return;
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    for (int k = 0; k < npend; ++k) mbar_arrive(&sf_full[pend[k]]);
                npend = 0;
            };
            for (int i = 0; ok && i < total; ++i) {
                const uint32_t st = static_cast<uint32_t>(i % S), par = static_cast<uint32_t>(i / S) & 1u;
                const bool got = mbar_wait(&full[st], par, args.timeout_ns, abort_flag, args.status);
                if (!__all_sync(0xffffffffu, got)) break;
                const uint8_t *src = ring + st * C::kStageBytes + C::kAStage + lane * 16;
                const int ks = i % kslabs;
                uint32_t av[32];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 a = ld_shared_v4(src + j * 512);
                    av[4 * j] = a.x; av[4 * j + 1] = a.y; av[4 * j + 2] = a.z; av[4 * j + 3] = a.w;
                    const int gk = 4 * ks + j;
                    av[16 + 4 * j] = (lane < 16 && gk < ksteps) ? sfw[gk * 16 + lane] : 0u;
                    av[17 + 4 * j] = 0u;
                    av[18 + 4 * j] = 0u;
                    av[19 + 4 * j] = 0u;
                }
                tmem_st_32x32b_x32(lane_base + C::kSlotCol + C::kSlotCols * st, av);
                pend[npend++] = st;
                if (npend == 2) flush();
            }
            flush();
        } else {
            // ------------------------------------------------------------ epilogue
            const float alpha = __fmul_rn(g, *args.gw);
            YMax ym;                       // largest |y| this thread stores
            uint32_t acc = 0, acc_phase = 0;
            for (int tt = 0; ok && tt < my_tiles; ++tt) {
                const int t = static_cast<int>(blockIdx.x) + tt * static_cast<int>(gridDim.x);
                const bool got = mbar_wait(&tfull[acc], acc_phase, args.timeout_ns, abort_flag, args.status);
                if (!__all_sync(0xffffffffu, got)) break;
                tc_fence_after();
                uint32_t r4[C::kAcc][16];
#pragma unroll
                for (int a = 0; a < C::kAcc; ++a) tmem_ld_32x32b_x16(lane_base + acc * C::kAccCols + a * C::kN, r4[a]);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[acc]);
                // acc0 + acc1 + acc2 + acc3 in that order; accumulators that
                // no K step reached (K < 256) hold no data and are skipped
                float r[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float v = __uint_as_float(r4[0][i]);
#pragma unroll
                    for (int a = 1; a < C::kAcc; ++a)
                        if (a < ksteps) v = __fadd_rn(v, __uint_as_float(r4[a][i]));
                    r[i] = v;
                }
                const int p = t * 128 + quarter * 32 + lane;     // weight row = output column
                if (p < args.N) {
                    OutT *y = static_cast<OutT *>(args.y);
#pragma unroll
                    for (int i = 0; i < C::kN; ++i) {
                        if (i < args.M &&
                            store_ok(y + static_cast<int64_t>(i) * args.ldy + p, sizeof(OutT), args.y,
                                     matrix_extent(args.M, args.N, args.ldy, sizeof(OutT)), args.status)) {
                            const OutT o = to_out<OutT>(__fmul_rn(r[i], alpha));
                            y[static_cast<int64_t>(i) * args.ldy + p] = o;
                            ym.add<OutT>(o);
                        }
                    }
                }
                acc ^= 1u;
                if (acc == 0) acc_phase ^= 1u;
            }
            float mm = ym.value();
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mm = fmaxf(mm, __shfl_xor_sync(0xffffffffu, mm, o));
            if (lane == 0) s_ymax[qw - 4] = mm;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && args.ymax_part != nullptr)
        args.ymax_part[blockIdx.x] = fmaxf(fmaxf(s_ymax[0], s_ymax[1]), fmaxf(s_ymax[2], s_ymax[3]));
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

// The ring is 10 stages deep where shared and tensor memory allow (K up to
// 5120), else 8 (K up to 5632).
static int decode_stages(int64_t K) {
    const int64_t kslabs = ceil_div(K, 256);
    // 640 bytes of headroom for the kernel's static shared memory (the
    // reciprocal table and the epilogue maxima, 528 bytes)
    if (kslabs <= DecodeCfg<10>::kMaxSlabs && decode_smem_bytes<10>(K) + 640 <= 232448) return 10;
    return 8;
}

bool decode_fused_usable(int64_t M, int64_t N, int64_t K) {
    // Opt-in (NVFP4_DECODE_FUSED=1): measured on B200 at M = 8, N = 17408,
    // K = 5120 the quantizer + GEMM path takes 17 us per call and this
    // kernel 20.5 us (its in-kernel quantization of x holds back the first
    // MMAs by ~8 us, longer than its ring of weight stages covers).
    const char *opt = getenv("NVFP4_DECODE_FUSED");
    if (opt == nullptr || opt[0] != '1') return false;
    return M >= 1 && M <= DecodeCfg<8>::kN && N >= 1 && K >= 64 && K % 64 == 0 &&
           ceil_div(K, 256) <= DecodeCfg<8>::kMaxSlabs;
}

template <typename T, typename OutT, int S>
static cudaError_t run_decode(const CUtensorMap &tmW, const DecodeArgs &a, int grid, cudaStream_t stream) {
    auto kern = gemm_decode_kernel<T, OutT, S>;
    const size_t smem = decode_smem_bytes<S>(a.K);
    // set on every launch: the attribute belongs to the current device
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(DecodeCfg<S>::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tmW, a);
}

template <int S>
static cudaError_t run_decode_s(const CUtensorMap &tmW, const DecodeArgs &a, bool x_bf16, bool y_bf16, int grid,
                                cudaStream_t stream) {
    if (x_bf16)
        return y_bf16 ? run_decode<__nv_bfloat16, __nv_bfloat16, S>(tmW, a, grid, stream)
                      : run_decode<__nv_bfloat16, float, S>(tmW, a, grid, stream);
    return y_bf16 ? run_decode<float, __nv_bfloat16, S>(tmW, a, grid, stream)
                  : run_decode<float, float, S>(tmW, a, grid, stream);
}

cudaError_t launch_gemm_decode(const void *x, bool x_bf16, int64_t M, int64_t K, int64_t ldx, const Operand &wgt,
                               void *y, bool y_bf16, int64_t ldy, uint8_t *xq_codes, uint8_t *xq_scales,
                               float *xq_g, uint32_t *status, uint64_t timeout_ns, int num_sms,
                               cudaStream_t stream, float *ymax_part, int *nparts) {
    const int64_t N = wgt.rows;
    CUtensorMap tmW;
    if (encode_tensor_map_u8(&tmW, wgt.codes, K / 2, N, 128, 128) != CUDA_SUCCESS) return cudaErrorInvalidValue;
    DecodeArgs a;
    a.x = x;
    a.ldx = ldx;
    a.M = static_cast<int32_t>(M);
    a.K = static_cast<int32_t>(K);
    a.N = static_cast<int32_t>(N);
    a.num_tiles = static_cast<int32_t>(ceil_div(N, 128));
    a.sfw = wgt.scales;
    a.gw = wgt.g;
    a.y = y;
    a.ldy = ldy;
    a.xq_codes = xq_codes;
    a.xq_scales = xq_scales;
    a.xq_g = xq_g;
    a.ymax_part = ymax_part;
    a.status = status;
    a.timeout_ns = timeout_ns;
    const int grid = static_cast<int>(a.num_tiles < num_sms ? a.num_tiles : num_sms);
    if (nparts) *nparts = grid;
    return decode_stages(K) == 10 ? run_decode_s<10>(tmW, a, x_bf16, y_bf16, grid, stream)
                                  : run_decode_s<8>(tmW, a, x_bf16, y_bf16, grid, stream);
}

}  // namespace nvfp4
