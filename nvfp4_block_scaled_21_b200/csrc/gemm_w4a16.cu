// gemm_w4a16.cu -- the W4A16 linear layer: NVFP4 weights, 16-bit (bf16)
// activations.
//
// W4A16 is the scheme the aixq.cc article on Unsloth Dynamic NVFP4 (section
// "核心差异：W4A4 vs W4A16") compares W4A4 against: the weights are 4-bit but
// the activations stay 16-bit, so the weights are dequantized to 16 bits
// before the matrix product.  Here every weight value e * s (E2M1 element
// times its E4M3 block scale) is exact in bf16 (at most 2 + 4 significant
// bits, magnitudes 2^-10 .. 2688), so the dequantized operand loses nothing;
// the FP32 tensor scale is applied to the fp32 accumulator in the epilogue:
//     y[m][n] = fl32(acc[m][n] * gw),  acc = sum_k x[m][k] * (e * s)[n][k]
// accumulated in fp32 by the bf16 tensor cores (kind::f16).
//
// Small M ("swapped", like the W4A4 decode path): the weights ride the MMA's
// M = 128 and 16 activation rows its N.  Converter warps dequantize each
// weight slab straight into tensor memory (tcgen05.st), where the MMA reads
// its A operand, so the 16-bit weights never pass through shared memory;
// the activations come by TMA as the MMA's B operand.  Larger M runs the same
// tiles over every 16-row group of activations (the weight stream is read
// once per group).
//
// Warps (448 threads):
//   0       TMA producer: per 256-deep K slab, the 128-row weight tile (packed
//           E2M1, 128-byte swizzle), its four 512-byte scale atoms, and four
//           64-column chunks of the 16 activation rows (bf16, 128-byte
//           swizzle), S-deep ring.
//   1       TMEM allocator and MMA issuer: 16 MMAs (M = 128, N = 16, K = 16,
//           A from tensor memory) per slab, MMA i of a slab into accumulator
//           i % 8 (an MMA this small takes far less time than the latency of
//           the previous one into the same accumulator).
//   2..9    converters: two warps per TMEM lane quarter (one weight row per
//           thread), each dequantizing two of the slab's four 64-wide K steps
//           into one of two tensor-memory A slots.
//   10..13  epilogue: acc = the 8 accumulators added in order, y = acc * gw,
//           stored as y[m][n].
// Every wait is bounded; a timeout sets the status word and winds the CTA
// down after its copies and MMAs in flight have landed.
#include <cstdlib>
#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace nvfp4 {

namespace {

struct W16Args {
    const uint8_t *sfw;      // tiled scales of the weights
    const float *gw;         // weight tensor scale
    void *y;                 // [M][N], row pitch ldy elements
    int64_t ldy;
    int32_t M, N, K;
    int32_t num_wt, num_xt;  // 128-row weight tiles, 16-row activation tiles
    uint32_t *status;
    uint64_t timeout_ns;
};

struct W16Cfg {
    static constexpr int kStages = 7;
    static constexpr int kWStage = 128 * 128;              // 128 weight rows x 128 B (256 values)
    static constexpr int kSfStage = 4 * 512;               // 4 K steps x one 512-byte atom
    static constexpr int kXChunk = 16 * 128;               // 16 activation rows x 64 bf16
    static constexpr int kXStage = 4 * kXChunk;
    static constexpr int kStageBytes = kWStage + kSfStage + kXStage;   // 26 KB
    static constexpr int kN = 16;
    static constexpr int kThreads = 448;
    static constexpr int kNumAcc = 8;                      // accumulators, kN columns each
    static constexpr uint32_t kASlotCol = kNumAcc * kN;    // A slots after the accumulators
    static constexpr uint32_t kASlotCols = 128;            // 256 bf16 per row
    static constexpr uint32_t kTmemCols = 512;
    static constexpr int kBarBytes = 8 * (2 * kStages + 8) + 16;
    static constexpr int kSmemBytes = kStages * kStageBytes + kBarBytes + 1024;
    static_assert(kStageBytes % 1024 == 0, "stages must stay 1024-byte aligned");
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static_assert(kASlotCol + 2 * kASlotCols <= kTmemCols, "tensor memory budget");
};

// Instruction descriptor of kind::f16 with bf16 A and B, fp32 accumulation,
// K-major operands, M = 128 and the given N.
__host__ __device__ constexpr uint32_t make_idesc_bf16(uint32_t n) {
    return (1u << 4)            // D format: F32
         | (1u << 7)            // A format: BF16
         | (1u << 10)           // B format: BF16
         | ((n >> 3) << 17)     // N >> 3
         | ((128u >> 4) << 24); // M >> 4
}

// D[tmem] (+)= A[tmem] . B[smem]^T, bf16 inputs, fp32 accumulation.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Four E2M1 code bytes (8 values, element 2j in the low nibble of byte j)
// times one block scale given as an f16 pair (s, s), as four bf16 pairs.
// E2M1 -> f16 and the f16 product are exact (e * s has at most 6
// significant bits and lies in 2^-10 .. 2688); f16 -> fp32 -> bf16 is exact
// for the same reason.
__device__ __forceinline__ void dequant_x8_bf16(uint32_t codes, uint32_t s2, uint32_t (&out)[4]) {
    uint32_t h[4];
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(codes));
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        uint32_t p;
        asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(p) : "r"(h[k]), "r"(s2));
        const float lo = __half2float(__ushort_as_half(static_cast<unsigned short>(p & 0xffffu)));
        const float hi = __half2float(__ushort_as_half(static_cast<unsigned short>(p >> 16)));
        __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
        out[k] = *reinterpret_cast<uint32_t *>(&b);
    }
}

// Four E4M3 scale bytes as four f16 pairs (s_i, s_i).
__device__ __forceinline__ void scales_f16x2(uint32_t word, uint32_t (&s2)[4]) {
    uint32_t lo, hi;
    asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(word));
    s2[0] = (lo & 0xffffu) * 0x10001u;
    s2[1] = (lo >> 16) * 0x10001u;
    s2[2] = (hi & 0xffffu) * 0x10001u;
    s2[3] = (hi >> 16) * 0x10001u;
}

template <typename OutT>
__global__ void __launch_bounds__(W16Cfg::kThreads, 1)
gemm_w4a16_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                  const __grid_constant__ W16Args args) {
    using C = W16Cfg;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + S * C::kStageBytes);
    uint64_t *empty = full + S;
    uint64_t *a_full = empty + S;      // [2] a slab's weights dequantized into an A slot
    uint64_t *a_empty = a_full + 2;    // [2] the MMAs reading an A slot have completed
    uint64_t *tfull = a_empty + 2;
    uint64_t *tempty = tfull + 1;
    uint64_t *mma_done = tempty + 1;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile uint32_t *abort_flag = tmem_holder + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        prefetch_tensormap(&tmW);
        prefetch_tensormap(&tmX);
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&a_full[s], 8);      // one arrive per converter warp
            mbar_init(&a_empty[s], 1);
        }
        mbar_init(tfull, 1);
        mbar_init(tempty, 4);              // one arrive per epilogue warp
        mbar_init(mma_done, 1);
        *abort_flag = 0u;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_holder, C::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    const int ksteps = args.K / 64;
    const int kslabs = (ksteps + 3) / 4;
    const int num_tiles = args.num_wt * args.num_xt;
    const int my_tiles = static_cast<int>(blockIdx.x) < num_tiles
                             ? (num_tiles - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1
                             : 0;
    const int total = my_tiles * kslabs;
    // tile order: the activation tiles of one weight tile are consecutive
    auto tile_of = [&](int tt, int &wt, int &xt) {
        const int t = static_cast<int>(blockIdx.x) + tt * static_cast<int>(gridDim.x);
        wt = t / args.num_xt;
        xt = t - wt * args.num_xt;
    };

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------------ producer
            const uint64_t pol_w = policy_evict_first(), pol_x = policy_evict_last();
            int issued = 0;
            for (int i = 0; i < total; ++i) {
                int wt, xt;
                tile_of(i / kslabs, wt, xt);
                const int ks = i % kslabs;
                const int nk = min(4, ksteps - 4 * ks);
                const uint32_t st = static_cast<uint32_t>(i % S);
                if (i >= S &&
                    !mbar_wait(&empty[st], static_cast<uint32_t>(i / S - 1) & 1u, args.timeout_ns, abort_flag,
                               args.status))
                    break;
                uint8_t *sp = smem + st * C::kStageBytes;
                mbar_arrive_expect_tx(&full[st], C::kWStage + nk * 512 + nk * C::kXChunk);
                tma_load_2d(sp, &tmW, &full[st], ks * 128, wt * 128, pol_w);
                bulk_load(sp + C::kWStage, args.sfw + (static_cast<int64_t>(wt) * ksteps + 4 * ks) * 512, nk * 512,
                          &full[st], pol_w);
                for (int c = 0; c < nk; ++c)
                    tma_load_2d(sp + C::kWStage + C::kSfStage + c * C::kXChunk, &tmX, &full[st], (4 * ks + c) * 64,
                                xt * C::kN, pol_x);
                ++issued;
            }
            volatile uint32_t keep_waiting = 0u;
            for (int j = issued > S ? issued - S : 0; j < issued; ++j)
                mbar_wait(&full[j % S], static_cast<uint32_t>(j / S) & 1u, args.timeout_ns, &keep_waiting,
                          args.status);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------------------ MMA issuer
            constexpr uint32_t idesc = make_idesc_bf16(C::kN);
            const uint32_t smem_base = smem_addr(smem);
            uint32_t tphase = 0;
            for (int i = 0; i < total; ++i) {
                const int ks = i % kslabs;
                const uint32_t st = static_cast<uint32_t>(i % S), par = static_cast<uint32_t>(i / S) & 1u;
                const uint32_t slot = static_cast<uint32_t>(i & 1), spar = static_cast<uint32_t>(i >> 1) & 1u;
                if (ks == 0) {
                    // the previous tile's accumulator has been read
                    if (i > 0 && !mbar_wait(tempty, tphase ^ 1u, args.timeout_ns, abort_flag, args.status)) break;
                    tc_fence_after();
                }
                if (!mbar_wait(&full[st], par, args.timeout_ns, abort_flag, args.status) ||
                    !mbar_wait(&a_full[slot], spar, args.timeout_ns, abort_flag, args.status))
                    break;
                tc_fence_after();
                const int nk = min(4, ksteps - 4 * ks);
                const uint32_t a0 = tmem_base + C::kASlotCol + slot * C::kASlotCols;
                const uint32_t x0 = smem_base + st * C::kStageBytes + C::kWStage + C::kSfStage;
                for (int c = 0; c < nk; ++c) {
                    const uint64_t bdesc = make_operand_desc(x0 + c * C::kXChunk);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {   // K = 16 per MMA: 8 TMEM columns, 32 bytes of a row
                        // MMA 4c + q of the slab -> accumulator (4c + q) % 8,
                        // overwritten by its first MMA of the tile (slab 0:
                        // K % 64 == 0, so every slab has K steps 0 and 1)
                        const int a = (4 * c + q) % C::kNumAcc;
                        mma_bf16_ts(tmem_base + a * C::kN, a0 + 32 * c + 8 * q, bdesc + 2 * q, idesc,
                                    (ks != 0 || 4 * c + q >= C::kNumAcc) ? 1u : 0u);
                    }
                }
                tc_commit(&empty[st]);
                tc_commit(&a_empty[slot]);
                if (ks == kslabs - 1) {
                    tc_commit(tfull);
                    tphase ^= 1u;
                }
            }
            tc_commit(mma_done);
            volatile uint32_t keep_waiting = 0u;
            mbar_wait(mma_done, 0, args.timeout_ns, &keep_waiting, args.status);
        }
    } else if (warp < 10) {
        // ---------------------------------------------------------------- converters
        // Thread: weight row r = 32 * quarter + lane of the tile; K steps
        // 2h and 2h + 1 of each slab.  Its row of the weight tile sits at
        // r * 128 in the stage, 16-byte chunk c at chunk c ^ (r % 8); its four
        // scale bytes of K step j at (r % 32) * 16 + ((r / 32) % 4) * 4 of atom j.
        const int quarter = warp & 3, h = (warp - 2) >> 2;
        const int r = quarter * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
        for (int i = 0; i < total; ++i) {
            const int ks = i % kslabs;
            const uint32_t st = static_cast<uint32_t>(i % S), par = static_cast<uint32_t>(i / S) & 1u;
            const uint32_t slot = static_cast<uint32_t>(i & 1);
            bool got = mbar_wait(&full[st], par, args.timeout_ns, abort_flag, args.status);
            if (i >= 2)
                got = got && mbar_wait(&a_empty[slot], static_cast<uint32_t>((i >> 1) - 1) & 1u, args.timeout_ns,
                                       abort_flag, args.status);
            if (!__all_sync(0xffffffffu, got)) break;
            tc_fence_after();
            const int nk = min(4, ksteps - 4 * ks);
            const uint8_t *sp = smem + st * C::kStageBytes;
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int j = 2 * h + jj;
                if (j < nk) {
                    const uint4 c0 = ld_shared_v4(sp + r * 128 + (((2 * j) ^ (r & 7)) << 4));
                    const uint4 c1 = ld_shared_v4(sp + r * 128 + (((2 * j + 1) ^ (r & 7)) << 4));
                    const uint32_t sw = *reinterpret_cast<const uint32_t *>(
                        sp + C::kWStage + j * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4);
                    uint32_t s2[4];
                    scales_f16x2(sw, s2);
                    uint32_t v[32];
                    const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                    for (int b = 0; b < 8; ++b)   // word b: values 8b .. 8b+7, block b / 2
                        dequant_x8_bf16(cw[b], s2[b >> 1], *reinterpret_cast<uint32_t(*)[4]>(v + 4 * b));
                    tmem_st_32x32b_x32(lane_base + C::kASlotCol + slot * C::kASlotCols + 32 * j, v);
                }
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[slot]);
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        const int quarter = warp & 3;
        const float gw = *args.gw;
        uint32_t tphase = 0;
        for (int tt = 0; tt < my_tiles; ++tt) {
            int wt, xt;
            tile_of(tt, wt, xt);
            const bool got = mbar_wait(tfull, tphase, args.timeout_ns, abort_flag, args.status);
            if (!__all_sync(0xffffffffu, got)) break;
            tphase ^= 1u;
            tc_fence_after();
            // ((a0 + a1) + a2) + ... in fp32, over the accumulators written:
            // four MMAs per K step, so K = 64 (one K step) writes a0..a3 only
            const uint32_t lb = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
            const int nacc = min(C::kNumAcc, 4 * min(4, ksteps));
            uint32_t acc[16];
            tmem_ld_32x32b_x16(lb, acc);
            tmem_ld_wait();
            for (int a = 1; a < nacc; ++a) {
                uint32_t t[16];
                tmem_ld_32x32b_x16(lb + a * C::kN, t);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    acc[i] = __float_as_uint(__fadd_rn(__uint_as_float(acc[i]), __uint_as_float(t[i])));
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty);
            const int p = wt * 128 + quarter * 32 + lane;       // weight row = output column
            if (p < args.N) {
                OutT *y = static_cast<OutT *>(args.y);
#pragma unroll
                for (int i = 0; i < C::kN; ++i) {
                    const int m = xt * C::kN + i;
                    if (m < args.M && store_ok(y + static_cast<int64_t>(m) * args.ldy + p, sizeof(OutT), args.y,
                                               matrix_extent(args.M, args.N, args.ldy, sizeof(OutT)), args.status))
                        y[static_cast<int64_t>(m) * args.ldy + p] = to_out<OutT>(__fmul_rn(__uint_as_float(acc[i]), gw));
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

}  // namespace

cudaError_t launch_gemm_w4a16(const void *x, int64_t M, int64_t K, int64_t ldx, const Operand &wgt, void *y,
                              bool y_bf16, int64_t ldy, uint32_t *status, uint64_t timeout_ns, int num_sms,
                              cudaStream_t stream) {
    using C = W16Cfg;
    const int64_t N = wgt.rows;
    CUtensorMap tmW, tmX;
    // activations: boxes of 16 rows x 64 columns (128 bytes) with the 128-byte
    // swizzle the MMA's B operand descriptor expects; rows past M read as zero
    if (encode_tensor_map_u8(&tmW, wgt.codes, K / 2, N, 128, 128) != CUDA_SUCCESS ||
        encode_output_map_bf16(&tmX, const_cast<void *>(x), static_cast<uint64_t>(M), static_cast<uint64_t>(K),
                               static_cast<uint64_t>(ldx), 64, C::kN) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    W16Args a;
    a.sfw = wgt.scales;
    a.gw = wgt.g;
    a.y = y;
    a.ldy = ldy;
    a.M = static_cast<int32_t>(M);
    a.N = static_cast<int32_t>(N);
    a.K = static_cast<int32_t>(K);
    a.num_wt = static_cast<int32_t>(ceil_div(N, 128));
    a.num_xt = static_cast<int32_t>(ceil_div(M, C::kN));
    a.status = status;
    a.timeout_ns = timeout_ns;
    const int64_t tiles = static_cast<int64_t>(a.num_wt) * a.num_xt;
    auto kern = y_bf16 ? gemm_w4a16_kernel<__nv_bfloat16> : gemm_w4a16_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles < num_sms ? tiles : num_sms));
    cfg.blockDim = dim3(C::kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tmW, tmX, a);
}

}  // namespace nvfp4
