/*
 * nvfp4.h -- C ABI of the B200 (sm_100a) NVFP4 library: quantize, dequantize,
 * block-scaled W4A4 GEMM and the fused linear / MLP step.
 *
 * The format (NVFP4 wiki page, newton.com.tw, section "技術原理"): each value
 * is a 4-bit E2M1 element (1 sign, 2 exponent, 1 mantissa bit; magnitudes
 * 0, 0.5, 1, 1.5, 2, 3, 4, 6); every 16 consecutive values along a row share
 * one E4M3 FP8 block scale; one FP32 scale covers the whole tensor.  That is
 * about 4.5 bits per value.
 *
 * The GEMM consumes NVFP4 weights AND NVFP4 activations directly on the
 * block-scaled FP4 tensor cores, with no dequantize-to-16-bit step (aixq.cc
 * article on Unsloth Dynamic NVFP4, section "核心差异：W4A4 vs W4A16").
 *
 * Arithmetic (the pages give the structure; these are the rules):
 *   tensor scale   g = fl32(amax / 2688)                 (2688 = 6 * 448)
 *   block scale    s = E4M3_rne_satfinite(fl32(bamax / fl32(6 * g)))  (g==0: s=0)
 *   element        d = fl32(dec(s) * g); r = fl32(1/d); v = fl32(x * r);
 *                  code = E2M1_rne_satfinite(v) (ties to the even magnitude
 *                  index; sign kept for values that round to zero);
 *                  a block with d == 0 or 1/d == inf has all codes 0.
 *   dequantize     y = fl32(fl32(e * dec(s)) * g)
 *   GEMM           y[m][n] = fl32(acc[m][n] * fl32(gA * gB)),
 *                  acc = sum_k (eA*sA)(eB*sB) accumulated in fp32 by the tensor
 *                  cores; bf16 output is the RNE rounding of that fp32 value.
 *
 * Conventions for every entry point:
 *   - All pointers are DEVICE pointers owned by the caller, 16-byte aligned.
 *     Row pitches (ld, in elements) must keep every row 16-byte aligned.  An
 *     empty matrix (a zero dimension) is never read or written: its data
 *     pointer may be NULL and its pointer and pitch are not checked (a pitch
 *     must still be at least the row length).
 *   - Calls are asynchronous and stream-ordered on `stream`; none allocates
 *     memory and none synchronises, except nvfp4_get_device_status.
 *   - Argument errors are returned synchronously and launch nothing.
 *     NVFP4_ERR_CUDA wraps a failed launch (the CUDA error is left for
 *     cudaGetLastError).  Device-side give-ups (a bounded wait that ran out)
 *     are OR-ed into the status word at the start of the workspace and read by
 *     nvfp4_get_device_status.
 *   - Requires a compute-capability 10.0 GPU (B200); NVFP4_ERR_ARCH otherwise.
 *     There is no CPU fallback.
 *   - Workspace: `ws` points to at least nvfp4_workspace_bytes(...) bytes of
 *     device memory.  Zero-fill it once after allocating; the library keeps a
 *     sticky status word in its first 16 bytes and the grid-wide meeting
 *     point of its cooperative kernels at bytes 128..135 (back at zero after
 *     every completed call), and uses the rest as scratch.  After a device-side
 *     give-up (NVFP4_ERR_TIMEOUT) zero-fill it again before reusing it.
 *     GEMMs with few output tiles split K across SMs and add fp32 partial
 *     sums in the scratch (zero-filled by the call itself, so workspaces may
 *     be shared between operations and shapes that do not overlap in time).
 *     Calls that share one workspace must not overlap on the GPU.
 *   - Kernel choice is automatic.  Environment switches, read at each call,
 *     exist for A/B measurements: NVFP4_GEMM_CTA_PAIR=0 keeps large-M GEMMs
 *     on the one-CTA kernel; NVFP4_GEMM_STREAMK=0 disables the split-K
 *     (stream-K) path for GEMMs with few output tiles (a cooperative launch
 *     of one CTA per SM: a context limited to fewer SMs than the device has
 *     gets NVFP4_ERR_CUDA from it and should set this); NVFP4_DECODE_FUSED=1
 *     runs nvfp4_linear_fused's STORE form for M <= 16 as one kernel that
 *     quantizes x itself; NVFP4_MLP_FUSED_REQUANT=0 keeps the SiLU form's
 *     re-quantization of h in a separate encode pass (by default the gate/up
 *     kernel does it in its epilogue when its tiles fit one per SM);
 *     NVFP4_QUANTIZE_ONEPASS=1 quantizes large contiguous tensors with one
 *     cooperative kernel that reads x once (slower than the two passes on
 *     B200 as measured; kept for A/B runs).
 *     Results stay within the same tolerance either way (x_q and y_q
 *     bit-identical).
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                      /* same type as cudaStream_t */
typedef struct CUstream_st *nvfp4_stream_t;

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,           /* NULL pointer, negative size, mismatched shapes */
    NVFP4_ERR_UNSUPPORTED_SHAPE = 2,     /* cols % 16 (quantize) or K % 64 (GEMM) not 0; a GEMM
                                            with M or N above 2^30 - 1 or K above 2^31 (the
                                            kernels' 32-bit row and tile-coordinate range) */
    NVFP4_ERR_MISALIGNED = 3,            /* a pointer or row pitch not 16-byte aligned */
    NVFP4_ERR_WORKSPACE = 4,             /* ws NULL or smaller than required */
    NVFP4_ERR_CUDA = 5,                  /* a CUDA runtime/driver call or launch failed */
    NVFP4_ERR_TIMEOUT = 6,               /* a device-side bounded wait gave up */
    NVFP4_ERR_ARCH = 7,                  /* current device is not sm_100 */
    NVFP4_ERR_BOUNDS = 8                 /* debug build only (libnvfp4_debug.so): a kernel's store
                                            fell outside its buffer and was skipped */
} nvfp4_status;

typedef enum {
    NVFP4_F32 = 0,
    NVFP4_BF16 = 1
} nvfp4_dtype;

typedef enum {
    NVFP4_OP_QUANTIZE = 0,
    NVFP4_OP_DEQUANTIZE = 1,
    NVFP4_OP_GEMM = 2,
    NVFP4_OP_LINEAR_FUSED = 3,           /* nvfp4_linear_fused with NVFP4_EPI_STORE */
    NVFP4_OP_LINEAR_FUSED_SILU = 4,      /* nvfp4_linear_fused with NVFP4_EPI_SILU_MUL_REQUANT */
    NVFP4_OP_GEMM_REQUANT = 5,           /* nvfp4_gemm_requant */
    NVFP4_OP_W4A16 = 6,                  /* nvfp4_w4a16_linear (the status word only) */
    NVFP4_OP_W4A8_LINEAR = 7             /* nvfp4_w4a8_linear */
} nvfp4_op;

typedef enum {
    NVFP4_EPI_STORE = 0,                 /* y = x_q . w_q^T * gx * gw */
    NVFP4_EPI_SILU_MUL_REQUANT = 1       /* h = SiLU(x.w^T) * (x.w_up^T), quantized to NVFP4 */
} nvfp4_epilogue;

/*
 * One NVFP4 tensor [rows][cols], quantized along cols (the GEMM's K).
 *   codes        [rows][cols/2] bytes; byte j of a row holds element 2j in its
 *                low nibble and element 2j+1 in its high nibble; sign in bit 3.
 *   scales       E4M3 block scales in the tiled layout the tensor cores read:
 *                rows padded to R128 = roundup(rows,128), blocks per row padded
 *                to KB4 = roundup(cols/16, 4).  The scale of block kb of row r
 *                is the byte at
 *                  ((r/128)*(KB4/4) + kb/4)*512 + (r%32)*16 + ((r/32)%4)*4 + kb%4
 *                so each 128-row x 64-column slab is one contiguous 512-byte
 *                atom.  Padding bytes are written as 0 by nvfp4_quantize.
 *                Size: nvfp4_scales_bytes(rows, cols).
 *   tensor_scale one fp32 in device memory: g = amax / 2688.
 */
typedef struct {
    uint8_t *codes;
    uint8_t *scales;
    float *tensor_scale;
    int64_t rows;
    int64_t cols;
} nvfp4_tensor;

/* Bytes of the packed codes: rows * cols / 2. */
NVFP4_API size_t nvfp4_codes_bytes(int64_t rows, int64_t cols);

/* Bytes of the tiled scale array: roundup(rows,128) * roundup(cols/16,4). */
NVFP4_API size_t nvfp4_scales_bytes(int64_t rows, int64_t cols);

/* Workspace bytes an operation needs for the given shape (M rows of
 * activations, N rows of weights, K reduction length; quantize/dequantize use
 * M = rows, K = cols).  Always at least 256 (the status word). */
NVFP4_API size_t nvfp4_workspace_bytes(nvfp4_op op, int64_t M, int64_t N, int64_t K);

/*
 * Quantize x [rows][cols] (row pitch ld elements, dtype xt) to NVFP4 into
 * `out` (out->rows == rows, out->cols == cols, cols % 16 == 0).
 * Two passes: a reduction of the tensor amax into per-CTA partial maxima in
 * ws, then a pass that derives g on the device (no host synchronisation),
 * writes *out->tensor_scale, and encodes each 16-element block.
 * NVFP4 wiki page, section "技術原理" (two-level microblock scaling).
 */
NVFP4_API nvfp4_status nvfp4_quantize(const void *x, nvfp4_dtype xt, int64_t rows, int64_t cols,
                            int64_t ld, const nvfp4_tensor *out, void *ws, size_t ws_bytes,
                            nvfp4_stream_t stream);

/*
 * The quantizer's two halves for a tensor split across GPUs by rows (tensor
 * parallelism).  Every NVFP4 tensor has one FP32 tensor scale over all of it
 * (NVFP4 wiki page, section "技術原理"), so the ranks holding parts of one
 * tensor must agree on its amax before any block is encoded:
 *   nvfp4_amax                 *amax = max |x| over this rank's rows (one
 *                              fp32 in device memory; the first pass of
 *                              nvfp4_quantize, reduced on the device);
 *   (the caller all-reduces the ranks' amax with MAX: one float);
 *   nvfp4_quantize_with_amax   nvfp4_quantize's second pass with g =
 *                              fl32(*amax / 2688) from the given amax instead
 *                              of this rank's own.
 * The codes and scales of each rank's rows then equal those of the same rows
 * of the whole tensor quantized at once, and every rank's tensor_scale is
 * the whole tensor's.  Arguments, alignment and errors as nvfp4_quantize;
 * `amax` is one fp32 of device memory owned by the caller (4-byte aligned,
 * else NVFP4_ERR_MISALIGNED; null: NVFP4_ERR_INVALID_ARG); ws as for
 * NVFP4_OP_QUANTIZE (nvfp4_amax keeps its partial maxima there).
 * An empty x gives *amax = 0 (nvfp4_amax) and still writes tensor_scale
 * (nvfp4_quantize_with_amax).
 */
NVFP4_API nvfp4_status nvfp4_amax(const void *x, nvfp4_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                                  float *amax, void *ws, size_t ws_bytes, nvfp4_stream_t stream);
NVFP4_API nvfp4_status nvfp4_quantize_with_amax(const void *x, nvfp4_dtype xt, int64_t rows, int64_t cols,
                                                int64_t ld, const float *amax, const nvfp4_tensor *out,
                                                void *ws, size_t ws_bytes, nvfp4_stream_t stream);

/*
 * Dequantize q into y [q->rows][q->cols] (row pitch ldy elements, dtype yt):
 * y = fl32(fl32(e * dec(s)) * g), rounded to bf16 by RNE when yt is BF16.
 * This is the decode step a W4A16 path would run before a 16-bit GEMM
 * (aixq.cc article, section "核心差异：W4A4 vs W4A16"); here it is an
 * inspection / interoperability path, not part of the GEMM.
 */
NVFP4_API nvfp4_status nvfp4_dequantize(const nvfp4_tensor *q, void *y, nvfp4_dtype yt, int64_t ldy,
                              nvfp4_stream_t stream);

/*
 * y[M][N] = (A . B^T) * gA * gB with A = a [M][K], B = b [N][K] (K = a->cols
 * = b->cols, K % 64 == 0), both NVFP4, consumed directly by tcgen05
 * block-scaled FP4 MMAs with fp32 accumulation in tensor memory.  y has row
 * pitch ldy (elements) and dtype yt (BF16 or F32); y may be NULL when M*N == 0
 * (nothing is written), and K == 0 zero-fills y.  W4A4 linear layer: a is
 * the activations, b the weights.  Both operands stay 4-bit all the way into
 * the tensor cores, with no dequantize-to-16-bit step (aixq.cc article on
 * Unsloth Dynamic NVFP4, section "核心差异：W4A4 vs W4A16"); the tensor
 * cores apply the E4M3 block scales themselves and the two FP32 tensor scales
 * are applied once per output (NVFP4 wiki page, section "技術原理").
 */
NVFP4_API nvfp4_status nvfp4_gemm(const nvfp4_tensor *a, const nvfp4_tensor *b, void *y, nvfp4_dtype yt,
                        int64_t ldy, void *ws, size_t ws_bytes, nvfp4_stream_t stream);

/*
 * nvfp4_gemm, and the output re-quantized to NVFP4 for the next layer:
 * y_q (y_q->rows == M, y_q->cols == N, N % 16 == 0) receives y AS STORED
 * (after rounding to y's dtype) quantized with the rules above, with its own
 * tensor scale over all of y -- the same bytes nvfp4_quantize(y) would give.
 * Every NVFP4 tensor carries its own two-level scaling (NVFP4 wiki page,
 * section "技術原理"), so the next layer's activations get a fresh tensor
 * scale.  The GEMM's epilogue records the largest |y| each CTA stores, so
 * only the quantizer's encode pass runs afterwards (one more read of y).
 * K == 0 gives y = 0 and an all-zero y_q with g = 0; M == 0 or N == 0 writes
 * only y_q's g (0).  Workspace: nvfp4_workspace_bytes(NVFP4_OP_GEMM_REQUANT, ...).
 */
NVFP4_API nvfp4_status nvfp4_gemm_requant(const nvfp4_tensor *a, const nvfp4_tensor *b, void *y, nvfp4_dtype yt,
                                          int64_t ldy, const nvfp4_tensor *y_q, void *ws, size_t ws_bytes,
                                          nvfp4_stream_t stream);

/*
 * The W4A4 linear layer from high-precision activations (aixq.cc article on
 * Unsloth Dynamic NVFP4, section "核心差异：W4A4 vs W4A16": weights and
 * activations both 4-bit, straight into the FP4 tensor cores).
 *   x [M][K] (pitch ldx, dtype xt) is quantized to NVFP4 on the device on
 *   every call, its scales derived from this call's values (the mobdome post
 *   on Qwen3.6-27B-NVFP4, section "第二層：動態縮放（Dynamic Scaling）"), then
 *   multiplied with the pre-quantized weights.
 *   epilogue == NVFP4_EPI_STORE: y [M][w->rows] = x_q . w^T * gx * gw
 *     (w_up ignored; y required, dtype yt, pitch ldy).  If y_q is not NULL,
 *     y as stored is also quantized to NVFP4 into y_q (y_q->rows == M,
 *     y_q->cols == w->rows, a multiple of 16), with its own tensor scale, as
 *     nvfp4_gemm_requant does; K == 0 then gives an all-zero y_q, N == 0 only
 *     its g (0).  For M <= 16 (decode) the activation quantizer runs inside
 *     the GEMM kernel, one launch per call (two with y_q).
 *   epilogue == NVFP4_EPI_SILU_MUL_REQUANT: gate = x_q . w^T, up = x_q . w_up^T
 *     (w_up->rows == w->rows), h = SiLU(gate) * up in fp32, SiLU(z) =
 *     z / (1 + exp(-z)); h is quantized to NVFP4 into y_q (y_q->rows == M,
 *     y_q->cols == w->rows) with its own tensor scale over all of h, ready to be
 *     the activation operand of the next (down-projection) nvfp4_gemm.  If y is
 *     not NULL it receives h itself in fp32 (yt must be F32), for inspection.
 *   If x_q is not NULL it receives the quantized activations (x_q->rows == M,
 *   x_q->cols == K); otherwise they live in ws.
 *   K == 0 is an empty reduction: the STORE form zero-fills y; the SiLU form
 *   gives h = 0, so y_q gets zero codes and scales and g = 0 (and y, if
 *   given, zeros).  M == 0 writes nothing; N == 0 writes only y_q's g (0).
 */
NVFP4_API nvfp4_status nvfp4_linear_fused(const void *x, nvfp4_dtype xt, int64_t M, int64_t K, int64_t ldx,
                                const nvfp4_tensor *w, const nvfp4_tensor *w_up,
                                nvfp4_epilogue epilogue, void *y, nvfp4_dtype yt, int64_t ldy,
                                const nvfp4_tensor *y_q, const nvfp4_tensor *x_q,
                                void *ws, size_t ws_bytes, nvfp4_stream_t stream);

/*
 * nvfp4_linear_noalloc: the same W4A4 linear layer as nvfp4_linear_fused with
 * NVFP4_EPI_STORE (quantize x on the device, then y = x_q . w^T * gx * gw),
 * for callers that cannot allocate device memory and so cannot pass a
 * workspace: a plugin whose host framework's caching allocator owns every
 * device byte and forbids raw cudaMalloc, a runtime whose memory plan is fixed
 * before it runs, a latency-critical loop that must not risk the implicit
 * device synchronisation of cudaMalloc/cudaFree, or a foreign-language caller
 * that only holds pointers it was given.  The pages have no counterpart: this
 * is an interface convenience, not part of the method.
 *   Scratch: one 4 MiB file-scope __device__ array inside the library, held on
 *   every GPU that loads the library until the process exits.  It carries the
 *   status word, the quantizer's partial maxima and the quantized activations,
 *   so M * K/2 + roundup(M,128) * roundup(K/16,4) must stay within about
 *   4 MiB - 17 KiB (about 1.3k rows at K = 5120); larger shapes are rejected
 *   with NVFP4_ERR_UNSUPPORTED_SHAPE and nothing is launched.
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.  The address is kept for the rest of the
 *   process: call from the device's primary context (the CUDA runtime's) only,
 *   and not after a cudaDeviceReset, after which the array may sit elsewhere.
 *   Every call shares the one array and finds the previous call's contents in
 *   it: calls that overlap on the GPU race on it.  Each call clears the status
 *   word first and rewrites everything else.  Device-side waits give up after
 *   the bound set by nvfp4_set_wait_timeout_us, like every other entry
 *   point's; there is no status readback for this entry point (use
 *   nvfp4_linear_fused with a workspace to observe one).
 *   Other arguments, layouts and errors as nvfp4_linear_fused; allocates
 *   nothing (no cudaMalloc, cudaFree or allocating library routine).
 */
NVFP4_API nvfp4_status nvfp4_linear_noalloc(const void *x, nvfp4_dtype xt, int64_t M, int64_t K,
                                            int64_t ldx, const nvfp4_tensor *w, void *y,
                                            nvfp4_dtype yt, int64_t ldy, nvfp4_stream_t stream);

/*
 * MXFP4 (eefocus.com article on FP4 vs INT4, section
 * "FP4被视为下一代AI计算的核心标准"; the OCP MX format): E2M1 elements, 32
 * consecutive elements along a row share one E8M0 scale (a power of two),
 * about 4.25 bits per value, no second-level tensor scale.
 *   scale   X = 2^e, e = ceil(log2(bamax / 6)) clamped to [-127, 127]: the
 *           smallest power of two with bamax <= 6 X (an all-zero block gets
 *           byte 0); the page gives no rule, this one never saturates.
 *   element code = E2M1_rne_satfinite(x / X) (exact division), with the NVFP4
 *           tie and sign rules.
 * Layout as nvfp4_tensor, with kb counting 32-element blocks: scale byte of
 * block kb of row r at ((r/128)*(KB4/4) + kb/4)*512 + (r%32)*16 +
 * ((r/32)%4)*4 + kb%4, KB4 = roundup(cols/32, 4); one 512-byte atom covers
 * 128 rows x 128 columns.
 */
typedef struct {
    uint8_t *codes;                      /* [rows][cols/2], element 2j in the low nibble of byte j */
    uint8_t *scales;                     /* nvfp4_mx_scales_bytes(rows, cols) bytes, tiled as above */
    int64_t rows;
    int64_t cols;                        /* a multiple of 32 */
} nvfp4_mx_tensor;

/* Bytes of the tiled MXFP4 scale array: roundup(rows,128) * roundup(cols/32,4). */
NVFP4_API size_t nvfp4_mx_scales_bytes(int64_t rows, int64_t cols);

/*
 * Quantize x [rows][cols] (pitch ld elements, dtype xt; cols % 32 == 0) to
 * MXFP4 into out.  One pass (no tensor amax, no workspace); padding of the
 * scale layout is written as 0.
 */
NVFP4_API nvfp4_status nvfp4_mx_quantize(const void *x, nvfp4_dtype xt, int64_t rows, int64_t cols,
                                         int64_t ld, const nvfp4_mx_tensor *out, nvfp4_stream_t stream);

/*
 * y[M][N] = A . B^T for MXFP4 A [M][K] and B [N][K] (K % 64 == 0) on the
 * block-scaled FP4 tensor cores (kind::mxf4, one UE8M0 scale per 32
 * elements), fp32 accumulation; kernels, output dtypes, pitches and
 * workspace (nvfp4_workspace_bytes(NVFP4_OP_GEMM, M, N, K)) as nvfp4_gemm.
 */
NVFP4_API nvfp4_status nvfp4_mx_gemm(const nvfp4_mx_tensor *a, const nvfp4_mx_tensor *b, void *y, nvfp4_dtype yt,
                                     int64_t ldy, void *ws, size_t ws_bytes, nvfp4_stream_t stream);

/*
 * W4A8: FP4 weights times FP8 activations, the eefocus.com article's W4A8
 * (the Zhouyi X3 passage: weights quantized to FP4, activations to FP8).  On
 * B200 the native mixed FP4 x FP8 tensor-core product is block-scaled with one
 * UE8M0 scale per 32 elements on both operands (kind::mxf8f6f4), so the
 * weights are MXFP4 (nvfp4_mx_tensor) and the activations MXFP8:
 *   scale   X = 2^e, e = ceil(log2(bamax / 448)) clamped to [-127, 127]: the
 *           smallest power of two with bamax <= 448 X (an all-zero block gets
 *           byte 0); the page gives no rule, this one never saturates.
 *   element E4M3 (OCP "fn") RNE of x / X (exact division), sign kept.
 * Layout: elements [rows][cols] one byte each, scales tiled as MXFP4's.
 */
typedef struct {
    uint8_t *elems;                      /* [rows][cols] E4M3 bytes */
    uint8_t *scales;                     /* nvfp4_mx_scales_bytes(rows, cols) bytes, tiled */
    int64_t rows;
    int64_t cols;                        /* a multiple of 32 */
} nvfp4_mx8_tensor;

/* Quantize x [rows][cols] (pitch ld, dtype xt; cols % 32 == 0) to MXFP8; one pass. */
NVFP4_API nvfp4_status nvfp4_mx8_quantize(const void *x, nvfp4_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                                          const nvfp4_mx8_tensor *out, nvfp4_stream_t stream);

/*
 * y[M][N] = A . B^T with MXFP8 activations A [M][K] and MXFP4 weights B [N][K]
 * (K % 128 == 0, else NVFP4_ERR_UNSUPPORTED_SHAPE: the copy that unpacks the
 * weights into 8-bit shared-memory containers moves 128 values per row; the
 * weights' codes 32-byte aligned, else NVFP4_ERR_MISALIGNED) on the block-scaled
 * tensor cores (kind::mxf8f6f4, fp32 accumulation; no tensor scales).  Output
 * dtypes, pitches and workspace (nvfp4_workspace_bytes(NVFP4_OP_GEMM, ...)) as
 * nvfp4_gemm.
 */
NVFP4_API nvfp4_status nvfp4_w4a8_gemm(const nvfp4_mx8_tensor *a, const nvfp4_mx_tensor *b, void *y, nvfp4_dtype yt,
                                       int64_t ldy, void *ws, size_t ws_bytes, nvfp4_stream_t stream);

/*
 * The W4A8 linear layer from high-precision activations: x [M][K] (pitch ldx,
 * dtype xt) is quantized to MXFP8 on the device, then y = x_q . w^T as
 * nvfp4_w4a8_gemm (same K and alignment rules).  If x_q is not NULL it
 * receives the quantized activations.
 * Workspace: nvfp4_workspace_bytes(NVFP4_OP_W4A8_LINEAR, M, N, K).
 */
NVFP4_API nvfp4_status nvfp4_w4a8_linear(const void *x, nvfp4_dtype xt, int64_t M, int64_t K, int64_t ldx,
                                         const nvfp4_mx_tensor *w, void *y, nvfp4_dtype yt, int64_t ldy,
                                         const nvfp4_mx8_tensor *x_q, void *ws, size_t ws_bytes,
                                         nvfp4_stream_t stream);

/*
 * W4A16 linear layer: y[M][N] = x . deq(w)^T with 16-bit activations x
 * [M][K] (xt must be NVFP4_BF16, pitch ldx) and NVFP4 weights w [N][K]
 * (K % 64 == 0), the scheme the aixq.cc article on Unsloth Dynamic NVFP4
 * (section "核心差异：W4A4 vs W4A16") compares W4A4 against: the weights are
 * dequantized to 16 bits before a 16-bit matrix product.  Each weight value
 * e * s (E2M1 element times E4M3 block scale) is exact in bf16, so the
 * kernel dequantizes in registers straight into the tensor cores' operand
 * memory and applies the tensor scale to the fp32 accumulator:
 *   y = fl32(acc * g_w), acc = sum_k x[m][k] * (e*s)[n][k] accumulated in fp32,
 * then RNE to bf16 for a bf16 y.  Tiles of 128 weight rows x 16 activation
 * rows; larger M repeats the weight stream per 16 activation rows (the
 * decode-shaped path, not a prefill tile).  Workspace: the status word
 * (nvfp4_workspace_bytes(NVFP4_OP_W4A16, ...) = 256 bytes).
 */
NVFP4_API nvfp4_status nvfp4_w4a16_linear(const void *x, nvfp4_dtype xt, int64_t M, int64_t K, int64_t ldx,
                                          const nvfp4_tensor *w, void *y, nvfp4_dtype yt, int64_t ldy, void *ws,
                                          size_t ws_bytes, nvfp4_stream_t stream);

/*
 * Synchronise `stream`, read the sticky device status word in ws, clear it,
 * and return it (NVFP4_OK when no device-side wait gave up since the last
 * read).  Also returns NVFP4_ERR_CUDA if the stream reports an error.
 */
NVFP4_API nvfp4_status nvfp4_get_device_status(void *ws, nvfp4_stream_t stream);

/*
 * Launch one single-thread kernel that waits, with the library's bounded wait,
 * on a shared-memory barrier that nothing ever completes, giving up after
 * timeout_us microseconds.  The give-up path records NVFP4_ERR_TIMEOUT in the
 * status word of ws, exactly as a stalled pipeline stage of the GEMM would.
 * Used to test the failure-detection path without hanging a GPU.
 */
NVFP4_API nvfp4_status nvfp4_selftest_bounded_wait(void *ws, uint32_t timeout_us, nvfp4_stream_t stream);

/* Bound, in microseconds, of every device-side wait of later launches
 * (default 2,000,000).  Returns the previous value. */
NVFP4_API uint32_t nvfp4_set_wait_timeout_us(uint32_t timeout_us);

/* Human-readable name of a status code. */
NVFP4_API const char *nvfp4_status_string(nvfp4_status status);

/* Library version: major * 10000 + minor * 100 + patch. */
NVFP4_API int nvfp4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H */
