// kernels.cuh -- host launchers of the CUDA kernels (internal to the library).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace nvfp4 {

// With grid_bar and status (a workspace's meeting point and status word),
// large contiguous tensors take the one-read cooperative quantizer
// (quantize_onepass_usable); otherwise the two passes run.
cudaError_t launch_quantize(const void *x, bool bf16, int64_t rows, int64_t cols, int64_t ld,
                            uint8_t *codes, uint8_t *scales, float *g_out, float *partials,
                            int num_sms, cudaStream_t stream, uint32_t *grid_bar = nullptr,
                            uint32_t *status = nullptr, uint64_t timeout_ns = 0);
bool quantize_onepass_usable(int64_t rows, int64_t cols, int64_t ld, bool bf16);
cudaError_t launch_quantize_onepass(const void *x, bool bf16, int64_t rows, int64_t cols, uint8_t *codes,
                                    uint8_t *scales, float *g_out, float *partials, uint32_t *grid_bar,
                                    uint32_t *status, uint64_t timeout_ns, int num_sms, cudaStream_t stream);

cudaError_t launch_dequantize(const uint8_t *codes, const uint8_t *scales, const float *g,
                              int64_t rows, int64_t cols, void *y, bool bf16, int64_t ldy,
                              int num_sms, cudaStream_t stream, uint32_t *status = nullptr);

// One GEMM operand as the GEMM kernel reads it.
struct Operand {
    const uint8_t *codes;    // [rows][K/2]
    const uint8_t *scales;   // tiled layout
    const float *g;          // tensor scale (device); null for MXFP4 operands
    int64_t rows;
};

// y[M][N] = (A . B^T) * gA * gB, A = act [M][K], B = wgt [N][K].
// weights_ready: the weights were not written by the kernel launched just
// before (they may be streamed before the programmatic-dependent-launch wait).
// splitk_ws: splitk_ws_bytes(M, N) bytes of scratch (or null: no stream-K);
// any contents (the kernel zero-fills what it uses).  With it, `status` must
// be the workspace's start: the stream-K CTAs meet at the header's meeting
// point.
// ymax_part (optional): every CTA writes the largest |y| it stored (the value
// as stored, after rounding to y's dtype) to ymax_part[blockIdx.x], the
// quantizer's first-pass format; *nparts receives the grid size (<= 4096).
cudaError_t launch_gemm(const Operand &act, const Operand &wgt, int64_t K, void *y, bool y_bf16,
                        int64_t ldy, uint32_t *status, uint64_t timeout_ns, int num_sms,
                        cudaStream_t stream, bool weights_ready = false, void *splitk_ws = nullptr,
                        float *ymax_part = nullptr, int *nparts = nullptr);

// Bytes of stream-K scratch a GEMM of M activation rows and N weight rows may use (0: never).
size_t splitk_ws_bytes(int64_t M, int64_t N);

// Two-CTA (cta_group::2) GEMM for large M: usable when enough 256x256 tiles
// exist to fill the GPU with CTA pairs.
bool pair_gemm_usable(int64_t M, int64_t N, int num_sms);
// fmt: kFmtNV, kFmtMX (MXFP4 operands) or kFmtW4A8 (MXFP8 activations, MXFP4
// weights read by the unpacking copy; K % 128 == 0).
cudaError_t launch_gemm_pair(const Operand &act, const Operand &wgt, int64_t K, void *y, bool y_bf16,
                             int64_t ldy, uint32_t *status, uint64_t timeout_ns, cudaStream_t stream,
                             float *ymax_part = nullptr, int *nparts = nullptr, int fmt = 0);

// y[M][N] = A . B^T for MXFP4 operands (E2M1 codes, UE8M0 scales per 32
// elements in the tiled layout with 32-element blocks, no tensor scales).
cudaError_t launch_gemm_mx(const Operand &act, const Operand &wgt, int64_t K, void *y, bool y_bf16,
                           int64_t ldy, uint32_t *status, uint64_t timeout_ns, int num_sms,
                           cudaStream_t stream, void *splitk_ws);

// W4A16: y[M][N] = x . dequant(wgt)^T * gw with bf16 activations x [M][K]
// (pitch ldx) and NVFP4 weights dequantized exactly to bf16 (e * s) inside
// the kernel, bf16 tensor cores, fp32 accumulation.
cudaError_t launch_gemm_w4a16(const void *x, int64_t M, int64_t K, int64_t ldx, const Operand &wgt, void *y,
                              bool y_bf16, int64_t ldy, uint32_t *status, uint64_t timeout_ns, int num_sms,
                              cudaStream_t stream);

// W4A8: y[M][N] = A . B^T with MXFP8 activations (E4M3 bytes [M][K], UE8M0
// scales per 32, tiled) and MXFP4 weights, kind::mxf8f6f4 (one-CTA kernel).
cudaError_t launch_gemm_w4a8(const Operand &act, const Operand &wgt, int64_t K, void *y, bool y_bf16,
                             int64_t ldy, uint32_t *status, uint64_t timeout_ns, int num_sms,
                             cudaStream_t stream, bool weights_ready, void *splitk_ws);

// Tensor map over packed E2M1 rows that unpacks them into the 8-bit-container
// shared-memory form (16 values per 16-byte chunk), boxes of 128 values.
CUresult encode_tensor_map_fp4_unpacked(CUtensorMap *map, const void *base, uint64_t k_elems, uint64_t rows,
                                        uint32_t box_rows);

// MXFP8 quantizer (one pass): E4M3 bytes [rows][cols], UE8M0 scales tiled.
cudaError_t launch_mx8_quantize(const void *x, bool bf16, int64_t rows, int64_t cols, int64_t ld, uint8_t *elems,
                                uint8_t *scales, int num_sms, cudaStream_t stream);

// MXFP4 quantizer (one pass): codes [rows][cols/2], UE8M0 scales tiled.
cudaError_t launch_mx_quantize(const void *x, bool bf16, int64_t rows, int64_t cols, int64_t ld, uint8_t *codes,
                               uint8_t *scales, int num_sms, cudaStream_t stream);

// The quantizer's second pass alone, on fp32 x whose first pass (max |x| per
// part, num_partials values) was produced elsewhere.
// status: the workspace status word (the debug build's store checks record
// there), or null.
cudaError_t launch_encode_f32(const float *x, int64_t rows, int64_t cols, int64_t ld, const float *partials,
                              int num_partials, uint8_t *codes, uint8_t *scales, float *g_out, int num_sms,
                              cudaStream_t stream, uint32_t *status = nullptr);
// The quantizer's first pass on its own: *amax = max |x| (device fp32), via
// per-CTA partial maxima (at most kMaxAmaxPartials floats of scratch).
cudaError_t launch_amax(const void *x, bool bf16, int64_t rows, int64_t cols, int64_t ld, float *partials,
                        float *amax, int num_sms, cudaStream_t stream);
// The same for bf16 or fp32 x.
cudaError_t launch_encode(const void *x, bool bf16, int64_t rows, int64_t cols, int64_t ld, const float *partials,
                          int num_partials, uint8_t *codes, uint8_t *scales, float *g_out, int num_sms,
                          cudaStream_t stream, uint32_t *status = nullptr);

// h[M][N] = SiLU(x wg^T * gx*gwg) * (x wu^T * gx*gwu) in fp32 (128x128 tiles,
// both products per tile), and max |h| per CTA into partials (the quantizer's
// first-pass format); *num_partials receives how many were written
// (<= max_partials).
// h_q non-null: the fused form (one tile per CTA, cooperative launch; see
// dual_fused_requant_usable) re-quantizes h in the epilogue; h may then be null.
// grid_bar: the two-word grid meeting point (see grid_meet), zero-filled once.
cudaError_t launch_gemm_dual_silu(const Operand &act, const Operand &wg, const Operand &wu, int64_t K,
                                  float *h, int64_t ldh, float *partials, int max_partials, int *num_partials,
                                  uint32_t *status, uint64_t timeout_ns, int num_sms, cudaStream_t stream,
                                  bool weights_ready, uint8_t *hq_codes, uint8_t *hq_scales, float *hq_g,
                                  uint32_t *grid_bar);
bool dual_fused_requant_usable(int64_t M, int64_t N, int num_sms, int max_partials);


// The W4A4 linear layer for M <= 16 activation rows with the activation
// quantizer inside the GEMM (gemm_decode.cu): x [M][K] (bf16 or fp32, pitch
// ldx) is quantized by every CTA, y [M][N] = x_q . wgt^T * gx * gw; if
// xq_codes is not null, x_q (codes, tiled scales, tensor scale) is written too.
bool decode_fused_usable(int64_t M, int64_t N, int64_t K);
cudaError_t launch_gemm_decode(const void *x, bool x_bf16, int64_t M, int64_t K, int64_t ldx, const Operand &wgt,
                               void *y, bool y_bf16, int64_t ldy, uint8_t *xq_codes, uint8_t *xq_scales,
                               float *xq_g, uint32_t *status, uint64_t timeout_ns, int num_sms,
                               cudaStream_t stream, float *ymax_part = nullptr, int *nparts = nullptr);

cudaError_t launch_wait_selftest(uint32_t *status, uint64_t timeout_ns, cudaStream_t stream);

// Bound of every device-side wait of the next launches, in nanoseconds (set
// through nvfp4_set_wait_timeout_us).
uint64_t wait_timeout_ns();

// cuTensorMapEncodeTiled through the runtime's driver entry point.
CUresult encode_tensor_map_u8(CUtensorMap *map, const void *base, uint64_t inner_bytes,
                              uint64_t rows, uint32_t box_inner, uint32_t box_rows);

// Tensor map over a tiled scale array: [row_tiles][k_steps][512-byte atom],
// box = box_atoms atoms x box_tiles row tiles (zero fill past either edge).
CUresult encode_scale_map(CUtensorMap *map, const void *scales, uint64_t k_steps, uint64_t row_tiles,
                          uint32_t box_tiles, uint32_t box_atoms = 4);

// Tensor map over a bf16 output y[rows][cols] with row pitch ld elements,
// 128-byte swizzled boxes of box_rows x box_cols (box_cols * 2 <= 128).
CUresult encode_output_map_bf16(CUtensorMap *map, void *y, uint64_t rows, uint64_t cols, uint64_t ld,
                                uint32_t box_cols, uint32_t box_rows);

}  // namespace nvfp4
