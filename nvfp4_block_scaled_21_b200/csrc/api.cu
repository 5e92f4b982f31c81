// api.cu -- the extern "C" boundary declared in include/nvfp4.h: argument
// validation (synchronous, no launch on error), workspace carving and the
// kernel launches.  No allocation, no synchronisation except in
// nvfp4_get_device_status.
#include <atomic>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "nvfp4.h"

using namespace nvfp4;

namespace {

std::atomic<uint32_t> g_wait_timeout_us{2000000u};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device properties of the current device, cached per device ordinal.
struct DevInfo {
    int sms = 0;
    int major = 0;
    int minor = 0;
};

nvfp4_status current_device(DevInfo *out) {
    static DevInfo cache[64];
    static std::atomic<bool> have[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return NVFP4_ERR_CUDA;
    if (dev < 64 && have[dev].load(std::memory_order_acquire)) {
        *out = cache[dev];
    } else {
        DevInfo d;
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        if (dev < 64) {
            // one writer per entry: a thread that lost the race leaves it alone
            static std::mutex fill;
            std::lock_guard<std::mutex> lock(fill);
            if (!have[dev].load(std::memory_order_relaxed)) {
                cache[dev] = d;
                have[dev].store(true, std::memory_order_release);
            }
        }
        *out = d;
    }
    if (out->major != 10 || out->minor != 0) return NVFP4_ERR_ARCH;
    return NVFP4_OK;
}

bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

nvfp4_status check_tensor(const nvfp4_tensor *t, int64_t rows, int64_t cols) {
    if (!t || !t->tensor_scale) return NVFP4_ERR_INVALID_ARG;
    if (t->rows != rows || t->cols != cols || rows < 0 || cols < 0) return NVFP4_ERR_INVALID_ARG;
    // an empty tensor may have NULL codes and scales (nothing is read or written)
    if (rows * cols != 0 && (!t->codes || !t->scales)) return NVFP4_ERR_INVALID_ARG;
    if (cols % kBlock) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(t->codes) || !aligned16(t->scales) || !aligned16(t->tensor_scale))
        return NVFP4_ERR_MISALIGNED;
    return NVFP4_OK;
}

nvfp4_status check_ws(void *ws, size_t ws_bytes, size_t need) {
    if (!ws || ws_bytes < need) return NVFP4_ERR_WORKSPACE;
    if (!aligned16(ws)) return NVFP4_ERR_MISALIGNED;
    return NVFP4_OK;
}

uint8_t *ws_at(void *ws, size_t off) { return static_cast<uint8_t *>(ws) + off; }

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Workspace carving (offsets in bytes).  The first kWsStatusBytes hold the
// status word (offset 0) and the grid meeting point of the cooperative
// kernels (offset 128: arrival count, generation; back at zero after every
// completed meeting).
constexpr size_t kPartialsOff = kWsStatusBytes;
constexpr size_t kPartialsBytes = kMaxAmaxPartials * sizeof(float);
constexpr size_t kQuantizeWs = kPartialsOff + kPartialsBytes;

size_t quantized_bytes(int64_t rows, int64_t cols) {
    return align256(static_cast<size_t>(rows * cols / 2)) +
           align256(static_cast<size_t>(round_up(rows, 128) * kb4_of(cols))) + 256;
}

nvfp4_status from_cuda(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

}  // namespace

namespace nvfp4 {
uint64_t wait_timeout_ns() { return static_cast<uint64_t>(g_wait_timeout_us.load()) * 1000ull; }
}  // namespace nvfp4

extern "C" {

size_t nvfp4_codes_bytes(int64_t rows, int64_t cols) {
    if (rows < 0 || cols < 0) return 0;
    return static_cast<size_t>(rows * cols / 2);
}

size_t nvfp4_scales_bytes(int64_t rows, int64_t cols) {
    if (rows < 0 || cols < 0) return 0;
    return static_cast<size_t>(round_up(rows, 128) * kb4_of(cols));
}

size_t nvfp4_workspace_bytes(nvfp4_op op, int64_t M, int64_t N, int64_t K) {
    if (M < 0 || N < 0 || K < 0) return 0;
    switch (op) {
    case NVFP4_OP_QUANTIZE:
        return kQuantizeWs;
    case NVFP4_OP_DEQUANTIZE:
        return kWsStatusBytes;
    case NVFP4_OP_GEMM:
        // status | stream-K scratch
        return kWsStatusBytes + splitk_ws_bytes(M, N);
    case NVFP4_OP_LINEAR_FUSED:
        // status, partials | x_q (codes, scales, g) | stream-K scratch
        return kQuantizeWs + quantized_bytes(M, K) + splitk_ws_bytes(M, N);
    case NVFP4_OP_LINEAR_FUSED_SILU:
        // status, partials | x_q | h (fp32 [M][N])
        return kQuantizeWs + quantized_bytes(M, K) + align256(static_cast<size_t>(M * N) * sizeof(float));
    case NVFP4_OP_GEMM_REQUANT:
        // status, partials (max |y| per GEMM CTA) | stream-K scratch
        return kQuantizeWs + splitk_ws_bytes(M, N);
    case NVFP4_OP_W4A16:
        return kWsStatusBytes;
    case NVFP4_OP_W4A8_LINEAR:
        // status | x_q (E4M3 bytes, scales) | stream-K scratch
        return kWsStatusBytes + align256(static_cast<size_t>(M * K)) + align256(nvfp4_mx_scales_bytes(M, K)) +
               splitk_ws_bytes(M, N);
    }
    return 0;
}

nvfp4_status nvfp4_quantize(const void *x, nvfp4_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                            const nvfp4_tensor *out, void *ws, size_t ws_bytes,
                            nvfp4_stream_t stream) {
    if ((!x && rows * cols != 0) || (xt != NVFP4_F32 && xt != NVFP4_BF16)) return NVFP4_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || ld < cols) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_tensor(out, rows, cols);
    if (st != NVFP4_OK) return st;
    const int eb = xt == NVFP4_BF16 ? 2 : 4;
    // an empty x is never read: its pointer and pitch are not checked
    if (rows * cols != 0 && (!aligned16(x) || (ld * eb) % 16)) return NVFP4_ERR_MISALIGNED;
    if ((st = check_ws(ws, ws_bytes, kQuantizeWs)) != NVFP4_OK) return st;
    DevInfo dev;
    if ((st = current_device(&dev)) != NVFP4_OK) return st;
    return from_cuda(launch_quantize(x, xt == NVFP4_BF16, rows, cols, ld, out->codes, out->scales,
                                     out->tensor_scale,
                                     reinterpret_cast<float *>(ws_at(ws, kPartialsOff)), dev.sms,
                                     reinterpret_cast<cudaStream_t>(stream),
                                     reinterpret_cast<uint32_t *>(ws_at(ws, kGridBarOff)),
                                     static_cast<uint32_t *>(ws), wait_timeout_ns()));
}

nvfp4_status nvfp4_amax(const void *x, nvfp4_dtype xt, int64_t rows, int64_t cols, int64_t ld, float *amax,
                        void *ws, size_t ws_bytes, nvfp4_stream_t stream) {
    if ((!x && rows * cols != 0) || !amax || (xt != NVFP4_F32 && xt != NVFP4_BF16)) return NVFP4_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || ld < cols) return NVFP4_ERR_INVALID_ARG;
    if (cols % 16) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    const int eb = xt == NVFP4_BF16 ? 2 : 4;
    if (rows * cols != 0 && (!aligned16(x) || (ld * eb) % 16)) return NVFP4_ERR_MISALIGNED;
    if (!aligned4(amax)) return NVFP4_ERR_MISALIGNED;
    nvfp4_status st = check_ws(ws, ws_bytes, kQuantizeWs);
    if (st != NVFP4_OK) return st;
    DevInfo dev;
    if ((st = current_device(&dev)) != NVFP4_OK) return st;
    return from_cuda(launch_amax(x, xt == NVFP4_BF16, rows, cols, ld,
                                 reinterpret_cast<float *>(ws_at(ws, kPartialsOff)), amax, dev.sms,
                                 reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_quantize_with_amax(const void *x, nvfp4_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                                      const float *amax, const nvfp4_tensor *out, void *ws, size_t ws_bytes,
                                      nvfp4_stream_t stream) {
    if ((!x && rows * cols != 0) || !amax || (xt != NVFP4_F32 && xt != NVFP4_BF16)) return NVFP4_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || ld < cols) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_tensor(out, rows, cols);
    if (st != NVFP4_OK) return st;
    const int eb = xt == NVFP4_BF16 ? 2 : 4;
    if (rows * cols != 0 && (!aligned16(x) || (ld * eb) % 16)) return NVFP4_ERR_MISALIGNED;
    if (!aligned4(amax)) return NVFP4_ERR_MISALIGNED;
    if ((st = check_ws(ws, ws_bytes, kQuantizeWs)) != NVFP4_OK) return st;
    DevInfo dev;
    if ((st = current_device(&dev)) != NVFP4_OK) return st;
    // the encode pass reduces its "partial maxima": here the one given amax
    return from_cuda(launch_encode(x, xt == NVFP4_BF16, rows, cols, ld, amax, 1, out->codes, out->scales,
                                   out->tensor_scale, dev.sms, reinterpret_cast<cudaStream_t>(stream),
                                   static_cast<uint32_t *>(ws)));
}

nvfp4_status nvfp4_dequantize(const nvfp4_tensor *q, void *y, nvfp4_dtype yt, int64_t ldy,
                              nvfp4_stream_t stream) {
    if (!q || (yt != NVFP4_F32 && yt != NVFP4_BF16)) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_tensor(q, q->rows, q->cols);
    if (st != NVFP4_OK) return st;
    const bool empty = q->rows * q->cols == 0;     // an empty y may be NULL, any pitch
    if (!y && !empty) return NVFP4_ERR_INVALID_ARG;
    const int eb = yt == NVFP4_BF16 ? 2 : 4;
    if (ldy < q->cols) return NVFP4_ERR_INVALID_ARG;
    if (!empty && (!aligned16(y) || (ldy * eb) % 16)) return NVFP4_ERR_MISALIGNED;
    DevInfo dev;
    if ((st = current_device(&dev)) != NVFP4_OK) return st;
    if (q->rows == 0 || q->cols == 0) return NVFP4_OK;
    return from_cuda(launch_dequantize(q->codes, q->scales, q->tensor_scale, q->rows, q->cols, y,
                                       yt == NVFP4_BF16, ldy, dev.sms,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

static nvfp4_status check_gemm(const nvfp4_tensor *a, const nvfp4_tensor *b, void *y,
                               nvfp4_dtype yt, int64_t ldy) {
    if (!a || !b || (yt != NVFP4_F32 && yt != NVFP4_BF16)) return NVFP4_ERR_INVALID_ARG;
    if (!y && a->rows * b->rows != 0) return NVFP4_ERR_INVALID_ARG;   // an empty y may be NULL
    if (a->cols != b->cols) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_tensor(a, a->rows, a->cols);
    if (st != NVFP4_OK) return st;
    if ((st = check_tensor(b, b->rows, b->cols)) != NVFP4_OK) return st;
    if (a->cols % 64) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (a->rows > kMaxGemmRows || b->rows > kMaxGemmRows || a->cols > kMaxGemmK)
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (ldy < b->rows) return NVFP4_ERR_INVALID_ARG;
    const int eb = yt == NVFP4_BF16 ? 2 : 4;
    if (a->rows * b->rows != 0 && (!aligned16(y) || (ldy * eb) % 16)) return NVFP4_ERR_MISALIGNED;
    return NVFP4_OK;
}

// An all-zero NVFP4 tensor: g = 0, and (when it has elements) zero codes and
// zero scales -- what the quantizer gives for an all-zero or empty input.
static nvfp4_status zero_quantized(const nvfp4_tensor *q, cudaStream_t stream) {
    if (cudaMemsetAsync(q->tensor_scale, 0, sizeof(float), stream) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (q->rows * q->cols == 0) return NVFP4_OK;
    if (cudaMemsetAsync(q->codes, 0, nvfp4_codes_bytes(q->rows, q->cols), stream) != cudaSuccess ||
        cudaMemsetAsync(q->scales, 0, nvfp4_scales_bytes(q->rows, q->cols), stream) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return NVFP4_OK;
}

// The quantizer's encode pass on y as stored, from the per-CTA maxima the
// GEMM's epilogue wrote: y_q gets its own tensor scale over all of y.
static nvfp4_status requant_output(const void *y, nvfp4_dtype yt, int64_t ldy, const nvfp4_tensor *y_q,
                                   const float *partials, int nparts, int num_sms, cudaStream_t stream,
                                   uint32_t *status) {
    return from_cuda(launch_encode(y, yt == NVFP4_BF16, y_q->rows, y_q->cols, ldy, partials, nparts,
                                   y_q->codes, y_q->scales, y_q->tensor_scale, num_sms, stream, status));
}

// weights_ready: b was not written by the kernel launched just before (true
// inside nvfp4_linear_fused, whose first kernel is launched without a
// programmatic dependency, so every earlier writer of b has finished).
// y_q (optional): y is also quantized to NVFP4, as stored, with the per-CTA
// maxima of |y| in `partials` (kMaxAmaxPartials floats).
static nvfp4_status gemm_impl(const nvfp4_tensor *a, const nvfp4_tensor *b, void *y,
                              nvfp4_dtype yt, int64_t ldy, uint32_t *status, int num_sms,
                              cudaStream_t stream, bool weights_ready, void *splitk,
                              const nvfp4_tensor *y_q = nullptr, float *partials = nullptr) {
    if (a->rows == 0 || b->rows == 0) return y_q ? zero_quantized(y_q, stream) : NVFP4_OK;
    if (a->cols == 0) {   // empty reduction: y = 0, so y_q is all zero
        if (cudaMemset2DAsync(y, ldy * (yt == NVFP4_BF16 ? 2 : 4), 0, b->rows * (yt == NVFP4_BF16 ? 2 : 4),
                              a->rows, stream) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        return y_q ? zero_quantized(y_q, stream) : NVFP4_OK;
    }
    Operand act{a->codes, a->scales, a->tensor_scale, a->rows};
    Operand wgt{b->codes, b->scales, b->tensor_scale, b->rows};
    int nparts = 0;
    const nvfp4_status st = from_cuda(launch_gemm(act, wgt, a->cols, y, yt == NVFP4_BF16, ldy, status,
                                                  wait_timeout_ns(), num_sms, stream, weights_ready, splitk,
                                                  y_q ? partials : nullptr, y_q ? &nparts : nullptr));
    if (st != NVFP4_OK || !y_q) return st;
    return requant_output(y, yt, ldy, y_q, partials, nparts, num_sms, stream, status);
}

nvfp4_status nvfp4_gemm(const nvfp4_tensor *a, const nvfp4_tensor *b, void *y, nvfp4_dtype yt,
                        int64_t ldy, void *ws, size_t ws_bytes, nvfp4_stream_t stream) {
    nvfp4_status st = check_gemm(a, b, y, yt, ldy);
    if (st != NVFP4_OK) return st;
    const size_t sk = splitk_ws_bytes(a->rows, b->rows);
    if ((st = check_ws(ws, ws_bytes, kWsStatusBytes + sk)) != NVFP4_OK) return st;
    DevInfo dev;
    if ((st = current_device(&dev)) != NVFP4_OK) return st;
    return gemm_impl(a, b, y, yt, ldy, static_cast<uint32_t *>(ws), dev.sms,
                     reinterpret_cast<cudaStream_t>(stream), false, sk ? ws_at(ws, kWsStatusBytes) : nullptr);
}

nvfp4_status nvfp4_gemm_requant(const nvfp4_tensor *a, const nvfp4_tensor *b, void *y, nvfp4_dtype yt,
                                int64_t ldy, const nvfp4_tensor *y_q, void *ws, size_t ws_bytes,
                                nvfp4_stream_t stream) {
    nvfp4_status st = check_gemm(a, b, y, yt, ldy);
    if (st != NVFP4_OK) return st;
    if ((st = check_tensor(y_q, a->rows, b->rows)) != NVFP4_OK) return st;
    const size_t sk = splitk_ws_bytes(a->rows, b->rows);
    if ((st = check_ws(ws, ws_bytes, kQuantizeWs + sk)) != NVFP4_OK) return st;
    DevInfo dev;
    if ((st = current_device(&dev)) != NVFP4_OK) return st;
    return gemm_impl(a, b, y, yt, ldy, static_cast<uint32_t *>(ws), dev.sms,
                     reinterpret_cast<cudaStream_t>(stream), false, sk ? ws_at(ws, kQuantizeWs) : nullptr, y_q,
                     reinterpret_cast<float *>(ws_at(ws, kPartialsOff)));
}

nvfp4_status nvfp4_linear_fused(const void *x, nvfp4_dtype xt, int64_t M, int64_t K, int64_t ldx,
                                const nvfp4_tensor *w, const nvfp4_tensor *w_up,
                                nvfp4_epilogue epilogue, void *y, nvfp4_dtype yt, int64_t ldy,
                                const nvfp4_tensor *y_q, const nvfp4_tensor *x_q, void *ws,
                                size_t ws_bytes, nvfp4_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if ((!x && M * K != 0) || !w || (xt != NVFP4_F32 && xt != NVFP4_BF16)) return NVFP4_ERR_INVALID_ARG;
    if (M < 0 || K < 0 || ldx < K) return NVFP4_ERR_INVALID_ARG;
    if (epilogue != NVFP4_EPI_STORE && epilogue != NVFP4_EPI_SILU_MUL_REQUANT)
        return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_tensor(w, w->rows, K);
    if (st != NVFP4_OK) return st;
    if (K % 64) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    const int xeb = xt == NVFP4_BF16 ? 2 : 4;
    if (M * K != 0 && (!aligned16(x) || (ldx * xeb) % 16)) return NVFP4_ERR_MISALIGNED;
    const int64_t N = w->rows;
    if (M > kMaxGemmRows || N > kMaxGemmRows || K > kMaxGemmK) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (epilogue == NVFP4_EPI_STORE) {
        if ((!y && M * N != 0) || (yt != NVFP4_F32 && yt != NVFP4_BF16) || ldy < N)
            return NVFP4_ERR_INVALID_ARG;
        if (M * N != 0 && (!aligned16(y) || (ldy * (yt == NVFP4_BF16 ? 2 : 4)) % 16))
            return NVFP4_ERR_MISALIGNED;
        if (y_q && (st = check_tensor(y_q, M, N)) != NVFP4_OK) return st;
    } else {
        if (!w_up || (st = check_tensor(w_up, N, K)) != NVFP4_OK)
            return st != NVFP4_OK ? st : NVFP4_ERR_INVALID_ARG;
        if ((st = check_tensor(y_q, M, N)) != NVFP4_OK) return st;
        if (y && (yt != NVFP4_F32 || ldy < N)) return NVFP4_ERR_INVALID_ARG;
        if (y && M * N != 0 && (!aligned16(y) || (ldy * 4) % 16)) return NVFP4_ERR_MISALIGNED;
    }
    if (x_q && (st = check_tensor(x_q, M, K)) != NVFP4_OK) return st;
    const nvfp4_op op = epilogue == NVFP4_EPI_STORE ? NVFP4_OP_LINEAR_FUSED : NVFP4_OP_LINEAR_FUSED_SILU;
    if ((st = check_ws(ws, ws_bytes, nvfp4_workspace_bytes(op, M, N, K))) != NVFP4_OK) return st;
    DevInfo dev;
    if ((st = current_device(&dev)) != NVFP4_OK) return st;
    if (M == 0) return NVFP4_OK;

    uint32_t *status = static_cast<uint32_t *>(ws);
    float *partials = reinterpret_cast<float *>(ws_at(ws, kPartialsOff));
    // A few activation rows (decode): one kernel quantizes them inside the
    // GEMM, while the weight stream is already in flight.
    if (epilogue == NVFP4_EPI_STORE && decode_fused_usable(M, N, K)) {
        Operand wgt{w->codes, w->scales, w->tensor_scale, N};
        int nparts = 0;
        st = from_cuda(launch_gemm_decode(x, xt == NVFP4_BF16, M, K, ldx, wgt, y, yt == NVFP4_BF16, ldy,
                                          x_q ? x_q->codes : nullptr, x_q ? x_q->scales : nullptr,
                                          x_q ? x_q->tensor_scale : nullptr, status, wait_timeout_ns(), dev.sms,
                                          stream, y_q ? partials : nullptr, y_q ? &nparts : nullptr));
        if (st != NVFP4_OK || !y_q) return st;
        return requant_output(y, yt, ldy, y_q, partials, nparts, dev.sms, stream, status);
    }

    // Quantized activations: caller's buffers or carved from the workspace.
    size_t off = kQuantizeWs;
    nvfp4_tensor xq;
    if (x_q) {
        xq = *x_q;
    } else {
        xq.codes = ws_at(ws, off);
        off += align256(static_cast<size_t>(M * K / 2));
        xq.scales = ws_at(ws, off);
        off += align256(nvfp4_scales_bytes(M, K));
        xq.tensor_scale = reinterpret_cast<float *>(ws_at(ws, off));
        off += 256;
        xq.rows = M;
        xq.cols = K;
    }
    if (!x_q) off = kQuantizeWs + quantized_bytes(M, K);
    // MLP with one gate/up tile per SM: h is re-quantized inside the GEMM's
    // epilogue, whose CTAs meet at the workspace's grid meeting point.
    const bool fused_requant = epilogue == NVFP4_EPI_SILU_MUL_REQUANT && N != 0 && K != 0 &&
                               dual_fused_requant_usable(M, N, dev.sms, static_cast<int>(kMaxAmaxPartials));
    uint32_t *grid_bar = reinterpret_cast<uint32_t *>(ws_at(ws, kGridBarOff));
    cudaError_t e = launch_quantize(x, xt == NVFP4_BF16, M, K, ldx, xq.codes, xq.scales,
                                    xq.tensor_scale, partials, dev.sms, stream, grid_bar, status,
                                    wait_timeout_ns());
    if (e != cudaSuccess) return NVFP4_ERR_CUDA;
    // (The GEMM writes its per-CTA maxima of |y| into the same partials only
    // at its end, after its dependent-launch wait, so the activation encode
    // pass that reads them has finished by then.)
    if (epilogue == NVFP4_EPI_STORE)
        return gemm_impl(&xq, w, y, yt, ldy, status, dev.sms, stream, true,
                         splitk_ws_bytes(M, N) != 0 ? ws_at(ws, kQuantizeWs + quantized_bytes(M, K)) : nullptr,
                         y_q, partials);

    // An empty reduction (K == 0) makes gate = up = 0, so h = SiLU(0) * 0 = 0:
    // y_q gets all-zero codes and scales and g = 0, y (if given) zeros.  With
    // N == 0 only the tensor scale is written.
    if (N == 0 || K == 0) {
        if (cudaMemsetAsync(y_q->tensor_scale, 0, sizeof(float), stream) != cudaSuccess) return NVFP4_ERR_CUDA;
        if (N == 0) return NVFP4_OK;
        if (cudaMemsetAsync(y_q->codes, 0, nvfp4_codes_bytes(M, N), stream) != cudaSuccess ||
            cudaMemsetAsync(y_q->scales, 0, nvfp4_scales_bytes(M, N), stream) != cudaSuccess)
            return NVFP4_ERR_CUDA;
        if (y) return from_cuda(cudaMemset2DAsync(y, ldy * sizeof(float), 0, N * sizeof(float), M, stream));
        return NVFP4_OK;
    }

    // Gate and up in one GEMM whose epilogue forms h = SiLU(gate) * up and the
    // per-CTA max |h|; h_q either in the same epilogue (fused_requant) or by
    // the quantizer's encode pass over h written to memory.
    Operand act{xq.codes, xq.scales, xq.tensor_scale, M};
    Operand og{w->codes, w->scales, w->tensor_scale, N};
    Operand ou{w_up->codes, w_up->scales, w_up->tensor_scale, N};
    int nparts = 0;
    if (fused_requant)
        return from_cuda(launch_gemm_dual_silu(act, og, ou, K, static_cast<float *>(y), y ? ldy : N, partials,
                                               kMaxAmaxPartials, &nparts, status, wait_timeout_ns(), dev.sms, stream,
                                               true, y_q->codes, y_q->scales, y_q->tensor_scale, grid_bar));
    float *h = y ? static_cast<float *>(y) : reinterpret_cast<float *>(ws_at(ws, off));
    const int64_t ldh = y ? ldy : N;
    if (launch_gemm_dual_silu(act, og, ou, K, h, ldh, partials, kMaxAmaxPartials, &nparts, status,
                              wait_timeout_ns(), dev.sms, stream, true, nullptr, nullptr, nullptr, nullptr) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return from_cuda(launch_encode_f32(h, M, N, ldh, partials, nparts, y_q->codes, y_q->scales,
                                       y_q->tensor_scale, dev.sms, stream, status));
}

// ---------------------------------------------------------------------------
// MXFP4
// ---------------------------------------------------------------------------

static nvfp4_status check_mx_tensor(const nvfp4_mx_tensor *t, int64_t rows, int64_t cols) {
    if (!t || t->rows != rows || t->cols != cols || rows < 0 || cols < 0) return NVFP4_ERR_INVALID_ARG;
    if (rows * cols != 0 && (!t->codes || !t->scales)) return NVFP4_ERR_INVALID_ARG;
    if (cols % 32) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(t->codes) || !aligned16(t->scales)) return NVFP4_ERR_MISALIGNED;
    return NVFP4_OK;
}

size_t nvfp4_mx_scales_bytes(int64_t rows, int64_t cols) {
    if (rows < 0 || cols < 0) return 0;
    return static_cast<size_t>(round_up(rows, 128) * round_up(cols / 32, 4));
}

nvfp4_status nvfp4_mx_quantize(const void *x, nvfp4_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                               const nvfp4_mx_tensor *out, nvfp4_stream_t stream) {
    if ((!x && rows * cols != 0) || (xt != NVFP4_F32 && xt != NVFP4_BF16)) return NVFP4_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || ld < cols) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_mx_tensor(out, rows, cols);
    if (st != NVFP4_OK) return st;
    const int eb = xt == NVFP4_BF16 ? 2 : 4;
    if (rows * cols != 0 && (!aligned16(x) || (ld * eb) % 16)) return NVFP4_ERR_MISALIGNED;
    DevInfo dev;
    if ((st = current_device(&dev)) != NVFP4_OK) return st;
    return from_cuda(launch_mx_quantize(x, xt == NVFP4_BF16, rows, cols, ld, out->codes, out->scales, dev.sms,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

nvfp4_status nvfp4_mx_gemm(const nvfp4_mx_tensor *a, const nvfp4_mx_tensor *b, void *y, nvfp4_dtype yt,
                           int64_t ldy, void *ws, size_t ws_bytes, nvfp4_stream_t stream_) {
    if (!a || !b || (yt != NVFP4_F32 && yt != NVFP4_BF16)) return NVFP4_ERR_INVALID_ARG;
    if (!y && a->rows * b->rows != 0) return NVFP4_ERR_INVALID_ARG;
    if (a->cols != b->cols) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_mx_tensor(a, a->rows, a->cols);
    if (st != NVFP4_OK) return st;
    if ((st = check_mx_tensor(b, b->rows, b->cols)) != NVFP4_OK) return st;
    if (a->cols % 64) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (a->rows > kMaxGemmRows || b->rows > kMaxGemmRows || a->cols > kMaxGemmK) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (ldy < b->rows) return NVFP4_ERR_INVALID_ARG;
    const int eb = yt == NVFP4_BF16 ? 2 : 4;
    if (a->rows * b->rows != 0 && (!aligned16(y) || (ldy * eb) % 16)) return NVFP4_ERR_MISALIGNED;
    const size_t sk = splitk_ws_bytes(a->rows, b->rows);
    if ((st = check_ws(ws, ws_bytes, kWsStatusBytes + sk)) != NVFP4_OK) return st;
    DevInfo dev;
    if ((st = current_device(&dev)) != NVFP4_OK) return st;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (a->rows == 0 || b->rows == 0) return NVFP4_OK;
    if (a->cols == 0)
        return from_cuda(cudaMemset2DAsync(y, ldy * eb, 0, b->rows * eb, a->rows, stream));
    Operand act{a->codes, a->scales, nullptr, a->rows};
    Operand wgt{b->codes, b->scales, nullptr, b->rows};
    return from_cuda(launch_gemm_mx(act, wgt, a->cols, y, yt == NVFP4_BF16, ldy, static_cast<uint32_t *>(ws),
                                    wait_timeout_ns(), dev.sms, stream, sk ? ws_at(ws, kWsStatusBytes) : nullptr));
}

// ---------------------------------------------------------------------------
// W4A8: MXFP8 activations x MXFP4 weights
// ---------------------------------------------------------------------------

static nvfp4_status check_mx8_tensor(const nvfp4_mx8_tensor *t, int64_t rows, int64_t cols) {
    if (!t || t->rows != rows || t->cols != cols || rows < 0 || cols < 0) return NVFP4_ERR_INVALID_ARG;
    if (rows * cols != 0 && (!t->elems || !t->scales)) return NVFP4_ERR_INVALID_ARG;
    if (cols % 32) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(t->elems) || !aligned16(t->scales)) return NVFP4_ERR_MISALIGNED;
    return NVFP4_OK;
}

nvfp4_status nvfp4_mx8_quantize(const void *x, nvfp4_dtype xt, int64_t rows, int64_t cols, int64_t ld,
                                const nvfp4_mx8_tensor *out, nvfp4_stream_t stream) {
    if ((!x && rows * cols != 0) || (xt != NVFP4_F32 && xt != NVFP4_BF16)) return NVFP4_ERR_INVALID_ARG;
    if (rows < 0 || cols < 0 || ld < cols) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_mx8_tensor(out, rows, cols);
    if (st != NVFP4_OK) return st;
    const int eb = xt == NVFP4_BF16 ? 2 : 4;
    if (rows * cols != 0 && (!aligned16(x) || (ld * eb) % 16)) return NVFP4_ERR_MISALIGNED;
    DevInfo dev;
    if ((st = current_device(&dev)) != NVFP4_OK) return st;
    return from_cuda(launch_mx8_quantize(x, xt == NVFP4_BF16, rows, cols, ld, out->elems, out->scales, dev.sms,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

// The weights' codes are read by a copy that unpacks them into 8-bit
// containers: it moves 128 values of K per row and needs a row length that is
// a multiple of 128 values and a 32-byte aligned start.
static nvfp4_status check_w4a8_weights(const nvfp4_mx_tensor *w, int64_t K) {
    nvfp4_status st = check_mx_tensor(w, w ? w->rows : 0, K);
    if (st != NVFP4_OK) return st;
    if (K % 128) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (w->rows * K != 0 && (reinterpret_cast<uintptr_t>(w->codes) & 31u)) return NVFP4_ERR_MISALIGNED;
    return NVFP4_OK;
}

static nvfp4_status w4a8_gemm_impl(const nvfp4_mx8_tensor *a, const nvfp4_mx_tensor *b, void *y, nvfp4_dtype yt,
                                   int64_t ldy, uint32_t *status, int sms, cudaStream_t stream, bool weights_ready,
                                   void *splitk) {
    const int eb = yt == NVFP4_BF16 ? 2 : 4;
    if (a->rows == 0 || b->rows == 0) return NVFP4_OK;
    if (a->cols == 0) return from_cuda(cudaMemset2DAsync(y, ldy * eb, 0, b->rows * eb, a->rows, stream));
    Operand act{a->elems, a->scales, nullptr, a->rows};
    Operand wgt{b->codes, b->scales, nullptr, b->rows};
    return from_cuda(launch_gemm_w4a8(act, wgt, a->cols, y, yt == NVFP4_BF16, ldy, status, wait_timeout_ns(), sms,
                                      stream, weights_ready, splitk));
}

nvfp4_status nvfp4_w4a8_gemm(const nvfp4_mx8_tensor *a, const nvfp4_mx_tensor *b, void *y, nvfp4_dtype yt,
                             int64_t ldy, void *ws, size_t ws_bytes, nvfp4_stream_t stream) {
    if (!a || !b || (yt != NVFP4_F32 && yt != NVFP4_BF16)) return NVFP4_ERR_INVALID_ARG;
    if (!y && a->rows * b->rows != 0) return NVFP4_ERR_INVALID_ARG;
    if (a->cols != b->cols) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_mx8_tensor(a, a->rows, a->cols);
    if (st != NVFP4_OK) return st;
    if ((st = check_w4a8_weights(b, a->cols)) != NVFP4_OK) return st;
    if (a->rows > kMaxGemmRows || b->rows > kMaxGemmRows || a->cols > kMaxGemmK) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (ldy < b->rows) return NVFP4_ERR_INVALID_ARG;
    const int eb = yt == NVFP4_BF16 ? 2 : 4;
    if (a->rows * b->rows != 0 && (!aligned16(y) || (ldy * eb) % 16)) return NVFP4_ERR_MISALIGNED;
    const size_t sk = splitk_ws_bytes(a->rows, b->rows);
    if ((st = check_ws(ws, ws_bytes, kWsStatusBytes + sk)) != NVFP4_OK) return st;
    DevInfo dev;
    if ((st = current_device(&dev)) != NVFP4_OK) return st;
    return w4a8_gemm_impl(a, b, y, yt, ldy, static_cast<uint32_t *>(ws), dev.sms,
                          reinterpret_cast<cudaStream_t>(stream), false, sk ? ws_at(ws, kWsStatusBytes) : nullptr);
}

nvfp4_status nvfp4_w4a8_linear(const void *x, nvfp4_dtype xt, int64_t M, int64_t K, int64_t ldx,
                               const nvfp4_mx_tensor *w, void *y, nvfp4_dtype yt, int64_t ldy,
                               const nvfp4_mx8_tensor *x_q, void *ws, size_t ws_bytes, nvfp4_stream_t stream_) {
    if ((!x && M * K != 0) || !w || (xt != NVFP4_F32 && xt != NVFP4_BF16) || (yt != NVFP4_F32 && yt != NVFP4_BF16))
        return NVFP4_ERR_INVALID_ARG;
    if (M < 0 || K < 0 || ldx < K) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_w4a8_weights(w, K);
    if (st != NVFP4_OK) return st;
    const int64_t N = w->rows;
    if (M > kMaxGemmRows || N > kMaxGemmRows || K > kMaxGemmK) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if ((!y && M * N != 0) || ldy < N) return NVFP4_ERR_INVALID_ARG;
    const int xeb = xt == NVFP4_BF16 ? 2 : 4, yeb = yt == NVFP4_BF16 ? 2 : 4;
    if ((M * K != 0 && (!aligned16(x) || (ldx * xeb) % 16)) || (M * N != 0 && (!aligned16(y) || (ldy * yeb) % 16)))
        return NVFP4_ERR_MISALIGNED;
    if (x_q && (st = check_mx8_tensor(x_q, M, K)) != NVFP4_OK) return st;
    if ((st = check_ws(ws, ws_bytes, nvfp4_workspace_bytes(NVFP4_OP_W4A8_LINEAR, M, N, K))) != NVFP4_OK) return st;
    DevInfo dev;
    if ((st = current_device(&dev)) != NVFP4_OK) return st;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (M == 0) return NVFP4_OK;
    nvfp4_mx8_tensor xq;
    size_t off = kWsStatusBytes;
    if (x_q) {
        xq = *x_q;
    } else {
        xq.elems = ws_at(ws, off);
        off += align256(static_cast<size_t>(M * K));
        xq.scales = ws_at(ws, off);
        xq.rows = M;
        xq.cols = K;
    }
    off = kWsStatusBytes + align256(static_cast<size_t>(M * K)) + align256(nvfp4_mx_scales_bytes(M, K));
    if (launch_mx8_quantize(x, xt == NVFP4_BF16, M, K, ldx, xq.elems, xq.scales, dev.sms, stream) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    // the quantizer is launched without a programmatic dependency, so the
    // weights' earlier writers have finished: the GEMM may stream them early
    return w4a8_gemm_impl(&xq, w, y, yt, ldy, static_cast<uint32_t *>(ws), dev.sms, stream, true,
                          splitk_ws_bytes(M, N) != 0 ? ws_at(ws, off) : nullptr);
}

// ---------------------------------------------------------------------------
// W4A16
// ---------------------------------------------------------------------------

nvfp4_status nvfp4_w4a16_linear(const void *x, nvfp4_dtype xt, int64_t M, int64_t K, int64_t ldx,
                                const nvfp4_tensor *w, void *y, nvfp4_dtype yt, int64_t ldy, void *ws,
                                size_t ws_bytes, nvfp4_stream_t stream_) {
    if ((!x && M * K != 0) || !w || xt != NVFP4_BF16 || (yt != NVFP4_F32 && yt != NVFP4_BF16))
        return NVFP4_ERR_INVALID_ARG;
    if (M < 0 || K < 0 || ldx < K) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_tensor(w, w->rows, K);
    if (st != NVFP4_OK) return st;
    if (K % 64) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    const int64_t N = w->rows;
    if (M > kMaxGemmRows || N > kMaxGemmRows || K > kMaxGemmK) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if ((!y && M * N != 0) || ldy < N) return NVFP4_ERR_INVALID_ARG;
    const int yeb = yt == NVFP4_BF16 ? 2 : 4;
    if ((M * K != 0 && (!aligned16(x) || (ldx * 2) % 16)) || (M * N != 0 && (!aligned16(y) || (ldy * yeb) % 16)))
        return NVFP4_ERR_MISALIGNED;
    if ((st = check_ws(ws, ws_bytes, kWsStatusBytes)) != NVFP4_OK) return st;
    DevInfo dev;
    if ((st = current_device(&dev)) != NVFP4_OK) return st;
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if (M == 0 || N == 0) return NVFP4_OK;
    if (K == 0) return from_cuda(cudaMemset2DAsync(y, ldy * yeb, 0, N * yeb, M, stream));
    Operand wgt{w->codes, w->scales, w->tensor_scale, N};
    return from_cuda(launch_gemm_w4a16(x, M, K, ldx, wgt, y, yt == NVFP4_BF16, ldy, static_cast<uint32_t *>(ws),
                                       wait_timeout_ns(), dev.sms, stream));
}

nvfp4_status nvfp4_get_device_status(void *ws, nvfp4_stream_t stream) {
    if (!ws) return NVFP4_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    if (cudaMemcpyAsync(&word, ws, sizeof word, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (word) {
        if (cudaMemsetAsync(ws, 0, sizeof word, s) != cudaSuccess) return NVFP4_ERR_CUDA;
        if (cudaStreamSynchronize(s) != cudaSuccess) return NVFP4_ERR_CUDA;
    }
    for (int code = 1; code < 32; ++code)
        if (word & (1u << code)) return static_cast<nvfp4_status>(code);
    return NVFP4_OK;
}

nvfp4_status nvfp4_selftest_bounded_wait(void *ws, uint32_t timeout_us, nvfp4_stream_t stream) {
    nvfp4_status st = check_ws(ws, kWsStatusBytes, kWsStatusBytes);
    if (st != NVFP4_OK) return st;
    DevInfo dev;
    if ((st = current_device(&dev)) != NVFP4_OK) return st;
    return from_cuda(launch_wait_selftest(static_cast<uint32_t *>(ws),
                                          static_cast<uint64_t>(timeout_us) * 1000ull,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

uint32_t nvfp4_set_wait_timeout_us(uint32_t timeout_us) {
    return g_wait_timeout_us.exchange(timeout_us == 0 ? 1u : timeout_us);
}

const char *nvfp4_status_string(nvfp4_status s) {
    switch (s) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case NVFP4_ERR_MISALIGNED: return "misaligned pointer or pitch";
    case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
    case NVFP4_ERR_CUDA: return "CUDA error";
    case NVFP4_ERR_TIMEOUT: return "device-side wait timed out";
    case NVFP4_ERR_ARCH: return "device is not sm_100";
    case NVFP4_ERR_BOUNDS: return "device-side store out of bounds (debug build)";
    }
    return "unknown status";
}

int nvfp4_version(void) { return 100; }

}  // extern "C"
