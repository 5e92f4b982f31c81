// noalloc.cu -- nvfp4_linear_noalloc: the W4A4 linear layer (activation
// quantize + GEMM, the NVFP4_EPI_STORE case of nvfp4_linear_fused) for callers
// that cannot hand the library a workspace.
//
// Who cannot allocate: a caller that is not allowed to call cudaMalloc at all
// (a plugin inside a framework whose caching allocator owns every device
// byte), a caller whose memory plan is fixed before it runs (an inference
// runtime that reserves HBM for weights and KV cache up front, so a late
// allocation would fail or fragment), a caller on a latency-critical path that
// must not risk the implicit device synchronisation cudaMalloc/cudaFree can
// cause, and a foreign-language caller that only holds pointers to buffers it
// was given.  Such callers still own their inputs and outputs; only the
// scratch moves into the library.
//
// The scratch is one file-scope __device__ array.  Every GPU that loads the
// library holds it until the process exits.  In host code the array's name is
// only a host-side stand-in, never a device address, so its device address is
// looked up per device with cudaGetSymbolAddress, with that device current, on
// the first call made on that device; make that first call before any stream
// capture.  The address is cached per device ordinal for the life of the
// process, so it is only valid for the context it was looked up in: call this
// entry point from the device's primary context (the runtime's own) only, and
// not after cudaDeviceReset, which unloads the module so that the array may
// come back at another address.  Every call shares the one array and finds the previous call's
// contents in it: calls that overlap on the GPU (two streams, two threads, or
// a second call enqueued on another stream before the first finished) race on
// it and corrupt each other.  What must start at zero (the device status word)
// is cleared by each call before its kernels run; everything else is fully
// rewritten by every call.
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"
#include "nvfp4.h"

namespace {

using namespace nvfp4;

// 4 MiB: status word, the quantizer's partial maxima, then the quantized
// activations (codes, tiled scales, tensor scale) of up to about 1.3k rows at
// K = 5120 -- decode and small-batch shapes.
constexpr size_t kScratchBytes = size_t(4) << 20;
constexpr size_t kStatusOff = 0;
constexpr size_t kPartialsOff = kWsStatusBytes;                                   // 256
constexpr size_t kXqOff = kPartialsOff + kMaxAmaxPartials * sizeof(float);        // 16640

static __device__ __align__(256) uint8_t g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
uint8_t *g_scratch_addr[kMaxDevices] = {};

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device address of the scratch array on the current device (looked up once
// per device).
nvfp4_status scratch_on_current_device(uint8_t **out, int *sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_CUDA;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    if (major != 10 || minor != 0) return NVFP4_ERR_ARCH;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return NVFP4_ERR_CUDA;
        g_scratch_addr[dev] = static_cast<uint8_t *>(p);
    }
    *out = g_scratch_addr[dev];
    return NVFP4_OK;
}

nvfp4_status check_weights(const nvfp4_tensor *w, int64_t K) {
    if (!w || !w->tensor_scale || w->rows < 0 || w->cols != K) return NVFP4_ERR_INVALID_ARG;
    if (w->rows * K != 0 && (!w->codes || !w->scales)) return NVFP4_ERR_INVALID_ARG;
    if (!aligned16(w->codes) || !aligned16(w->scales) || !aligned16(w->tensor_scale))
        return NVFP4_ERR_MISALIGNED;
    return NVFP4_OK;
}

}  // namespace

extern "C" nvfp4_status nvfp4_linear_noalloc(const void *x, nvfp4_dtype xt, int64_t M, int64_t K,
                                             int64_t ldx, const nvfp4_tensor *w, void *y,
                                             nvfp4_dtype yt, int64_t ldy, nvfp4_stream_t stream_) {
    cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
    if ((!x && M * K != 0) || (xt != NVFP4_F32 && xt != NVFP4_BF16)) return NVFP4_ERR_INVALID_ARG;
    if (M < 0 || K < 0 || ldx < K) return NVFP4_ERR_INVALID_ARG;
    nvfp4_status st = check_weights(w, K);
    if (st != NVFP4_OK) return st;
    if (K % 64) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    const int64_t N = w->rows;
    if ((!y && M * N != 0) || (yt != NVFP4_F32 && yt != NVFP4_BF16) || ldy < N) return NVFP4_ERR_INVALID_ARG;
    const int xeb = xt == NVFP4_BF16 ? 2 : 4, yeb = yt == NVFP4_BF16 ? 2 : 4;
    // empty operands are never touched: their pointers and pitches are not checked
    if ((M * K != 0 && (!aligned16(x) || (ldx * xeb) % 16)) || (M * N != 0 && (!aligned16(y) || (ldy * yeb) % 16)))
        return NVFP4_ERR_MISALIGNED;
    if (M > kMaxGemmRows || N > kMaxGemmRows || K > kMaxGemmK) return NVFP4_ERR_UNSUPPORTED_SHAPE;

    // Quantized activations must fit in the static scratch.
    const size_t codes_bytes = align256(static_cast<size_t>(M) * static_cast<size_t>(K / 2));
    const size_t scales_bytes = align256(static_cast<size_t>(round_up(M, 128) * kb4_of(K)));
    if (kXqOff + codes_bytes + scales_bytes + 256 > kScratchBytes) return NVFP4_ERR_UNSUPPORTED_SHAPE;

    uint8_t *scratch = nullptr;
    int sms = 0;
    if ((st = scratch_on_current_device(&scratch, &sms)) != NVFP4_OK) return st;
    if (M == 0 || N == 0) return NVFP4_OK;

    uint32_t *status = reinterpret_cast<uint32_t *>(scratch + kStatusOff);
    float *partials = reinterpret_cast<float *>(scratch + kPartialsOff);
    uint8_t *xq_codes = scratch + kXqOff;
    uint8_t *xq_scales = xq_codes + codes_bytes;
    float *xq_g = reinterpret_cast<float *>(xq_scales + scales_bytes);

    if (cudaMemsetAsync(status, 0, sizeof(uint32_t), stream) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (launch_quantize(x, xt == NVFP4_BF16, M, K, ldx, xq_codes, xq_scales, xq_g, partials, sms,
                        stream, nullptr, status, wait_timeout_ns()) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    if (K == 0)
        return cudaMemset2DAsync(y, ldy * yeb, 0, N * yeb, M, stream) == cudaSuccess ? NVFP4_OK
                                                                                    : NVFP4_ERR_CUDA;
    Operand act{xq_codes, xq_scales, xq_g, M};
    Operand wgt{w->codes, w->scales, w->tensor_scale, N};
    return launch_gemm(act, wgt, K, y, yt == NVFP4_BF16, ldy, status, wait_timeout_ns(), sms, stream) ==
                   cudaSuccess
               ? NVFP4_OK
               : NVFP4_ERR_CUDA;
}
