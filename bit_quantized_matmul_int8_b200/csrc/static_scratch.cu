// Allocation-free forward for decode shapes (M <= 16 tokens).
//
// int8lt_forward takes its scratch (outlier bitmap and list, CA/SCA, the
// fp16 outlier activations, the GEMV's partial sums) from a caller-provided
// workspace. Some callers cannot provide one: a plugin or engine that hands
// this layer only its input and output buffers, a runtime whose device
// memory is owned entirely by its own pool, or a latency-critical decode
// loop that must not call cudaMalloc (which can synchronize the device).
// This entry point serves them: its scratch is a fixed array in this
// library's device image, so the call itself allocates nothing and calls no
// allocating routine.
//
// The array is kStaticScratchBytes (8 MiB). Every GPU on which the library
// is loaded holds it until the process exits. It is shared by all calls on
// that GPU and keeps the previous call's contents: the quantize pass of every
// call rewrites the outlier list, codes and scales and zeroes the GEMV's
// sums before they are accumulated, so nothing carries over; but two calls
// whose kernels overlap on the GPU (different streams without ordering, or
// different host threads) race on the array and corrupt each other.
//
// In host code `g_scratch` is only a host-side stand-in for the device
// symbol, not a device address. The device address is taken once per device
// with cudaGetSymbolAddress, with that device current, on the first call the
// process makes on that device; that first call should therefore come before
// any stream capture.
#include <mutex>

#include "int8lt_internal.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;

static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::once_flag g_setup_once[kMaxDevices];
void *g_scratch_ptr[kMaxDevices];
cudaError_t g_setup_err[kMaxDevices];

// Device address of g_scratch on the current device (set up on first use).
int scratch_on_current_device(void **ptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return INT8LT_ERR_CUDA;
    std::call_once(g_setup_once[dev], [dev] {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
        // Start from a zeroed scratch (as int8lt_workspace_init leaves a
        // workspace); synchronous, once.
        if (e == cudaSuccess) e = cudaMemset(p, 0, kStaticScratchBytes);
        g_setup_err[dev] = e;
        g_scratch_ptr[dev] = (e == cudaSuccess) ? p : nullptr;
    });
    if (g_setup_err[dev] != cudaSuccess || !g_scratch_ptr[dev]) return INT8LT_ERR_CUDA;
    *ptr = g_scratch_ptr[dev];
    return INT8LT_OK;
}

bool is_aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" int int8lt_forward_static_scratch(const void *X, int64_t M, int64_t N, int64_t K,
                                             const int8_t *CB, const float *SCB, const void *W_outlier,
                                             float threshold, const void *bias, void *Y, void *stream) {
    using namespace int8lt;
    if (M < 0 || N < 0 || K < 16 || K > kMaxK || (K % 16) != 0 || (N % 8) != 0) return INT8LT_ERR_SHAPE;
    if (M > kDecodeMaxM) return INT8LT_ERR_TOO_LARGE;
    if (M == 0 || N == 0) return INT8LT_OK;
    if (ws_layout(M, N, K).total > kStaticScratchBytes) return INT8LT_ERR_TOO_LARGE;
    if (!X || !CB || !SCB || !Y) return INT8LT_ERR_NULL;
    if (!is_aligned(X, 16) || !is_aligned(CB, 16) || !is_aligned(SCB, 4) || !is_aligned(Y, 16) ||
        (W_outlier && !is_aligned(W_outlier, 16)) || (bias && !is_aligned(bias, 2)))
        return INT8LT_ERR_ALIGN;
    if (threshold != threshold || threshold < 0.f) return INT8LT_ERR_VALUE;
    int major = 0, minor = 0, dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return INT8LT_ERR_CUDA;
    if (major != 10 || minor != 0) return INT8LT_ERR_UNSUPPORTED;
    void *ws = nullptr;
    if (int st = scratch_on_current_device(&ws)) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (int st = forward_quantize(X, M, N, K, CB, SCB, W_outlier, threshold, ws, s)) return st;
    return forward_matmul(M, N, K, CB, SCB, W_outlier, bias, Y, ws, s);
}
