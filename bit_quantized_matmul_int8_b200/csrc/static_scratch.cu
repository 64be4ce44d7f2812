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
// symbol, not a device address. The device address is taken with
// cudaGetSymbolAddress, with the device current, on the first call the
// process makes on that device, which also zeroes the whole array with a
// synchronous cudaMemset; that first call should therefore come before any
// stream capture. Only a successful set-up is kept: if it fails (for example
// because a capture is under way), the call reports INT8LT_ERR_CUDA and the
// next call on that device tries again.
//
// Device-side timeouts land in the array's own status word, which callers
// read (and clear) with int8lt_static_scratch_read_status.
#include <atomic>
#include <mutex>

#include "int8lt_internal.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;

static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
std::atomic<void *> g_scratch_ptr[kMaxDevices];

// Device address of g_scratch on the current device (set up on first use).
int scratch_on_current_device(void **ptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return INT8LT_ERR_CUDA;
    void *p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(g_setup_mu);
        p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
        if (!p) {
            // Start from a zeroed array, as int8lt_workspace_init leaves a
            // workspace. On failure clear the runtime's last error, so that a
            // later launch check does not report this call's failure again.
            if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p ||
                cudaMemset(p, 0, kStaticScratchBytes) != cudaSuccess) {
                (void)cudaGetLastError();
                return INT8LT_ERR_CUDA;
            }
            g_scratch_ptr[dev].store(p, std::memory_order_release);
        }
    }
    *ptr = p;
    return INT8LT_OK;
}

int device_supported() {
    int major = 0, minor = 0, dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return INT8LT_ERR_CUDA;
    return (major == 10 && minor == 0) ? INT8LT_OK : INT8LT_ERR_UNSUPPORTED;
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
    if (int st = device_supported()) return st;
    void *ws = nullptr;
    if (int st = scratch_on_current_device(&ws)) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (int st = forward_quantize(X, M, N, K, CB, SCB, W_outlier, threshold, ws, s)) return st;
    return forward_matmul(M, N, K, CB, SCB, W_outlier, bias, Y, ws, s);
}

// Synchronize the stream, then read the array's status word on the current
// device. A timeout also re-zeroes the header and the column bitmaps (the
// barrier counts of the quantize pass may be off after one), which is what
// int8lt_workspace_init does for a workspace; every other part of the array
// is rewritten by each call.
extern "C" int int8lt_static_scratch_read_status(void *stream) {
    using namespace int8lt;
    if (int st = device_supported()) return st;
    void *ws = nullptr;
    if (int st = scratch_on_current_device(&ws)) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t status = 0;
    if (cudaMemcpyAsync(&status, ws, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return INT8LT_ERR_CUDA;
    if (status == 0) return INT8LT_OK;
    if (cudaMemsetAsync(ws, 0, kWsInitBytes, s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
        return INT8LT_ERR_CUDA;
    if (status & kStatusTimeout) return INT8LT_ERR_TIMEOUT;
    return (status & kStatusBounds) ? INT8LT_ERR_BOUNDS : INT8LT_ERR_CUDA;
}

// Test entry: the quantize pass's grid-barrier wait run out against the
// array's header, as a real timeout would leave it.
extern "C" int int8lt_debug_static_scratch_timeout(int64_t limit_ns, void *stream) {
    using namespace int8lt;
    if (limit_ns < 1000 || limit_ns > 1000000000) return INT8LT_ERR_VALUE;
    if (int st = device_supported()) return st;
    void *ws = nullptr;
    if (int st = scratch_on_current_device(&ws)) return st;
    return launch_barrier_timeout(static_cast<WsHeader *>(ws), (uint64_t)limit_ns,
                                  static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? INT8LT_OK
               : INT8LT_ERR_CUDA;
}
