// C ABI of libint8lt: argument validation, workspace layout and dispatch.
// Every check runs on the host before the first launch; see include/int8lt.h
// for the contract of each entry point.
#include <algorithm>
#include <atomic>
#include <cmath>

#include "int8lt_internal.cuh"

namespace int8lt {

static size_t align_up(size_t v) { return (v + 1023) & ~size_t(1023); }

WsLayout ws_layout(int64_t M, int64_t N, int64_t K) {
    WsLayout L{};
    L.M = M; L.N = N; L.K = K;
    L.kwords = ceil_div(K, 32);
    L.kcap = round_up(K, 64);
    size_t off = 0;
    L.hdr = off;     off += align_up(sizeof(WsHeader));
    L.bitmaps = off; off += align_up(kWsInitBytes - kWsBitmapOffset);
    L.idx = off;   off += align_up((size_t)K * 4);
    L.sca = off;   off += align_up((size_t)M * 4);
    L.ca = off;    off += align_up((size_t)M * K);
    L.xo = off;    off += align_up((size_t)M * L.kcap * 2);
    L.zpa = off;   off += align_up((size_t)M * 8);
    if (M > kDecodeMaxM) {
        L.wo = off; off += align_up((size_t)N * L.kcap * 2);
        L.sk = off; off += align_up((size_t)kSkMaxPairs * 2 * kSkPartialBytes);
        L.acc = L.cnt = SIZE_MAX;
    } else {
        L.wo = SIZE_MAX;
        L.sk = SIZE_MAX;
        L.acc = off; off += align_up((size_t)round_up(N * M, 4) * 4);
        L.cnt = off; off += align_up((size_t)round_up(ceil_div(N, 8), 4) * 4);
    }
    L.total = off;
    return L;
}

}  // namespace int8lt

using namespace int8lt;

namespace {

template <typename T>
T *at(void *ws, size_t off) {
    return off == SIZE_MAX ? nullptr : reinterpret_cast<T *>(static_cast<char *>(ws) + off);
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool shape_ok(int64_t M, int64_t N, int64_t K) {
    return M >= 0 && N >= 0 && K >= 16 && K <= kMaxK && (K % 16) == 0 && (N % 8) == 0 &&
           M <= (int64_t)1 << 31 && N <= (int64_t)1 << 31;
}

// 0 = unknown, 1 = compute capability 10.0, 2 = other
std::atomic<int> g_dev_ok[64];

int check_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return INT8LT_ERR_CUDA;
    std::atomic<int> &slot = g_dev_ok[dev & 63];
    int st = slot.load(std::memory_order_relaxed);
    if (st == 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return INT8LT_ERR_CUDA;
        st = (major == 10 && minor == 0) ? 1 : 2;
        slot.store(st, std::memory_order_relaxed);
    }
    return st == 1 ? INT8LT_OK : INT8LT_ERR_UNSUPPORTED;
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? INT8LT_OK : INT8LT_ERR_CUDA; }

__global__ void wait_timeout_kernel(uint32_t *status, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_barrier_init();
        // Nothing ever arrives on `bar`: the bounded wait must give up.
        if (!mbar_wait_bounded(smem_u32(&bar), 0, limit_ns)) record_timeout(status);
    }
}

}  // namespace

namespace int8lt {
cudaError_t launch_wait_timeout(uint32_t *status, uint64_t limit_ns, cudaStream_t s) {
    wait_timeout_kernel<<<1, 32, 0, s>>>(status, limit_ns);
    return cudaGetLastError();
}
}  // namespace int8lt

namespace {

// Host-side checks shared by the forward entry points.
int check_forward_args(const void *X, int64_t M, int64_t N, int64_t K, const int8_t *CB, const float *SCB,
                       const void *W_outlier, float threshold, const void *bias, const void *Y, bool need_x,
                       bool need_y, void *ws, size_t ws_bytes) {
    if (!shape_ok(M, N, K)) return INT8LT_ERR_SHAPE;
    if (M == 0 || N == 0) return -1;  // empty output: nothing to read or write
    if ((need_x && !X) || !CB || !SCB || (need_y && !Y) || !ws) return INT8LT_ERR_NULL;
    if ((need_x && !aligned(X, 16)) || !aligned(CB, 16) || !aligned(SCB, 4) || (need_y && !aligned(Y, 16)) ||
        !aligned(ws, 16) || (W_outlier && !aligned(W_outlier, 16)) || (bias && !aligned(bias, 2)))
        return INT8LT_ERR_ALIGN;
    if (std::isnan(threshold) || threshold < 0.f) return INT8LT_ERR_VALUE;
    if (ws_bytes < ws_layout(M, N, K).total) return INT8LT_ERR_WORKSPACE;
    return check_device();
}

// The zeropoint forward's extra weight arrays (-1: empty output, nothing to check).
int check_zp_weight_args(int64_t M, int64_t N, int64_t K, const int32_t *ZB, const int32_t *SB) {
    if (!shape_ok(M, N, K)) return INT8LT_ERR_SHAPE;
    if (M == 0 || N == 0) return -1;
    if (!ZB || !SB) return INT8LT_ERR_NULL;
    if (!aligned(ZB, 4) || !aligned(SB, 4)) return INT8LT_ERR_ALIGN;
    return 0;
}

}  // namespace

namespace int8lt {

int forward_quantize(const void *X, int64_t M, int64_t N, int64_t K, const int8_t *CB, const float *SCB,
                     const void *W_outlier, float threshold, void *ws, cudaStream_t s) {
    const WsLayout L = ws_layout(M, N, K);
    const __half *x = static_cast<const __half *>(X);
    WsHeader *hdr = at<WsHeader>(ws, L.hdr);
    const bool decode = M <= kDecodeMaxM;
    QuantizeArgs q{};
    q.X = x; q.M = M; q.K = K;
    q.hdr = hdr; q.bitmaps = at<uint32_t>(ws, L.bitmaps); q.tbits = threshold_bits(threshold);
    q.CA = at<int8_t>(ws, L.ca); q.SCA = at<float>(ws, L.sca);
    q.outlier_idx = at<int32_t>(ws, L.idx); q.n_outliers = &hdr->n_outliers;
    q.Xo = at<__half>(ws, L.xo); q.kcap = L.kcap;
    q.W_outlier = static_cast<const __half *>(W_outlier); q.CB = CB; q.SCB = SCB; q.N = N;
    if (!decode) q.Wo = at<__half>(ws, L.wo);
    if (decode) {  // the GEMV's partial sums and k-block counters start at zero
        q.acc = at<int32_t>(ws, L.acc); q.acc_words = round_up(N * M, 4);
        q.cnt = at<uint32_t>(ws, L.cnt); q.cnt_words = round_up(ceil_div(N, 8), 4);
    }
    return from_cuda(launch_quantize(q, s));
}

int forward_matmul(int64_t M, int64_t N, int64_t K, const int8_t *CB, const float *SCB, const void *W_outlier,
                   const void *bias, void *Y, void *ws, cudaStream_t s) {
    const WsLayout L = ws_layout(M, N, K);
    WsHeader *hdr = at<WsHeader>(ws, L.hdr);
    if (M <= kDecodeMaxM) {
        GemvArgs g{};
        g.CA = at<int8_t>(ws, L.ca); g.CB = CB; g.SCA = at<float>(ws, L.sca); g.SCB = SCB;
        g.Xo = at<__half>(ws, L.xo); g.kcap = L.kcap;
        g.outlier_idx = at<int32_t>(ws, L.idx); g.n_outliers = &hdr->n_outliers;
        g.W_outlier = static_cast<const __half *>(W_outlier); g.bias = static_cast<const __half *>(bias);
        g.Y = static_cast<__half *>(Y);
        g.acc = at<int32_t>(ws, L.acc); g.cnt = at<uint32_t>(ws, L.cnt); g.status = &hdr->status;
        g.M = M; g.N = N; g.K = K;
        return from_cuda(launch_gemv(g, s));
    }
    GemmArgs g{};
    g.CA = at<int8_t>(ws, L.ca); g.CB = CB; g.SCA = at<float>(ws, L.sca); g.SCB = SCB;
    g.Xo = at<__half>(ws, L.xo); g.Wo = at<__half>(ws, L.wo); g.kcap = L.kcap; g.n_outliers = &hdr->n_outliers;
    g.bias = static_cast<const __half *>(bias); g.Y = static_cast<__half *>(Y);
    g.M = M; g.N = N; g.K = K; g.status = &hdr->status;
    g.sk_partial = at<int32_t>(ws, L.sk);
    g.sk_flags = at<uint32_t>(ws, kWsSkFlagOffset);
    return from_cuda(launch_gemm_tc(g, s));
}

}  // namespace int8lt

extern "C" {

const char *int8lt_status_string(int status) {
    switch (status) {
        case INT8LT_OK: return "INT8LT_OK";
        case INT8LT_ERR_NULL: return "INT8LT_ERR_NULL: a required pointer is NULL";
        case INT8LT_ERR_SHAPE: return "INT8LT_ERR_SHAPE: M, N or K outside the supported limits";
        case INT8LT_ERR_ALIGN: return "INT8LT_ERR_ALIGN: a pointer is not aligned as required";
        case INT8LT_ERR_VALUE: return "INT8LT_ERR_VALUE: threshold is NaN or negative";
        case INT8LT_ERR_WORKSPACE: return "INT8LT_ERR_WORKSPACE: workspace too small";
        case INT8LT_ERR_CUDA: return "INT8LT_ERR_CUDA: a CUDA call or launch failed";
        case INT8LT_ERR_TIMEOUT: return "INT8LT_ERR_TIMEOUT: a kernel gave up a bounded wait";
        case INT8LT_ERR_UNSUPPORTED: return "INT8LT_ERR_UNSUPPORTED: device is not compute capability 10.0";
        case INT8LT_ERR_TOO_LARGE:
            return "INT8LT_ERR_TOO_LARGE: M > 16 or the call's scratch exceeds the 8 MiB static array";
        case INT8LT_ERR_BOUNDS: return "INT8LT_ERR_BOUNDS: a kernel index failed its bounds check";
        default: return "INT8LT_ERR_UNKNOWN";
    }
}

int int8lt_version(void) { return 100; }

size_t int8lt_workspace_size(int64_t M, int64_t N, int64_t K) {
    if (!shape_ok(M, N, K)) return 0;
    return ws_layout(M, N, K).total;
}

int int8lt_workspace_init(void *ws, size_t ws_bytes, void *stream) {
    if (!ws) return INT8LT_ERR_NULL;
    if (ws_bytes < sizeof(WsHeader)) return INT8LT_ERR_WORKSPACE;
    if (!aligned(ws, 16)) return INT8LT_ERR_ALIGN;
    // Everything, so that the header (status, outlier count, quantize
    // generation and barrier counts), both column bitmaps and the split-tile
    // flags start at zero; later calls keep them consistent.
    return from_cuda(cudaMemsetAsync(ws, 0, ws_bytes, static_cast<cudaStream_t>(stream)));
}

int int8lt_read_device_status(void *ws, size_t ws_bytes, void *stream) {
    if (!ws) return INT8LT_ERR_NULL;
    if (ws_bytes < sizeof(WsHeader)) return INT8LT_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t status = 0;
    if (cudaMemcpyAsync(&status, ws, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess) return INT8LT_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return INT8LT_ERR_CUDA;
    if (status == 0) return INT8LT_OK;
    if (cudaMemsetAsync(ws, 0, 4, s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
        return INT8LT_ERR_CUDA;
    if (status & kStatusTimeout) return INT8LT_ERR_TIMEOUT;
    return (status & kStatusBounds) ? INT8LT_ERR_BOUNDS : INT8LT_ERR_CUDA;
}

size_t int8lt_weight_bytes(int64_t N, int64_t K) {
    if (N < 0 || K < 1 || K > ((int64_t)1 << 31) || N > ((int64_t)1 << 31)) return 0;
    return (size_t)weight_bytes(N, K);
}

size_t int8lt_layer_bytes(int64_t N, int64_t K, int keep_fp16_weight) {
    const size_t w = int8lt_weight_bytes(N, K);
    if (w == 0 && !(N == 0 && K >= 1)) return 0;
    return w + 4 * (size_t)N + (keep_fp16_weight ? 2 * (size_t)N * (size_t)K : 0);
}

static int convert_weight(bool pack, const int8_t *src, int64_t N, int64_t K, int8_t *dst, void *stream) {
    if (N < 0 || K < 1 || K > ((int64_t)1 << 31) || N > ((int64_t)1 << 31)) return INT8LT_ERR_SHAPE;
    if (N == 0) return INT8LT_OK;
    if (!src || !dst) return INT8LT_ERR_NULL;
    const int8_t *blocked = pack ? dst : src;
    const int8_t *rows = pack ? src : dst;
    if (!aligned(blocked, 16) || ((K % 16) == 0 && !aligned(rows, 16))) return INT8LT_ERR_ALIGN;
    if (int st = check_device()) return st;
    return from_cuda(launch_convert_weight(pack, const_cast<int8_t *>(blocked), const_cast<int8_t *>(rows), N, K,
                                           static_cast<cudaStream_t>(stream)));
}

int int8lt_pack_weight(const int8_t *CB_rows, int64_t N, int64_t K, int8_t *CB, void *stream) {
    return convert_weight(true, CB_rows, N, K, CB, stream);
}

int int8lt_unpack_weight(const int8_t *CB, int64_t N, int64_t K, int8_t *CB_rows, void *stream) {
    return convert_weight(false, CB, N, K, CB_rows, stream);
}

int int8lt_prepare_weight(const void *W, int64_t N, int64_t K, int8_t *CB, float *SCB, void *stream) {
    if (!W || !CB || !SCB) return INT8LT_ERR_NULL;
    if (N < 0 || K < 1 || K > ((int64_t)1 << 31)) return INT8LT_ERR_SHAPE;
    if (!aligned(W, 16) || !aligned(CB, 16) || !aligned(SCB, 4)) return INT8LT_ERR_ALIGN;
    if (N == 0) return INT8LT_OK;
    if (int st = check_device()) return st;
    return from_cuda(launch_prepare_weight(static_cast<const __half *>(W), N, K, CB, SCB,
                                           static_cast<cudaStream_t>(stream)));
}

int int8lt_quantize_rows(const void *X, int64_t M, int64_t K, float threshold, int8_t *CA, float *SCA,
                         int32_t *outlier_idx, int32_t *n_outliers, void *ws, size_t ws_bytes, void *stream) {
    if (!shape_ok(M, 8, K)) return INT8LT_ERR_SHAPE;
    if (!n_outliers || !ws) return INT8LT_ERR_NULL;
    if (M > 0 && (!X || !CA || !SCA || !outlier_idx)) return INT8LT_ERR_NULL;
    if ((M > 0 && (!aligned(X, 16) || !aligned(CA, 16) || !aligned(SCA, 4) || !aligned(outlier_idx, 4))) ||
        !aligned(n_outliers, 4) || !aligned(ws, 16))
        return INT8LT_ERR_ALIGN;
    if (std::isnan(threshold) || threshold < 0.f) return INT8LT_ERR_VALUE;
    const WsLayout L = ws_layout(M, 8, K);
    if (ws_bytes < L.total) return INT8LT_ERR_WORKSPACE;
    if (M == 0) {
        // |O| of an empty batch is 0.
        if (int st = check_device()) return st;
        return from_cuda(cudaMemsetAsync(n_outliers, 0, 4, static_cast<cudaStream_t>(stream)));
    }
    if (int st = check_device()) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    QuantizeArgs q{};
    q.X = static_cast<const __half *>(X);
    q.M = M; q.K = K;
    q.hdr = at<WsHeader>(ws, L.hdr); q.bitmaps = at<uint32_t>(ws, L.bitmaps);
    q.tbits = threshold_bits(threshold);
    q.CA = CA; q.SCA = SCA; q.outlier_idx = outlier_idx; q.n_outliers = n_outliers;
    q.kcap = L.kcap;
    return from_cuda(launch_quantize(q, s));
}

int int8lt_forward(const void *X, int64_t M, int64_t N, int64_t K, const int8_t *CB, const float *SCB,
                   const void *W_outlier, float threshold, const void *bias, void *Y, void *ws,
                   size_t ws_bytes, void *stream) {
    int st = check_forward_args(X, M, N, K, CB, SCB, W_outlier, threshold, bias, Y, true, true, ws, ws_bytes);
    if (st) return st < 0 ? INT8LT_OK : st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = forward_quantize(X, M, N, K, CB, SCB, W_outlier, threshold, ws, s))) return st;
    return forward_matmul(M, N, K, CB, SCB, W_outlier, bias, Y, ws, s);
}

int int8lt_forward_quantize(const void *X, int64_t M, int64_t N, int64_t K, const int8_t *CB, const float *SCB,
                            const void *W_outlier, float threshold, void *ws, size_t ws_bytes, void *stream) {
    int st = check_forward_args(X, M, N, K, CB, SCB, W_outlier, threshold, nullptr, nullptr, true, false, ws,
                                ws_bytes);
    if (st) return st < 0 ? INT8LT_OK : st;
    return forward_quantize(X, M, N, K, CB, SCB, W_outlier, threshold, ws, static_cast<cudaStream_t>(stream));
}

int int8lt_forward_matmul(int64_t M, int64_t N, int64_t K, const int8_t *CB, const float *SCB,
                          const void *W_outlier, const void *bias, void *Y, void *ws, size_t ws_bytes,
                          void *stream) {
    int st = check_forward_args(nullptr, M, N, K, CB, SCB, W_outlier, 0.f, bias, Y, false, true, ws, ws_bytes);
    if (st) return st < 0 ? INT8LT_OK : st;
    return forward_matmul(M, N, K, CB, SCB, W_outlier, bias, Y, ws, static_cast<cudaStream_t>(stream));
}

int int8lt_quantize_rows_zp(const void *X, int64_t R, int64_t K, int8_t *Q, float *ND, int32_t *ZP,
                            int32_t *SUM, void *stream) {
    if (!shape_ok(R, 8, K)) return INT8LT_ERR_SHAPE;
    if (R == 0) return INT8LT_OK;
    if (!X || !Q || !ND || !ZP || !SUM) return INT8LT_ERR_NULL;
    if (!aligned(X, 16) || !aligned(Q, 16) || !aligned(ND, 4) || !aligned(ZP, 4) || !aligned(SUM, 4))
        return INT8LT_ERR_ALIGN;
    if (int st = check_device()) return st;
    ZpQuantArgs z{};
    z.X = static_cast<const __half *>(X); z.R = R; z.K = K;
    z.Q = Q; z.ND = ND; z.ZP = ZP; z.SUM = SUM;
    return from_cuda(launch_zp_quantize(z, static_cast<cudaStream_t>(stream)));
}

int int8lt_prepare_weight_zp(const void *W, int64_t N, int64_t K, int8_t *CB, float *NDB, int32_t *ZB,
                             int32_t *SB, void *stream) {
    if (!shape_ok(8, N, K)) return INT8LT_ERR_SHAPE;
    if (N == 0) return INT8LT_OK;
    if (!W || !CB || !NDB || !ZB || !SB) return INT8LT_ERR_NULL;
    if (!aligned(W, 16) || !aligned(CB, 16) || !aligned(NDB, 4) || !aligned(ZB, 4) || !aligned(SB, 4))
        return INT8LT_ERR_ALIGN;
    if (int st = check_device()) return st;
    ZpQuantArgs z{};
    z.X = static_cast<const __half *>(W); z.R = N; z.K = K;
    z.Q = CB; z.blocked = true; z.ND = NDB; z.ZP = ZB; z.SUM = SB;
    return from_cuda(launch_zp_quantize(z, static_cast<cudaStream_t>(stream)));
}

int int8lt_forward_zp_quantize(const void *X, int64_t M, int64_t N, int64_t K, void *ws, size_t ws_bytes,
                               void *stream) {
    if (!shape_ok(M, N, K)) return INT8LT_ERR_SHAPE;
    if (M == 0 || N == 0) return INT8LT_OK;
    if (!X || !ws) return INT8LT_ERR_NULL;
    if (!aligned(X, 16) || !aligned(ws, 16)) return INT8LT_ERR_ALIGN;
    const WsLayout L = ws_layout(M, N, K);
    if (ws_bytes < L.total) return INT8LT_ERR_WORKSPACE;
    if (int st = check_device()) return st;
    ZpQuantArgs z{};
    z.X = static_cast<const __half *>(X); z.R = M; z.K = K;
    z.Q = at<int8_t>(ws, L.ca); z.ND = at<float>(ws, L.sca);
    z.ZP = at<int32_t>(ws, L.zpa); z.SUM = z.ZP + M;
    if (M <= kDecodeMaxM) {  // the GEMV's partial sums and counters start at zero
        z.acc = at<int32_t>(ws, L.acc); z.acc_words = round_up(N * M, 4);
        z.cnt = at<uint32_t>(ws, L.cnt); z.cnt_words = round_up(ceil_div(N, 8), 4);
    }
    return from_cuda(launch_zp_quantize(z, static_cast<cudaStream_t>(stream)));
}

int int8lt_forward_zp_matmul(int64_t M, int64_t N, int64_t K, const int8_t *CB, const float *NDB,
                             const int32_t *ZB, const int32_t *SB, const void *bias, void *Y, void *ws,
                             size_t ws_bytes, void *stream) {
    int st = check_zp_weight_args(M, N, K, ZB, SB);
    if (!st) st = check_forward_args(nullptr, M, N, K, CB, NDB, nullptr, 0.f, bias, Y, false, true, ws, ws_bytes);
    if (st) return st < 0 ? INT8LT_OK : st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const WsLayout L = ws_layout(M, N, K);
    WsHeader *hdr = at<WsHeader>(ws, L.hdr);
    const int8_t *CA = at<int8_t>(ws, L.ca);
    const float *NDA = at<float>(ws, L.sca);
    const int32_t *ZA = at<int32_t>(ws, L.zpa), *SA = ZA + M;
    if (M <= kDecodeMaxM) {
        GemvArgs g{};
        g.CA = CA; g.CB = CB; g.SCA = NDA; g.SCB = NDB;
        g.ZA = ZA; g.SA = SA; g.ZB = ZB; g.SB = SB;
        g.bias = static_cast<const __half *>(bias); g.Y = static_cast<__half *>(Y);
        g.acc = at<int32_t>(ws, L.acc); g.cnt = at<uint32_t>(ws, L.cnt); g.status = &hdr->status;
        g.M = M; g.N = N; g.K = K;
        return from_cuda(launch_gemv(g, s));
    }
    GemmArgs g{};
    g.CA = CA; g.CB = CB; g.SCA = NDA; g.SCB = NDB;
    g.ZA = ZA; g.SA = SA; g.ZB = ZB; g.SB = SB;
    g.bias = static_cast<const __half *>(bias); g.Y = static_cast<__half *>(Y);
    g.M = M; g.N = N; g.K = K; g.status = &hdr->status;
    g.sk_partial = at<int32_t>(ws, L.sk);
    g.sk_flags = at<uint32_t>(ws, kWsSkFlagOffset);
    return from_cuda(launch_gemm_tc(g, s));
}

int int8lt_forward_zp(const void *X, int64_t M, int64_t N, int64_t K, const int8_t *CB, const float *NDB,
                      const int32_t *ZB, const int32_t *SB, const void *bias, void *Y, void *ws, size_t ws_bytes,
                      void *stream) {
    int st = check_zp_weight_args(M, N, K, ZB, SB);
    if (!st) st = check_forward_args(X, M, N, K, CB, NDB, nullptr, 0.f, bias, Y, true, true, ws, ws_bytes);
    if (st) return st < 0 ? INT8LT_OK : st;
    if ((st = int8lt_forward_zp_quantize(X, M, N, K, ws, ws_bytes, stream))) return st;
    return int8lt_forward_zp_matmul(M, N, K, CB, NDB, ZB, SB, bias, Y, ws, ws_bytes, stream);
}

int int8lt_debug_gemm_i32(const int8_t *CA, const int8_t *CB, int64_t M, int64_t N, int64_t K, int32_t *C,
                          void *ws, size_t ws_bytes, void *stream) {
    if (!shape_ok(M, N, K)) return INT8LT_ERR_SHAPE;
    if (M == 0 || N == 0) return INT8LT_OK;
    if (!CA || !CB || !C || !ws) return INT8LT_ERR_NULL;
    if (!aligned(CA, 16) || !aligned(CB, 16) || !aligned(C, 16) || !aligned(ws, 16)) return INT8LT_ERR_ALIGN;
    const WsLayout L = ws_layout(M, N, K);
    if (ws_bytes < L.total) return INT8LT_ERR_WORKSPACE;
    if (int st = check_device()) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    WsHeader *hdr = at<WsHeader>(ws, L.hdr);
    if (M <= kDecodeMaxM) {
        GemvArgs g{};
        g.CA = CA; g.CB = CB; g.C32 = C;
        g.M = M; g.N = N; g.K = K; g.status = &hdr->status;
        g.acc = at<int32_t>(ws, L.acc);
        g.cnt = at<uint32_t>(ws, L.cnt);
        if (cudaMemsetAsync(g.acc, 0, (size_t)N * M * 4, s) != cudaSuccess ||
            cudaMemsetAsync(g.cnt, 0, (size_t)ceil_div(N, 8) * 4, s) != cudaSuccess)
            return INT8LT_ERR_CUDA;
        return from_cuda(launch_gemv(g, s));
    }
    GemmArgs g{};
    g.CA = CA; g.CB = CB; g.C32 = C;
    g.M = M; g.N = N; g.K = K; g.status = &hdr->status;
    g.sk_partial = at<int32_t>(ws, L.sk);
    g.sk_flags = at<uint32_t>(ws, kWsSkFlagOffset);
    return from_cuda(launch_gemm_tc(g, s));
}

int int8lt_debug_wait_timeout(void *ws, size_t ws_bytes, int64_t limit_ns, void *stream) {
    if (!ws) return INT8LT_ERR_NULL;
    if (ws_bytes < sizeof(WsHeader)) return INT8LT_ERR_WORKSPACE;
    if (!aligned(ws, 16)) return INT8LT_ERR_ALIGN;
    if (limit_ns < 1000 || limit_ns > 1000000000) return INT8LT_ERR_VALUE;
    if (int st = check_device()) return st;
    WsHeader *hdr = static_cast<WsHeader *>(ws);
    return from_cuda(launch_wait_timeout(&hdr->status, (uint64_t)limit_ns, static_cast<cudaStream_t>(stream)));
}

int int8lt_debug_barrier_timeout(void *ws, size_t ws_bytes, int64_t limit_ns, void *stream) {
    if (!ws) return INT8LT_ERR_NULL;
    if (ws_bytes < kWsInitBytes) return INT8LT_ERR_WORKSPACE;
    if (!aligned(ws, 16)) return INT8LT_ERR_ALIGN;
    if (limit_ns < 1000 || limit_ns > 1000000000) return INT8LT_ERR_VALUE;
    if (int st = check_device()) return st;
    return from_cuda(launch_barrier_timeout(static_cast<WsHeader *>(ws), (uint64_t)limit_ns,
                                            static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
