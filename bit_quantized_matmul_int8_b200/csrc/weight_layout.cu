// The blocked weight layout of CB and its conversions from and to plain
// row-major int8 codes [N, K].
//
// The layout (4 KB blocks of 32 output channels x 128 bytes of K, row block
// by row block, zero codes in the padding) is this library's storage choice
// for the B200, not a format the method defines: the decode GEMV streams one
// contiguous range of blocks per warp, and the prefill GEMM's TMA reads a
// 128-channel k-block as four whole blocks. These conversions let codes made
// elsewhere (row-major CB, e.g. from another LLM.int8() implementation) be
// used here, and let row-major codes be read back.
#include <algorithm>

#include "int8lt_internal.cuh"

namespace int8lt {

namespace {

constexpr int kThreads = 256;

// One 16-byte piece of the blocked layout per thread (grid-stride).
template <bool kPack>
__global__ void __launch_bounds__(kThreads) convert_kernel(int8_t *blocked, int8_t *rows, int64_t N, int64_t K) {
    const int64_t KB = wblocks_k(K);
    const int64_t pieces = weight_bytes(N, K) / 16;
    const bool vec = (K % 16) == 0;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < pieces; i += (int64_t)gridDim.x * kThreads) {
        const int64_t o = i * 16, b = o / kWBlockBytes, in = o % kWBlockBytes;
        const int64_t j = (b / KB) * kWBlockRows + in / kWBlockCols;
        const int64_t k = (b % KB) * kWBlockCols + in % kWBlockCols;
        uint4 *dst4 = reinterpret_cast<uint4 *>(blocked + o);
        if (kPack) {
            if (j < N && k < K && vec) {
                *dst4 = *reinterpret_cast<const uint4 *>(rows + j * K + k);
            } else {
                alignas(16) int8_t v[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] = (j < N && k + e < K) ? rows[j * K + k + e] : (int8_t)0;
                *dst4 = *reinterpret_cast<const uint4 *>(v);
            }
        } else if (j < N && k < K) {
            if (vec) {
                *reinterpret_cast<uint4 *>(rows + j * K + k) = *dst4;
            } else {
                for (int e = 0; e < 16 && k + e < K; ++e) rows[j * K + k + e] = blocked[o + e];
            }
        }
    }
}

}  // namespace

cudaError_t launch_convert_weight(bool pack, int8_t *blocked, int8_t *rows, int64_t N, int64_t K, cudaStream_t s) {
    const int64_t pieces = weight_bytes(N, K) / 16;
    if (pieces == 0) return cudaSuccess;
    const unsigned grid = (unsigned)std::min<int64_t>(ceil_div(pieces, kThreads), 148 * 16);
    if (pack)
        convert_kernel<true><<<grid, kThreads, 0, s>>>(blocked, rows, N, K);
    else
        convert_kernel<false><<<grid, kThreads, 0, s>>>(blocked, rows, N, K);
    return cudaGetLastError();
}

}  // namespace int8lt
