// Zeropoint (asymmetric) row quantization: "8-bit Data Types and
// Quantization", zeropoint quantization (LLM.int8() paper summary).
//
// Each row x of an fp16 matrix [R, K] (a token of X, or an output channel of
// W) is scaled by its normalized dynamic range nd = 254 / (max x - min x)
// and shifted by its zeropoint zp = rint(nd min x) + 127, so that its codes
// clamp(rint(nd x) - zp, -127, 127) span the whole int8 range; x is
// recovered as (code + zp) / nd. A constant row takes nd = 1. Every step
// is one fp32 operation rounded to nearest even (254 / range, nd * min,
// nd * x), which is what makes the codes reproducible bit for bit. Besides
// the codes the pass writes nd, zp and the sum of the row's codes, the three
// per-row terms that the unrolled product (A + zp_a)(B + zp_b) needs.
//
// Weight rows (output channels) are written in the blocked weight layout
// (4 KB blocks of 32 rows x 128 bytes, padding zeroed), activation rows
// row-major. One CTA (8 warps) per row for long rows or few rows, one warp
// per row otherwise; rows are read twice with 16-byte loads (min/max, then codes),
// the second time mostly from L1. The pass also zeroes the decode GEMV's
// partial sums and counters when asked, as the absmax quantize pass does.
#include <algorithm>

#include "int8lt_internal.cuh"

namespace int8lt {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ uint4 ld_row(const __half *p) { return __ldg(reinterpret_cast<const uint4 *>(p)); }

__device__ __forceinline__ void minmax8(const uint4 &v, __half2 &mn, __half2 &mx) {
    const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        mn = __hmin2(mn, h[i]);
        mx = __hmax2(mx, h[i]);
    }
}

// Codes of 8 values, packed little-endian into 8 bytes; adds them to sum.
__device__ __forceinline__ uint2 codes8(const uint4 &v, float nd, int32_t zp, int32_t &sum) {
    const __half2 *h = reinterpret_cast<const __half2 *>(&v);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(h[i]);
        int32_t c0 = __float2int_rn(__fmul_rn(f.x, nd)) - zp;
        int32_t c1 = __float2int_rn(__fmul_rn(f.y, nd)) - zp;
        c0 = c0 > 127 ? 127 : (c0 < -127 ? -127 : c0);
        c1 = c1 > 127 ? 127 : (c1 < -127 ? -127 : c1);
        sum += c0 + c1;
        w[i >> 1] |= (((uint32_t)c0 & 0xffu) | (((uint32_t)c1 & 0xffu) << 8)) << (16 * (i & 1));
    }
    return make_uint2(w[0], w[1]);
}

// kWarpsPerRow = 1: each warp owns a row (8 rows per CTA);
// kWarpsPerRow = 8: the whole CTA owns a row.
template <int kWarpsPerRow>
__global__ void __launch_bounds__(kThreads) zp_quantize_kernel(const ZpQuantArgs a) {
    constexpr int kRowsPerCta = kWarps / kWarpsPerRow;
    constexpr int kLanes = 32 * kWarpsPerRow;
    __shared__ float s_mn[kWarps], s_mx[kWarps];
    __shared__ int32_t s_sum[kWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = (warp % kWarpsPerRow) * 32 + lane;  // thread within the row's group

    // Decode GEMV partial sums and counters (zero before it accumulates).
    {
        const int64_t tid = (int64_t)blockIdx.x * kThreads + threadIdx.x;
        const int64_t nth = (int64_t)gridDim.x * kThreads;
        if (a.acc)
            for (int64_t i = tid; i < a.acc_words / 4; i += nth)
                reinterpret_cast<int4 *>(a.acc)[i] = make_int4(0, 0, 0, 0);
        if (a.cnt)
            for (int64_t i = tid; i < a.cnt_words / 4; i += nth)
                reinterpret_cast<uint4 *>(a.cnt)[i] = make_uint4(0, 0, 0, 0);
        // Blocked weight layout: rows past R inside the last row block are zero codes.
        if (a.blocked) {
            const int64_t KB = wblocks_k(a.K), per_row = KB * kWBlockCols / 16;
            const int64_t pad = (round_up(a.R, kWBlockRows) - a.R) * per_row;
            for (int64_t i = tid; i < pad; i += nth)
                *reinterpret_cast<uint4 *>(a.Q + cb_offset(a.R + i / per_row, (i % per_row) * 16, KB)) =
                    make_uint4(0, 0, 0, 0);
        }
    }

    const int64_t nvec = a.K / 8;
    const int64_t groups = ceil_div(a.R, kRowsPerCta);
    for (int64_t grp = blockIdx.x; grp < groups; grp += gridDim.x) {
        const int64_t row = grp * kRowsPerCta + warp / kWarpsPerRow;
        const bool live = row < a.R;  // uniform over the row's warps
        const __half *x = a.X + (live ? row : 0) * a.K;

        // Pass 1: min and max (fp16 comparisons are exact).
        __half2 hmn = __float2half2_rn(65504.f), hmx = __float2half2_rn(-65504.f);
        if (live)
            for (int64_t v = t; v < nvec; v += kLanes) minmax8(ld_row(x + v * 8), hmn, hmx);
        float mn = fminf(__low2float(hmn), __high2float(hmn));
        float mx = fmaxf(__low2float(hmx), __high2float(hmx));
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        if constexpr (kWarpsPerRow > 1) {
            if (lane == 0) {
                s_mn[warp] = mn;
                s_mx[warp] = mx;
            }
            __syncthreads();
#pragma unroll
            for (int w = 0; w < kWarpsPerRow; ++w) {
                mn = fminf(mn, s_mn[w]);
                mx = fmaxf(mx, s_mx[w]);
            }
        }

        // nd and zp, each one fp32 operation.
        const float range = __fsub_rn(mx, mn);
        const float nd = range > 0.f ? __fdiv_rn(254.f, range) : 1.f;
        const int32_t zp = __float2int_rn(__fmul_rn(mn, nd)) + 127;

        // Pass 2: codes and their sum.
        int32_t sum = 0;
        if (live && a.blocked) {
            const int64_t KB = wblocks_k(a.K);
            for (int64_t v = t; v < nvec; v += kLanes)
                *reinterpret_cast<uint2 *>(a.Q + cb_offset(row, v * 8, KB)) = codes8(ld_row(x + v * 8), nd, zp, sum);
            for (int64_t v = nvec + t; v < KB * kWBlockCols / 8; v += kLanes)  // padding columns
                *reinterpret_cast<uint2 *>(a.Q + cb_offset(row, v * 8, KB)) = make_uint2(0u, 0u);
        } else if (live) {
            for (int64_t v = t; v < nvec; v += kLanes)
                *reinterpret_cast<uint2 *>(a.Q + row * a.K + v * 8) = codes8(ld_row(x + v * 8), nd, zp, sum);
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if constexpr (kWarpsPerRow > 1) {
            if (lane == 0) s_sum[warp] = sum;
            __syncthreads();
            sum = 0;
#pragma unroll
            for (int w = 0; w < kWarpsPerRow; ++w) sum += s_sum[w];
            __syncthreads();  // s_mn / s_mx / s_sum free for the next row
        }
        if (live && t == 0) {
            a.ND[row] = nd;
            a.ZP[row] = zp;
            a.SUM[row] = sum;
        }
    }
}

}  // namespace

cudaError_t launch_zp_quantize(const ZpQuantArgs &a, cudaStream_t s) {
    if (a.R <= 0) return cudaSuccess;
    const bool per_cta = a.K >= 2048 || a.R < 4 * 148;
    const int64_t groups = per_cta ? a.R : ceil_div(a.R, kWarps);
    const int64_t pad = a.blocked ? (round_up(a.R, kWBlockRows) - a.R) * wblocks_k(a.K) * kWBlockCols / 4 : 0;
    const int64_t clear = ceil_div((a.acc ? a.acc_words : 0) + (a.cnt ? a.cnt_words : 0) + pad, 4 * kThreads);
    int64_t grid = std::max<int64_t>(groups, std::min<int64_t>(clear, 148 * 4));
    grid = std::min<int64_t>(grid, (int64_t)1 << 20);
    if (per_cta)
        zp_quantize_kernel<kWarps><<<(unsigned)grid, kThreads, 0, s>>>(a);
    else
        zp_quantize_kernel<1><<<(unsigned)grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace int8lt
