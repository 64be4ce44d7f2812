// Decode path (M <= 16 tokens) of the LLM.int8() forward.
//
// Same arithmetic as the prefill GEMM ("Int8 Matrix Multiplication with
// 16-bit Float Inputs and Outputs", "Vector-wise Quantization" and "The Core
// of LLM.int8(): Mixed-precision Decomposition", LLM.int8() paper summary),
// but with at most 16 tokens the work is bound by streaming CB from HBM
// (N*K bytes, e.g. 604 MB for a 49152 x 12288 projection), so the design
// goal is bytes in flight, not tensor throughput:
//   - one warp owns 32 output channels (4 groups of 8) and a K range;
//   - each lane issues 16-byte loads of CB rows (64 contiguous bytes per row
//     per warp-step) and of the matching CA bytes;
//   - mma.sync m16n8k32 (int8 -> int32) with the tokens as the 16-row A
//     operand and 8 weight rows as B. The K order inside one MMA is
//     irrelevant to an exact integer sum, so the 16 bytes a lane loaded are
//     used as they lie, with the same permutation applied to A and B;
//   - K is split across warps when N alone gives too few warps; the int32
//     partial sums are added with atomics (exact in any order) and the last
//     warp of a row group, found with an arrival counter, runs the epilogue
//     (the quantize pass zeroes the sums and the counters);
//   - launched with programmatic stream serialization, each warp starts
//     pulling the first kilobyte of its weight rows into L2 before it waits
//     for the quantize pass.
// Each warp reads 32 rows 128 bytes at a time. A read-bandwidth probe on
// this pool put that pattern at about 4.2-4.9 TB/s against 6.5-6.8 TB/s for
// reads of 1 KB or more per row; designs that stream longer pieces per row
// (TMA boxes of 64 rows x 128 bytes issued eight at a time, per-row 1 KB
// bulk copies) measured slower here, so this one stays.
#include <algorithm>

#include "int8lt_internal.cuh"

namespace int8lt {

namespace {

constexpr int kWarpsPerCta = 8;
constexpr int kRowsPerWarp = 32;
constexpr int kTargetWarps = 148 * 8;
constexpr int kHalves = 2;  // 64-byte pieces of K per row per step (the step is kHalves * 64 bytes)

// Warps that share the K range of one row group (1 = none).
int gemv_splits(int64_t N, int64_t K) {
    const int64_t rg = ceil_div(N, kRowsPerWarp);
    int64_t s = ceil_div(kTargetWarps, rg);
    s = std::min<int64_t>(s, std::max<int64_t>(1, K / 256));
    return (int)std::max<int64_t>(1, std::min<int64_t>(s, 64));
}

__device__ __forceinline__ void mma_16832_s8(int32_t (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ld_stream(const int8_t *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ float outlier_weight(const GemvArgs &a, int64_t j, int64_t col) {
    if (a.W_outlier) return __half2float(a.W_outlier[j * a.K + col]);
    const float p = __fmul_rn((float)a.CB[j * a.K + col], a.SCB[j]);
    return __half2float(__float2half_rn(__fdiv_rn(p, 127.f)));
}

// Final value of output (token t, channel j) from its int32 sum.
__device__ __forceinline__ void finish(const GemvArgs &a, int n_out, int64_t t, int64_t j, int32_t c,
                                       float &y) {
    if (a.ZB) {
        // Zeropoint mode: (A + zp_a)(B + zp_b) unrolled into the int8 sum and
        // three exact int64 corrections ("8-bit Data Types and Quantization").
        const int64_t za = a.ZA[t], zb = a.ZB[j];
        const int64_t ct = (int64_t)c + zb * ((int64_t)a.SA[t] + a.K * za) + za * (int64_t)a.SB[j];
        y = __fmul_rn(__ll2float_rn(ct), 1.0f / a.SCA[t]) * (1.0f / a.SCB[j]);
        if (a.bias) y += __half2float(a.bias[j]);
        return;
    }
    y = (float)c * (a.SCA[t] * (1.0f / 16129.0f) * a.SCB[j]);
    float p = 0.f;
    for (int o = 0; o < n_out; ++o)
        p += __half2float(a.Xo[t * a.kcap + o]) * outlier_weight(a, j, a.outlier_idx[o]);
    y += p;
    if (a.bias) y += __half2float(a.bias[j]);
}

__global__ void __launch_bounds__(kWarpsPerCta * 32)
gemv_i8_kernel(const GemvArgs a, const int64_t row_groups, const int splits) {
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, tig = lane & 3;
    const int64_t unit = (int64_t)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
    if (unit >= row_groups * splits) return;
    const int64_t rg = unit / splits;
    const int sp = (int)(unit % splits);
    const int64_t n0 = rg * kRowsPerWarp;
    const int64_t kchunk = round_up(ceil_div(a.K, splits), 64);
    const int64_t k0 = sp * kchunk, k1 = min(a.K, k0 + kchunk);

    // Until the quantize pass before this kernel has finished, only CB (which
    // it does not write) may be touched: pull the first kilobyte of each of
    // this warp's 32 weight rows into L2, then wait.
    {
        const int64_t j = n0 + lane;
        if (j < a.N && k0 < k1) {
            const uint32_t bytes = (uint32_t)(k1 - k0 < 1024 ? k1 - k0 : 1024);
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.CB + j * a.K + k0), "r"(bytes)
                         : "memory");
        }
    }
    grid_dep_wait();

    const bool tok_lo = g < a.M, tok_hi = g + 8 < a.M;
    const int8_t *xa = a.CA + (int64_t)g * a.K;
    const int8_t *xb = a.CA + (int64_t)(g + 8) * a.K;
    const int8_t *wr[4];
    bool wok[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int64_t j = n0 + 8 * q + g;
        wok[q] = j < a.N;
        wr[q] = a.CB + (wok[q] ? j : 0) * a.K;
    }

    int32_t d[4][4];
#pragma unroll
    for (int q = 0; q < 4; ++q) d[q][0] = d[q][1] = d[q][2] = d[q][3] = 0;

    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int64_t k = k0; k < k1; k += kHalves * 64) {
        uint4 w[kHalves][4], xl[kHalves], xh[kHalves];
#pragma unroll
        for (int h = 0; h < kHalves; ++h) {
            const int64_t kk = k + h * 64 + tig * 16;
            const bool kin = kk < k1;
#pragma unroll
            for (int q = 0; q < 4; ++q) w[h][q] = (kin && wok[q]) ? ld_stream(wr[q] + kk) : z;
            xl[h] = (kin && tok_lo) ? __ldg(reinterpret_cast<const uint4 *>(xa + kk)) : z;
            xh[h] = (kin && tok_hi) ? __ldg(reinterpret_cast<const uint4 *>(xb + kk)) : z;
        }
#pragma unroll
        for (int h = 0; h < kHalves; ++h) {
            const uint32_t a0[4] = {xl[h].x, xh[h].x, xl[h].y, xh[h].y};
            const uint32_t a1[4] = {xl[h].z, xh[h].z, xl[h].w, xh[h].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                mma_16832_s8(d[q], a0, w[h][q].x, w[h][q].y);
                mma_16832_s8(d[q], a1, w[h][q].z, w[h][q].w);
            }
        }
    }

    // Fragment owner: d[q][0..1] -> token g, channels n0 + 8q + 2tig + {0,1};
    //                 d[q][2..3] -> token g + 8, same channels.
    if (splits > 1) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int64_t t = g + (e >> 1) * 8, j = n0 + 8 * q + 2 * tig + (e & 1);
                if (t < a.M && j < a.N) atomicAdd(&a.acc[j * a.M + t], d[q][e]);
            }
        __threadfence();
        uint32_t old = 0;
        if (lane == 0) old = atomicAdd(&a.cnt[rg], 1u);
        old = __shfl_sync(0xffffffffu, old, 0);
        if (old != (uint32_t)splits - 1) return;
        __threadfence();
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int64_t t = g + (e >> 1) * 8, j = n0 + 8 * q + 2 * tig + (e & 1);
                d[q][e] = (t < a.M && j < a.N) ? __ldcg(&a.acc[j * a.M + t]) : 0;
            }
    }

    const int n_out = (a.n_outliers && !a.ZB) ? *a.n_outliers : 0;
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
            const int64_t t = g + hi * 8, j = n0 + 8 * q + 2 * tig;
            if (t >= a.M || j >= a.N) continue;  // N % 8 == 0: j + 1 < N too
            const int32_t c0 = d[q][2 * hi], c1 = d[q][2 * hi + 1];
            if (a.C32) {
                *reinterpret_cast<int2 *>(a.C32 + t * a.N + j) = make_int2(c0, c1);
            } else {
                float y0, y1;
                finish(a, n_out, t, j, c0, y0);
                finish(a, n_out, t, j + 1, c1, y1);
                *reinterpret_cast<__half2 *>(a.Y + t * a.N + j) = __floats2half2_rn(y0, y1);
            }
        }
}

}  // namespace

cudaError_t launch_gemv(const GemvArgs &a, cudaStream_t s) {
    const int64_t rg = ceil_div(a.N, kRowsPerWarp);
    const int splits = gemv_splits(a.N, a.K);
    const int64_t warps = rg * splits;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)ceil_div(warps, kWarpsPerCta), 1, 1);
    cfg.blockDim = dim3(kWarpsPerCta * 32, 1, 1);
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemv_i8_kernel, a, rg, splits);
}

}  // namespace int8lt
