// Decode path (M <= 16 tokens) of the LLM.int8() forward.
//
// Same arithmetic as the prefill GEMM ("Int8 Matrix Multiplication with
// 16-bit Float Inputs and Outputs", "Vector-wise Quantization" and "The Core
// of LLM.int8(): Mixed-precision Decomposition", LLM.int8() paper summary),
// but with at most 16 tokens the work is bound by streaming CB from HBM
// (N*K bytes, e.g. 604 MB for a 49152 x 12288 projection), so the design
// goal is sequential bytes in flight on every SM, not tensor throughput:
//   - CB is stored in 4 KB blocks of 32 output channels x 128 bytes of K,
//     row block by row block, so the whole of CB is one sequence of blocks;
//   - warp w streams blocks [w L, (w + 1) L) of that sequence: one contiguous
//     range per warp, the same length for every warp (balanced to one block
//     over the whole grid, 3 CTAs of 8 warps per SM);
//   - each lane issues 256-bit loads (4 per block, the block's 32 rows x 128
//     bytes over the warp; 16-byte loads when CB is only 16-byte aligned) and
//     the matching CA bytes; mma.sync m16n8k32
//     (int8 -> int32) with the tokens as the 16-row A operand and 8 weight
//     rows as B. The K order inside one MMA is irrelevant to an exact integer
//     sum, so the bytes a lane loaded are used as they lie, with the same
//     permutation applied to A and B;
//   - where a warp's range starts or ends inside a row block, its int32
//     partial sums are added with atomics (exact in any order) and the last
//     of the row block's warps, found with an arrival counter, runs the
//     epilogue (the quantize pass zeroes the sums and the counters);
//   - launched with programmatic stream serialization, each warp pulls the
//     first blocks of its range into L2 before it waits for the quantize pass.
// A read-bandwidth probe on this machine measured this pattern at 6.1-6.4 TB/s
// with 16-byte loads, against 4.5 TB/s for 32 row-major rows read 128 bytes
// at a time and 5.1-5.3 TB/s for blocked rows split by row block alone
// (uneven per SM); the 256-bit evict-first loads took the kernel to about
// 6.3-6.8 TB/s.
#include <algorithm>
#include <atomic>

#include "int8lt_internal.cuh"

namespace int8lt {

namespace {

constexpr int kWarpsPerCta = 8;
constexpr int kCtasPerSm = 3;
constexpr int64_t kMinBlocksPerWarp = 4;  // fewer would turn the sums into mostly atomics
constexpr int64_t kPrefetchBlocks = 4;    // blocks each warp pulls into L2 before the wait

__device__ __forceinline__ void mma_16832_s8(int32_t (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 32 contiguous bytes (one 256-bit load; p 32-byte aligned), read once:
// not kept in L1 and first out of L2, so that CA stays cached.
__device__ __forceinline__ void ld_stream32(const int8_t *p, uint4 &lo, uint4 &hi) {
    asm volatile("ld.global.nc.L1::no_allocate.L2::evict_first.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(lo.x), "=r"(lo.y), "=r"(lo.z), "=r"(lo.w), "=r"(hi.x), "=r"(hi.y), "=r"(hi.z), "=r"(hi.w)
                 : "l"(p));
}

__device__ __forceinline__ uint4 ld_stream(const int8_t *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ float outlier_weight(const GemvArgs &a, int64_t j, int64_t col) {
    if (!IN_BOUNDS(col >= 0 && col < a.K, a.status)) return 0.f;
    if (a.W_outlier) return __half2float(a.W_outlier[j * a.K + col]);
    const float p = __fmul_rn((float)a.CB[cb_offset(j, col, wblocks_k(a.K))], a.SCB[j]);
    return __half2float(__float2half_rn(__fdiv_rn(p, 127.f)));
}

// Final value of output (token t, channel j) from its int32 sum; p is the
// outlier product of (t, j) (0 without outliers).
__device__ __forceinline__ float finish(const GemvArgs &a, int64_t t, int64_t j, int32_t c, float p) {
    float y;
    if (a.ZB) {
        // Zeropoint mode: (A + zp_a)(B + zp_b) unrolled into the int8 sum and
        // three exact int64 corrections ("8-bit Data Types and Quantization").
        const int64_t za = a.ZA[t], zb = a.ZB[j];
        const int64_t ct = (int64_t)c + zb * ((int64_t)a.SA[t] + a.K * za) + za * (int64_t)a.SB[j];
        y = __fmul_rn(__ll2float_rn(ct), 1.0f / a.SCA[t]) * (1.0f / a.SCB[j]);
    } else {
        y = (float)c * (a.SCA[t] * (1.0f / 16129.0f) * a.SCB[j]) + p;
    }
    if (a.bias) y += __half2float(a.bias[j]);
    return y;
}

// Outlier product of the row block [n0, n0 + 32) for every token, into
// s_p[t][r] (r = row in the block): lane r owns channel n0 + r, loads its
// |O| fp16 outlier weights (four at a time, independent loads) and the
// tokens' outlier activations (small, cached), and sums in fp32.
__device__ __forceinline__ void outlier_rows(const GemvArgs &a, int n_out, int64_t n0, int lane,
                                          float (*s_p)[32]) {
    const int64_t j = n0 + lane;
    float p[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) p[t] = 0.f;
    if (j < a.N) {
        for (int o0 = 0; o0 < n_out; o0 += 4) {
            float wv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                wv[u] = o0 + u < n_out ? outlier_weight(a, j, a.outlier_idx[o0 + u]) : 0.f;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (o0 + u >= n_out) break;
#pragma unroll
                for (int t = 0; t < 16; ++t)
                    if (t < a.M) p[t] += __half2float(a.Xo[t * a.kcap + o0 + u]) * wv[u];
            }
        }
    }
#pragma unroll
    for (int t = 0; t < 16; ++t) s_p[t][lane] = p[t];
}

// Epilogue of one row block: Y (or the raw sums) of channels n0 .. n0 + 31.
// Fragment owner: d[q][0..1] -> token g, channels n0 + 8q + 2tig + {0,1};
//                 d[q][2..3] -> token g + 8, same channels.
__device__ __forceinline__ void row_block_out(const GemvArgs &a, int n_out, int64_t n0, int lane,
                                              const int32_t (&d)[4][4], float (*s_p)[32]) {
    const int g = lane >> 2, tig = lane & 3;
    if (n_out > 0 && !a.C32) {
        outlier_rows(a, n_out, n0, lane, s_p);
        __syncwarp();
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
            const int64_t t = g + hi * 8, j = n0 + 8 * q + 2 * tig;
            if (t >= a.M || j >= a.N) continue;  // N % 8 == 0: j + 1 < N too
            if (!IN_BOUNDS(t * a.N + j + 1 < a.M * a.N, a.status)) continue;
            const int32_t c0 = d[q][2 * hi], c1 = d[q][2 * hi + 1];
            if (a.C32) {
                *reinterpret_cast<int2 *>(a.C32 + t * a.N + j) = make_int2(c0, c1);
            } else {
                const int r = 8 * q + 2 * tig;
                const float p0 = n_out > 0 ? s_p[t][r] : 0.f, p1 = n_out > 0 ? s_p[t][r + 1] : 0.f;
                *reinterpret_cast<__half2 *>(a.Y + t * a.N + j) =
                    __floats2half2_rn(finish(a, t, j, c0, p0), finish(a, t, j + 1, c1, p1));
            }
        }
    if (n_out > 0 && !a.C32) __syncwarp();  // s_p is free for the next row block
}

// kHi: more than 8 tokens (the MMA's rows 8..15 are live). kOut: the
// absmax forward, whose outlier term is read from the workspace (|O| may still
// be 0); without it (zeropoint, raw int32 sums) no outlier code is compiled.
// kWide: CB is 32-byte aligned, and each lane reads its 32 bytes of a block
// row with one 256-bit load (else two 16-byte loads 64 bytes apart).
template <bool kHi, bool kOut, bool kWide>
__global__ void __launch_bounds__(kWarpsPerCta * 32, kCtasPerSm)
gemv_i8_kernel(const GemvArgs a, const int64_t L) {
    __shared__ float s_p[kOut ? kWarpsPerCta : 1][16][32];  // outlier products of a row block, per warp
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, tig = lane & 3;
    const int64_t w = (int64_t)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
    const int64_t KB = wblocks_k(a.K);
    const int64_t total = ceil_div(a.N, kWBlockRows) * KB;  // 4 KB blocks of CB
    int64_t s = w * L;
    const int64_t s1 = min(total, s + L);
    if (s >= s1) return;

    // Until the quantize pass before this kernel has finished, only CB (which
    // it does not write) may be touched: pull the first blocks of this warp's
    // range into L2, then wait.
    if (lane == 0) {
        const int64_t nb = min(s1 - s, kPrefetchBlocks);
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.CB + s * kWBlockBytes),
                     "r"((uint32_t)(nb * kWBlockBytes))
                     : "memory");
    }
    grid_dep_wait();

    const bool tok_lo = g < a.M, tok_hi = kHi && g + 8 < a.M;
    const int8_t *xa = a.CA + (int64_t)g * a.K;
    const int8_t *xb = a.CA + (int64_t)(g + 8) * a.K;
    int n_out = kOut ? *a.n_outliers : 0;
    if (!IN_BOUNDS(n_out >= 0 && n_out <= a.kcap, a.status)) n_out = 0;
    const uint4 z = make_uint4(0, 0, 0, 0);
    // This lane's 16-byte pieces of a block: rows 8q + g, bytes 64h + 16tig.
    const int lane_off = g * kWBlockCols + tig * (kWide ? 32 : 16);

    while (s < s1) {
        const int64_t rb = s / KB;                      // row block
        const int64_t seg_end = min(s1, (rb + 1) * KB);
        int32_t d[4][4];
#pragma unroll
        for (int q = 0; q < 4; ++q) d[q][0] = d[q][1] = d[q][2] = d[q][3] = 0;
        for (int64_t st = s; st < seg_end; ++st) {
            const int8_t *blk = a.CB + st * kWBlockBytes + lane_off;
            const int64_t kb = (st - rb * KB) * kWBlockCols;
            uint4 wv[2][4], xl[2], xh[2] = {z, z};
            if constexpr (kWide) {
#pragma unroll
                for (int q = 0; q < 4; ++q) ld_stream32(blk + q * 8 * kWBlockCols, wv[0][q], wv[1][q]);
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                // CB's padding columns are zero codes; CA stops at K. Piece h of
                // this lane holds the same K positions of A and of B.
                const int64_t kk = kb + (kWide ? tig * 32 + h * 16 : h * 64 + tig * 16);
                const bool kin = kk < a.K;
                if constexpr (!kWide) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) wv[h][q] = ld_stream(blk + q * 8 * kWBlockCols + h * 64);
                }
                xl[h] = (kin && tok_lo) ? __ldg(reinterpret_cast<const uint4 *>(xa + kk)) : z;
                if constexpr (kHi) xh[h] = (kin && tok_hi) ? __ldg(reinterpret_cast<const uint4 *>(xb + kk)) : z;
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t a0[4] = {xl[h].x, xh[h].x, xl[h].y, xh[h].y};
                const uint32_t a1[4] = {xl[h].z, xh[h].z, xl[h].w, xh[h].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    mma_16832_s8(d[q], a0, wv[h][q].x, wv[h][q].y);
                    mma_16832_s8(d[q], a1, wv[h][q].z, wv[h][q].w);
                }
            }
        }
        const int64_t n0 = rb * kWBlockRows;
        // Warps whose ranges meet this row block: the first and the last.
        const int64_t w_first = (rb * KB) / L, w_last = ((rb + 1) * KB - 1) / L;
        bool mine = true;
        if (w_first != w_last) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int64_t t = g + (e >> 1) * 8, j = n0 + 8 * q + 2 * tig + (e & 1);
                    if (t < a.M && j < a.N && IN_BOUNDS(j * a.M + t < a.N * a.M, a.status))
                        atomicAdd(&a.acc[j * a.M + t], d[q][e]);
                }
            __threadfence();
            uint32_t old = 0;
            if (lane == 0 && IN_BOUNDS(rb < ceil_div(a.N, 8), a.status)) old = atomicAdd(&a.cnt[rb], 1u);
            old = __shfl_sync(0xffffffffu, old, 0);
            mine = old == (uint32_t)(w_last - w_first);
            if (mine) {
                __threadfence();
#pragma unroll
                for (int q = 0; q < 4; ++q)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int64_t t = g + (e >> 1) * 8, j = n0 + 8 * q + 2 * tig + (e & 1);
                        d[q][e] = (t < a.M && j < a.N) ? __ldcg(&a.acc[j * a.M + t]) : 0;
                    }
            }
        }
        if (mine) row_block_out(a, n_out, n0, lane, d, s_p[kOut ? threadIdx.x >> 5 : 0]);
        s = seg_end;
    }
}

}  // namespace

cudaError_t launch_gemv(const GemvArgs &a, cudaStream_t s) {
    // CTAs of this kernel that fit on the device at once (0: not known yet;
    // threads that race on the first call compute and store the same value).
    static std::atomic<int> resident[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int ctas = resident[dev & 63].load(std::memory_order_relaxed);
    if (ctas == 0) {
        int sms = 0, per_sm = 0;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gemv_i8_kernel<true, true, true>,
                                                              kWarpsPerCta * 32, 0);
        if (e != cudaSuccess) return e;
        ctas = std::max(1, sms * per_sm);
        resident[dev & 63].store(ctas, std::memory_order_relaxed);
    }
    const int64_t total = ceil_div(a.N, kWBlockRows) * wblocks_k(a.K);
    const int64_t warps_max = (int64_t)ctas * kWarpsPerCta;
    const int64_t L = std::max(kMinBlocksPerWarp, ceil_div(total, warps_max));
    const int64_t warps = ceil_div(total, L);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)ceil_div(warps, kWarpsPerCta), 1, 1);
    cfg.blockDim = dim3(kWarpsPerCta * 32, 1, 1);
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const bool out = a.n_outliers && !a.ZB && !a.C32;
    const bool wide = (reinterpret_cast<uintptr_t>(a.CB) & 31) == 0;
    if (wide) {
        if (a.M > 8)
            return out ? cudaLaunchKernelEx(&cfg, gemv_i8_kernel<true, true, true>, a, L)
                       : cudaLaunchKernelEx(&cfg, gemv_i8_kernel<true, false, true>, a, L);
        return out ? cudaLaunchKernelEx(&cfg, gemv_i8_kernel<false, true, true>, a, L)
                   : cudaLaunchKernelEx(&cfg, gemv_i8_kernel<false, false, true>, a, L);
    }
    if (a.M > 8)
        return out ? cudaLaunchKernelEx(&cfg, gemv_i8_kernel<true, true, false>, a, L)
                   : cudaLaunchKernelEx(&cfg, gemv_i8_kernel<true, false, false>, a, L);
    return out ? cudaLaunchKernelEx(&cfg, gemv_i8_kernel<false, true, false>, a, L)
               : cudaLaunchKernelEx(&cfg, gemv_i8_kernel<false, false, false>, a, L);
}

}  // namespace int8lt
