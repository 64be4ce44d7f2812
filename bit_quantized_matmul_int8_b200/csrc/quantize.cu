// Outlier detection and vector-wise absmax quantization (sm_100a).
//
// Method: "LLM.int8() paper summary" (kurtkim.github.io), "8-bit Data Types
// and Quantization" (absmax equation), "Vector-wise Quantization" and "The
// Core of LLM.int8(): Mixed-precision Decomposition"; "Hugging Face LLM.int8()
// integration" (agentlenshq.com), three-step recipe and CB/SCB weights.
//
// Kernels (all HBM-bound streaming passes with 16-byte coalesced loads):
//   prepare_weight_kernel  W [N,K] -> CB, SCB          (one warp per row)
//   outlier_flags_kernel   X [M,K] -> partial column bitmaps (phase A)
//   quantize_kernel        X, bitmaps -> O, CA, SCA, Xo; gathers Wo; clears
//                          the split-K buffers of the GEMV      (phase B)
//
// Exactness: |x| >= threshold is decided on the fp16 bit pattern against the
// smallest fp16 pattern whose value reaches the fp32 threshold (the map from
// non-negative fp16 patterns to values is monotonic, so this is the fp32
// comparison). The absmax is a max of fp16 magnitudes (exact). The code is
// rint(x * fp32(127 / absmax)) with __fdiv_rn / __fmul_rn / __float2int_rn:
// one IEEE rounding per step, ties to even, never contracted into an FMA.
#include <algorithm>

#include "int8lt_internal.cuh"

namespace int8lt {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ int8_t quant_code(float x, float s) {
    int q = __float2int_rn(__fmul_rn(x, s));
    q = q > 127 ? 127 : (q < -127 ? -127 : q);
    return static_cast<int8_t>(q);
}

__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// max over the 8 fp16 magnitudes in a 16-byte vector, as a bit pattern.
__device__ __forceinline__ uint32_t vec_absmax_bits(uint4 v) {
    uint32_t m = __vmaxu2(__vmaxu2(v.x & 0x7fff7fffu, v.y & 0x7fff7fffu),
                          __vmaxu2(v.z & 0x7fff7fffu, v.w & 0x7fff7fffu));
    return max(m & 0xffffu, m >> 16);
}

__device__ __forceinline__ uint32_t pack4(int8_t a, int8_t b, int8_t c, int8_t d) {
    return (uint32_t)(uint8_t)a | ((uint32_t)(uint8_t)b << 8) | ((uint32_t)(uint8_t)c << 16) |
           ((uint32_t)(uint8_t)d << 24);
}

__device__ __forceinline__ uint2 quant_vec8(uint4 v, float s) {
    const __half2 *h = reinterpret_cast<const __half2 *>(&v);
    float2 f0 = __half22float2(h[0]), f1 = __half22float2(h[1]);
    float2 f2 = __half22float2(h[2]), f3 = __half22float2(h[3]);
    uint2 r;
    r.x = pack4(quant_code(f0.x, s), quant_code(f0.y, s), quant_code(f1.x, s), quant_code(f1.y, s));
    r.y = pack4(quant_code(f2.x, s), quant_code(f2.y, s), quant_code(f3.x, s), quant_code(f3.y, s));
    return r;
}

// ------------------------------------------------------ prepare_weight ----

__global__ void __launch_bounds__(kThreads)
prepare_weight_kernel(const __half *__restrict__ W, int64_t N, int64_t K, int8_t *__restrict__ CB,
                      float *__restrict__ SCB) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * kWarps;
    const bool vec = (K % 8) == 0;
    for (int64_t j = warp; j < N; j += nwarps) {
        const __half *w = W + j * K;
        int8_t *cb = CB + j * K;
        uint32_t amax = 0;
        if (vec) {
            const uint4 *w4 = reinterpret_cast<const uint4 *>(w);
            for (int64_t v = lane; v < K / 8; v += 32) amax = max(amax, vec_absmax_bits(__ldg(w4 + v)));
        } else {
            const uint16_t *wb = reinterpret_cast<const uint16_t *>(w);
            for (int64_t k = lane; k < K; k += 32) amax = max(amax, (uint32_t)(wb[k] & 0x7fffu));
        }
        amax = warp_max_u32(amax);
        const float a = __half2float(__ushort_as_half((unsigned short)amax));
        const float s = a > 0.f ? __fdiv_rn(127.f, a) : 0.f;
        if (vec) {
            const uint4 *w4 = reinterpret_cast<const uint4 *>(w);
            uint2 *c2 = reinterpret_cast<uint2 *>(cb);
            for (int64_t v = lane; v < K / 8; v += 32) c2[v] = quant_vec8(__ldg(w4 + v), s);
        } else {
            for (int64_t k = lane; k < K; k += 32) cb[k] = quant_code(__half2float(w[k]), s);
        }
        if (lane == 0) SCB[j] = a;
    }
}

// ------------------------------------------------------- phase A: flags ----

// Block (x, y): columns [256x, 256x + 256), row chunk y. Each lane owns 8
// consecutive columns (one 16-byte vector per row); the 8 warps stride over
// the chunk's rows. Writes flags[y][8x .. 8x + 8) without atomics.
__global__ void __launch_bounds__(kThreads)
outlier_flags_kernel(const __half *__restrict__ X, int64_t M, int64_t K, uint32_t tbits,
                     uint32_t *__restrict__ flags, int64_t kwords) {
    __shared__ uint32_t sflags[kColsPerFlagCta / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x < kColsPerFlagCta / 32) sflags[threadIdx.x] = 0;
    __syncthreads();
    const int64_t c0 = (int64_t)blockIdx.x * kColsPerFlagCta + lane * 8;
    const int64_t rows_per = ceil_div(M, gridDim.y);
    const int64_t r0 = (int64_t)blockIdx.y * rows_per;
    const int64_t r1 = min(M, r0 + rows_per);
    const uint32_t t2 = tbits | (tbits << 16);
    // hit[w]: per 16-bit half 0xffff where some |x| >= threshold; half 0 of
    // word w is column 2w of the lane's 8 columns, half 1 is column 2w + 1.
    uint32_t hit[4] = {0u, 0u, 0u, 0u};
    if (c0 < K) {
        const __half *xc = X + c0;
        int64_t r = r0 + warp;
        for (; r + 3 * kWarps < r1; r += 4 * kWarps) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                v[u] = __ldg(reinterpret_cast<const uint4 *>(xc + (r + u * kWarps) * K));
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                hit[0] |= __vcmpgeu2(v[u].x & 0x7fff7fffu, t2);
                hit[1] |= __vcmpgeu2(v[u].y & 0x7fff7fffu, t2);
                hit[2] |= __vcmpgeu2(v[u].z & 0x7fff7fffu, t2);
                hit[3] |= __vcmpgeu2(v[u].w & 0x7fff7fffu, t2);
            }
        }
        for (; r < r1; r += kWarps) {
            uint4 v = __ldg(reinterpret_cast<const uint4 *>(xc + r * K));
            hit[0] |= __vcmpgeu2(v.x & 0x7fff7fffu, t2);
            hit[1] |= __vcmpgeu2(v.y & 0x7fff7fffu, t2);
            hit[2] |= __vcmpgeu2(v.z & 0x7fff7fffu, t2);
            hit[3] |= __vcmpgeu2(v.w & 0x7fff7fffu, t2);
        }
    }
    uint32_t byte = 0;  // bit j: column c0 + j is an outlier column
#pragma unroll
    for (int w = 0; w < 4; ++w) byte |= ((hit[w] & 1u) << (2 * w)) | (((hit[w] >> 16) & 1u) << (2 * w + 1));
    if (byte) atomicOr(&sflags[lane >> 2], byte << ((lane & 3) * 8));
    __syncthreads();
    if (threadIdx.x < kColsPerFlagCta / 32) {
        const int64_t word = (int64_t)blockIdx.x * (kColsPerFlagCta / 32) + threadIdx.x;
        if (word < kwords) flags[(int64_t)blockIdx.y * kwords + word] = sflags[threadIdx.x];
    }
}

// -------------------------------------------------- phase B: quantize ----

// Exclusive prefix of popcounts over the smem bitmap; returns |O|.
__device__ int build_prefix(const uint32_t *bits, int32_t *prefix, int64_t kwords) {
    __shared__ int32_t warp_tot[kWarps];
    __shared__ int32_t total;
    const int64_t seg = ceil_div(kwords, kThreads);
    const int64_t w0 = threadIdx.x * seg, w1 = min(kwords, w0 + seg);
    int32_t mine = 0;
    for (int64_t w = w0; w < w1; ++w) mine += __popc(bits[w]);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int32_t incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (threadIdx.x == 0) {
        int32_t acc = 0;
        for (int i = 0; i < kWarps; ++i) {
            int32_t t = warp_tot[i];
            warp_tot[i] = acc;
            acc += t;
        }
        total = acc;
    }
    __syncthreads();
    int32_t run = warp_tot[warp] + incl - mine;
    for (int64_t w = w0; w < w1; ++w) {
        prefix[w] = run;
        run += __popc(bits[w]);
    }
    __syncthreads();
    return total;
}

// Column of the outlier with rank t (0-based) via the prefix array.
__device__ __forceinline__ int64_t outlier_column(const uint32_t *bits, const int32_t *prefix,
                                                  int64_t kwords, int32_t t) {
    int64_t lo = 0, hi = kwords - 1;  // last word with prefix <= t
    while (lo < hi) {
        int64_t mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= t) lo = mid; else hi = mid - 1;
    }
    uint32_t w = bits[lo];
    for (int32_t r = t - prefix[lo]; r > 0; --r) w &= w - 1;  // drop r lowest set bits
    return lo * 32 + (__ffs(w) - 1);
}

__global__ void __launch_bounds__(kThreads)
quantize_kernel(QuantizeArgs a, int64_t kwords, int row_ctas) {
    extern __shared__ uint32_t smem[];
    uint32_t *bits = smem;                                    // [kwords]
    int32_t *prefix = reinterpret_cast<int32_t *>(smem + kwords);  // [kwords]
    // O = OR of the phase-A partial bitmaps.
    for (int64_t w = threadIdx.x; w < kwords; w += kThreads) {
        uint32_t v = 0;
        for (int64_t c = 0; c < a.flag_chunks; ++c) v |= a.flags[c * kwords + w];
        if (w == kwords - 1 && (a.K & 31)) v &= (1u << (a.K & 31)) - 1u;
        bits[w] = v;
    }
    __syncthreads();
    const int32_t n_out = build_prefix(bits, prefix, kwords);
    const int32_t n16 = (n_out + 15) & ~15;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    if (blockIdx.x == 0) {
        if (threadIdx.x == 0 && a.n_outliers) *a.n_outliers = n_out;
        if (a.outlier_idx) {
            for (int64_t w = threadIdx.x; w < kwords; w += kThreads) {
                uint32_t v = bits[w];
                int32_t r = prefix[w];
                while (v) {
                    a.outlier_idx[r++] = (int32_t)(w * 32 + __ffs(v) - 1);
                    v &= v - 1;
                }
            }
        }
    }

    if ((int)blockIdx.x < row_ctas) {
        const int64_t nvec = a.K / 8;
        for (int64_t r = (int64_t)blockIdx.x * kWarps + warp; r < a.M; r += (int64_t)row_ctas * kWarps) {
            const uint4 *x4 = reinterpret_cast<const uint4 *>(a.X + r * a.K);
            uint32_t amax = 0;
            for (int64_t v = lane; v < nvec; v += 32) {
                uint4 x = __ldg(x4 + v);
                uint32_t m = (bits[(v * 8) >> 5] >> ((v * 8) & 31)) & 0xffu;
                if (m == 0) {
                    amax = max(amax, vec_absmax_bits(x));
                } else {
                    const uint16_t *e = reinterpret_cast<const uint16_t *>(&x);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (!((m >> j) & 1u)) amax = max(amax, (uint32_t)(e[j] & 0x7fffu));
                }
            }
            amax = warp_max_u32(amax);
            const float sa = __half2float(__ushort_as_half((unsigned short)amax));
            const float s = sa > 0.f ? __fdiv_rn(127.f, sa) : 0.f;
            uint2 *ca2 = reinterpret_cast<uint2 *>(a.CA + r * a.K);
            __half *xo = a.Xo ? a.Xo + r * a.kcap : nullptr;
            for (int64_t v = lane; v < nvec; v += 32) {
                uint4 x = __ldg(x4 + v);
                uint32_t m = (bits[(v * 8) >> 5] >> ((v * 8) & 31)) & 0xffu;
                uint2 q = quant_vec8(x, s);
                if (m) {
                    const __half *e = reinterpret_cast<const __half *>(&x);
                    uint32_t keep0 = 0, keep1 = 0;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        if ((m >> j) & 1u) {
                            if (xo) {
                                int64_t col = v * 8 + j;
                                int32_t rank = prefix[col >> 5] + __popc(bits[col >> 5] & ((1u << (col & 31)) - 1u));
                                xo[rank] = e[j];
                            }
                        } else {
                            if (j < 4) keep0 |= 0xffu << (8 * j); else keep1 |= 0xffu << (8 * (j - 4));
                        }
                    }
                    q.x &= keep0;
                    q.y &= keep1;
                }
                ca2[v] = q;
            }
            if (xo)
                for (int32_t t = n_out + lane; t < n16; t += 32) xo[t] = __float2half_rn(0.f);
            if (lane == 0) a.SCA[r] = sa;
        }
    } else {
        // Extra blocks: outlier-weight gather and split-K buffer clearing.
        const int64_t eb = blockIdx.x - row_ctas, neb = gridDim.x - row_ctas;
        if (a.Wo) {
            for (int64_t j = eb * kWarps + warp; j < a.N; j += neb * kWarps) {
                __half *wo = a.Wo + j * a.kcap;
                for (int32_t t = lane; t < n16; t += 32) {
                    __half val = __float2half_rn(0.f);
                    if (t < n_out) {
                        int64_t col = outlier_column(bits, prefix, kwords, t);
                        if (a.W_outlier) {
                            val = a.W_outlier[j * a.K + col];
                        } else {
                            float p = __fmul_rn((float)a.CB[j * a.K + col], a.SCB[j]);
                            val = __float2half_rn(__fdiv_rn(p, 127.f));
                        }
                    }
                    wo[t] = val;
                }
            }
        }
        const int64_t tid = eb * kThreads + threadIdx.x, nth = neb * kThreads;
        if (a.acc)
            for (int64_t i = tid; i < a.acc_words; i += nth) a.acc[i] = 0;
        if (a.cnt)
            for (int64_t i = tid; i < a.cnt_words; i += nth) a.cnt[i] = 0;
    }
}

}  // namespace

// --------------------------------------------------------------- host ----

uint16_t threshold_bits(float threshold) {
    // smallest non-negative fp16 pattern b (0 .. 0x7c00) with value(b) >= threshold
    if (!(threshold > 0.f)) return 0;
    uint32_t lo = 0, hi = 0x7c00;  // value(0x7c00) = +inf >= any threshold
    while (lo < hi) {
        uint32_t mid = (lo + hi) >> 1;
        __half_raw r;
        r.x = (unsigned short)mid;
        if (__half2float(__half(r)) >= threshold) hi = mid; else lo = mid + 1;
    }
    return (uint16_t)lo;
}

cudaError_t launch_prepare_weight(const __half *W, int64_t N, int64_t K, int8_t *CB, float *SCB,
                                  cudaStream_t s) {
    int64_t blocks = ceil_div(N, kWarps);
    if (blocks > 148 * 16) blocks = 148 * 16;
    prepare_weight_kernel<<<(unsigned)blocks, kThreads, 0, s>>>(W, N, K, CB, SCB);
    return cudaGetLastError();
}

cudaError_t launch_outlier_flags(const __half *X, int64_t M, int64_t K, uint16_t tbits,
                                 uint32_t *flags, int64_t flag_chunks, cudaStream_t s) {
    dim3 grid((unsigned)ceil_div(K, kColsPerFlagCta), (unsigned)flag_chunks);
    outlier_flags_kernel<<<grid, kThreads, 0, s>>>(X, M, K, tbits, flags, ceil_div(K, 32));
    return cudaGetLastError();
}

cudaError_t launch_quantize(const QuantizeArgs &a, cudaStream_t s) {
    const int64_t kwords = ceil_div(a.K, 32);
    int row_ctas = (int)std::min<int64_t>(ceil_div(a.M, kWarps), 148 * 8);
    int extra = 0;
    if (a.Wo) extra = (int)std::min<int64_t>(ceil_div(a.N, kWarps), 148 * 2);
    else if (a.acc) extra = (int)std::min<int64_t>(ceil_div(a.acc_words, 4096) + 1, 148);
    const size_t smem = (size_t)kwords * 8;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(quantize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    quantize_kernel<<<row_ctas + extra, kThreads, smem, s>>>(a, kwords, row_ctas);
    return cudaGetLastError();
}

}  // namespace int8lt
