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

// rint(x * s) with s = fp32(127 / absmax) and |x| <= absmax. No clamp is
// needed: |x * s| <= 127 * (1 + 2^-23) before rounding, so the fp32 product
// rounds to at most 127.00001 and rint gives at most 127 in magnitude.
__device__ __forceinline__ int32_t quant_code(float x, float s) { return __float2int_rn(__fmul_rn(x, s)); }

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

__device__ __forceinline__ uint32_t pack4(int32_t a, int32_t b, int32_t c, int32_t d) {
    // low bytes of four small integers -> one word (byte 0 = a)
    return __byte_perm(__byte_perm((uint32_t)a, (uint32_t)b, 0x0040), __byte_perm((uint32_t)c, (uint32_t)d, 0x0040),
                       0x5410);
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
            for (int64_t k = lane; k < K; k += 32) cb[k] = (int8_t)quant_code(__half2float(w[k]), s);
        }
        if (lane == 0) SCB[j] = a;
    }
}

// ------------------------------------------------------- phase A: flags ----

// Block (x, y): columns [64x, 64x + 64), row chunk y. Lane l reads the 16-byte
// vector (l & 7) of row (4 * warp + (l >> 3)) + 32 i of the chunk, 8 rows
// in flight per thread. Writes flags[y][2x], flags[y][2x + 1] (no atomics).
constexpr int kFlagUnroll = 8;

__global__ void __launch_bounds__(kThreads)
outlier_flags_kernel(const __half *__restrict__ X, int64_t M, int64_t K, uint32_t tbits,
                     uint32_t *__restrict__ flags, int64_t kwords) {
    __shared__ uint32_t sflags[2];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x < 2) sflags[threadIdx.x] = 0;
    __syncthreads();
    const int64_t c0 = (int64_t)blockIdx.x * kColsPerFlagCta + (lane & 7) * 8;
    const int64_t rows_per = ceil_div(M, gridDim.y);
    const int64_t r1 = min(M, (int64_t)blockIdx.y * rows_per + rows_per);
    const uint32_t t2 = tbits | (tbits << 16);
    // hit[w]: per 16-bit half 0xffff where some |x| >= threshold; half 0 of
    // word w is column 2w of the lane's 8 columns, half 1 is column 2w + 1.
    uint32_t hit[4] = {0u, 0u, 0u, 0u};
    if (c0 < K) {
        const __half *xc = X + c0;
        for (int64_t r = (int64_t)blockIdx.y * rows_per + warp * 4 + (lane >> 3); r < r1;
             r += kFlagUnroll * 32) {
            uint4 v[kFlagUnroll];
#pragma unroll
            for (int u = 0; u < kFlagUnroll; ++u) {
                const int64_t ru = r + u * 32;
                v[u] = ru < r1 ? __ldg(reinterpret_cast<const uint4 *>(xc + ru * K)) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < kFlagUnroll; ++u) {
                hit[0] |= __vcmpgeu2(v[u].x & 0x7fff7fffu, t2);
                hit[1] |= __vcmpgeu2(v[u].y & 0x7fff7fffu, t2);
                hit[2] |= __vcmpgeu2(v[u].z & 0x7fff7fffu, t2);
                hit[3] |= __vcmpgeu2(v[u].w & 0x7fff7fffu, t2);
            }
        }
    }
    // Zero-padded rows compare as |0| >= T, true only for T = 0, where every
    // column is an outlier anyway (and then only real columns are kept).
    uint32_t byte = 0;  // bit j: column c0 + j is an outlier column
#pragma unroll
    for (int w = 0; w < 4; ++w) byte |= ((hit[w] & 1u) << (2 * w)) | (((hit[w] >> 16) & 1u) << (2 * w + 1));
    byte |= __shfl_xor_sync(0xffffffffu, byte, 8);
    byte |= __shfl_xor_sync(0xffffffffu, byte, 16);
    if (lane < 8 && byte) atomicOr(&sflags[lane >> 2], byte << ((lane & 3) * 8));
    __syncthreads();
    if (threadIdx.x < 2) {
        const int64_t word = (int64_t)blockIdx.x * 2 + threadIdx.x;
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

// Outlier mask (bit j = column 8v + j) of the 16-byte vector v.
__device__ __forceinline__ uint32_t vec_mask(const uint32_t *bits, int64_t v) {
    return (bits[(v * 8) >> 5] >> ((v * 8) & 31)) & 0xffu;
}

// Slow paths for the few vectors holding outlier columns, kept out of line
// so the unrolled fast path does not reserve registers for them.
__device__ __noinline__ uint32_t masked_absmax_bits_slow(uint4 x, uint32_t m) {
    const uint16_t *e = reinterpret_cast<const uint16_t *>(&x);
    uint32_t amax = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j)
        if (!((m >> j) & 1u)) amax = max(amax, (uint32_t)(e[j] & 0x7fffu));
    return amax;
}

__device__ __forceinline__ uint32_t masked_absmax_bits(uint4 x, uint32_t m) {
    return m == 0 ? vec_absmax_bits(x) : masked_absmax_bits_slow(x, m);
}

// Codes of vector v (outlier columns -> 0, and their fp16 values -> Xo).
__device__ __noinline__ uint2 quant_masked_slow(uint4 x, uint32_t m, float s, int64_t v, const uint32_t *bits,
                                                const int32_t *prefix, __half *xo) {
    uint2 q = quant_vec8(x, s);
    {
        const __half *e = reinterpret_cast<const __half *>(&x);
        uint32_t keep0 = 0, keep1 = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if ((m >> j) & 1u) {
                if (xo) {
                    const int64_t col = v * 8 + j;
                    const int32_t rank = prefix[col >> 5] + __popc(bits[col >> 5] & ((1u << (col & 31)) - 1u));
                    xo[rank] = e[j];
                }
            } else {
                if (j < 4) keep0 |= 0xffu << (8 * j); else keep1 |= 0xffu << (8 * (j - 4));
            }
        }
        q.x &= keep0;
        q.y &= keep1;
    }
    return q;
}

__device__ __forceinline__ uint2 quant_masked(uint4 x, uint32_t m, float s, int64_t v, const uint32_t *bits,
                                              const int32_t *prefix, __half *xo) {
    return m == 0 ? quant_vec8(x, s) : quant_masked_slow(x, m, s, v, bits, prefix, xo);
}

// Max over the T threads of a row team (T = 32: one warp; T = 128: four
// warps synchronised by a named barrier private to the team).
template <int T>
__device__ __forceinline__ uint32_t team_max(uint32_t v, uint32_t *red, int team) {
    v = warp_max_u32(v);
    if (T == 32) return v;
    const int tw = (threadIdx.x & (T - 1)) >> 5;
    if ((threadIdx.x & 31) == 0) red[team * (T / 32) + tw] = v;
    asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(T) : "memory");
    uint32_t r = red[team * (T / 32)];
#pragma unroll
    for (int i = 1; i < T / 32; ++i) r = max(r, red[team * (T / 32) + i]);
    asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(T) : "memory");  // red reusable
    return r;
}

// One row per team of T threads; the team's row is held in V 16-byte
// registers per thread (V * T * 8 >= K), or re-read when V == 0.
template <int T, int V>
__device__ void quantize_rows_team(const QuantizeArgs &a, const uint32_t *bits, const int32_t *prefix,
                                   int32_t n_out, int row_ctas, uint32_t *red) {
    const int teams = kThreads / T;
    const int team = threadIdx.x / T, tl = threadIdx.x & (T - 1);
    const int64_t nvec = a.K / 8;
    const int32_t n16 = (n_out + 15) & ~15;
    for (int64_t r = (int64_t)blockIdx.x * teams + team; r < a.M; r += (int64_t)row_ctas * teams) {
        const uint4 *x4 = reinterpret_cast<const uint4 *>(a.X + r * a.K);
        uint2 *ca2 = reinterpret_cast<uint2 *>(a.CA + r * a.K);
        __half *xo = a.Xo ? a.Xo + r * a.kcap : nullptr;
        uint32_t amax = 0;
        float sa, s;
        if constexpr (V > 0) {
            uint4 x[V];
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int64_t v = tl + (int64_t)i * T;
                x[i] = v < nvec ? __ldg(x4 + v) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int64_t v = tl + (int64_t)i * T;
                if (v < nvec) amax = max(amax, masked_absmax_bits(x[i], vec_mask(bits, v)));
            }
            amax = team_max<T>(amax, red, team);
            sa = __half2float(__ushort_as_half((unsigned short)amax));
            s = sa > 0.f ? __fdiv_rn(127.f, sa) : 0.f;
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int64_t v = tl + (int64_t)i * T;
                if (v < nvec) ca2[v] = quant_masked(x[i], vec_mask(bits, v), s, v, bits, prefix, xo);
            }
        } else {
            for (int64_t v = tl; v < nvec; v += T) amax = max(amax, masked_absmax_bits(__ldg(x4 + v), vec_mask(bits, v)));
            amax = team_max<T>(amax, red, team);
            sa = __half2float(__ushort_as_half((unsigned short)amax));
            s = sa > 0.f ? __fdiv_rn(127.f, sa) : 0.f;
            for (int64_t v = tl; v < nvec; v += T)
                ca2[v] = quant_masked(__ldg(x4 + v), vec_mask(bits, v), s, v, bits, prefix, xo);
        }
        if (xo)
            for (int32_t t = n_out + tl; t < n16; t += T) xo[t] = __float2half_rn(0.f);
        if (tl == 0) a.SCA[r] = sa;
    }
}

template <int T, int V>
__global__ void __launch_bounds__(kThreads, 2)
quantize_kernel(QuantizeArgs a, int64_t kwords, int row_ctas) {
    extern __shared__ uint32_t smem[];
    __shared__ uint32_t red[kWarps];
    uint32_t *bits = smem;                                         // [kwords]
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
        quantize_rows_team<T, V>(a, bits, prefix, n_out, row_ctas, red);
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

namespace {

template <int T, int V>
cudaError_t launch_quantize_tv(const QuantizeArgs &a, int64_t kwords, int row_ctas, int extra,
                               cudaStream_t s) {
    const size_t smem = (size_t)kwords * 8;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(quantize_kernel<T, V>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    quantize_kernel<T, V><<<row_ctas + extra, kThreads, smem, s>>>(a, kwords, row_ctas);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize(const QuantizeArgs &a, cudaStream_t s) {
    const int64_t kwords = ceil_div(a.K, 32);
    const int64_t nvec = a.K / 8;
    // Row team: one warp per row up to K = 4096 (16 vectors per lane), four
    // warps per row up to K = 16384; longer rows are read twice.
    const int T = nvec <= 128 ? 32 : 128;
    const int teams = kThreads / T;
    int row_ctas = (int)std::min<int64_t>(ceil_div(a.M, teams), 148 * 8);
    int extra = 0;
    if (a.Wo) extra = (int)std::min<int64_t>(ceil_div(a.N, 64), 128);
    else if (a.acc) extra = (int)std::min<int64_t>(ceil_div(a.acc_words, 4096) + 1, 148);
    const int64_t v = ceil_div(nvec, T);
    if (T == 32) return launch_quantize_tv<32, 4>(a, kwords, row_ctas, extra, s);
    if (v <= 4) return launch_quantize_tv<128, 4>(a, kwords, row_ctas, extra, s);
    if (v <= 8) return launch_quantize_tv<128, 8>(a, kwords, row_ctas, extra, s);
    if (v <= 16) return launch_quantize_tv<128, 16>(a, kwords, row_ctas, extra, s);
    return launch_quantize_tv<128, 0>(a, kwords, row_ctas, extra, s);
}

}  // namespace int8lt
