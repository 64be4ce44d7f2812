// Outlier detection and vector-wise absmax quantization (sm_100a).
//
// Method: "LLM.int8() paper summary" (kurtkim.github.io), "8-bit Data Types
// and Quantization" (absmax equation), "Vector-wise Quantization" and "The
// Core of LLM.int8(): Mixed-precision Decomposition"; "Hugging Face LLM.int8()
// integration" (agentlenshq.com), three-step recipe and CB/SCB weights.
//
// Kernels (all HBM-bound streaming passes with 16-byte coalesced loads):
//   prepare_weight_kernel  W [N,K] -> CB, SCB          (one warp per row)
//   quantize_kernel        one cooperative launch: phase A ORs the outlier
//                          columns of every row into a bitmap, a grid
//                          barrier, then phase B writes O, CA, SCA, Xo,
//                          gathers Wo and clears the split-K buffers of the
//                          GEMV
//
// Exactness: |x| >= threshold is decided on the fp16 bit pattern against the
// smallest fp16 pattern whose value reaches the fp32 threshold (the map from
// non-negative fp16 patterns to values is monotonic, so this is the fp32
// comparison). The absmax is a max of fp16 magnitudes (exact). The code is
// rint(x * fp32(127 / absmax)) with __fdiv_rn / __fmul_rn / __float2int_rn:
// one IEEE rounding per step, ties to even, never contracted into an FMA.
#include <algorithm>
#include <mutex>

#include "int8lt_internal.cuh"

namespace int8lt {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// Code of x: rint(fp32(x * s)) with s = fp32(127 / absmax) and |x| <= absmax.
// No clamp is needed: |x * s| <= 127 * (1 + 2^-23) before rounding, so the
// fp32 product is at most 127.00001 and its rint at most 127 in magnitude.
// rint(v) for |v| < 2^22 is taken by adding 1.5 * 2^23 in fp32: the sum lies
// in [2^23, 2^24), where consecutive fp32 values are consecutive integers, so
// IEEE round-to-nearest-even of the addition is rint(v) + 1.5 * 2^23; the low
// byte of the sum's bit pattern is then the low byte of rint(v) (two's
// complement), because 1.5 * 2^23 = 0xC00000 has a zero low byte. Both steps
// are separate _rn operations, so they are never fused into one FMA.
__device__ __forceinline__ uint32_t code_bits(float x, float s) {
    return __float_as_uint(__fadd_rn(__fmul_rn(x, s), 12582912.0f));
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

__device__ __forceinline__ uint32_t pack4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    // low bytes of four words -> one word (byte 0 = a)
    return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Codes of the 8 fp16 values of a 16-byte vector (scalar fp32 multiply and
// add per value, as code_bits()).
__device__ __forceinline__ uint2 quant_vec8(uint4 v, float s) {
    const __half2 *h = reinterpret_cast<const __half2 *>(&v);
    const float2 f0 = __half22float2(h[0]), f1 = __half22float2(h[1]);
    const float2 f2 = __half22float2(h[2]), f3 = __half22float2(h[3]);
    uint2 r;
    r.x = pack4(code_bits(f0.x, s), code_bits(f0.y, s), code_bits(f1.x, s), code_bits(f1.y, s));
    r.y = pack4(code_bits(f2.x, s), code_bits(f2.y, s), code_bits(f3.x, s), code_bits(f3.y, s));
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
            for (int64_t k = lane; k < K; k += 32) cb[k] = (int8_t)(code_bits(__half2float(w[k]), s) & 0xffu);
        }
        if (lane == 0) SCB[j] = a;
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
__device__ __forceinline__ uint32_t vec_mask(const uint32_t *bits, int v) {
    return (bits[v >> 2] >> ((v & 3) * 8)) & 0xffu;
}

// Slow paths for the few vectors holding outlier columns, kept out of line
// so the unrolled fast path does not reserve registers for them.
// Phase A test of one vector of 8 halves: set bit (v*8 + k) of `bits` for
// every element k with |x| >= threshold (t2 = the threshold's binary16 bits,
// twice). A vector with no hit, the usual case, costs four compares.
__device__ __forceinline__ void flag_vec(uint4 x, uint32_t t2, int v, uint32_t *bits) {
    const uint32_t h0 = __vcmpgeu2(x.x & 0x7fff7fffu, t2), h1 = __vcmpgeu2(x.y & 0x7fff7fffu, t2);
    const uint32_t h2 = __vcmpgeu2(x.z & 0x7fff7fffu, t2), h3 = __vcmpgeu2(x.w & 0x7fff7fffu, t2);
    if ((h0 | h1 | h2 | h3) == 0u) return;
    const uint32_t b = (h0 & 1u) | ((h0 >> 15) & 2u) | ((h1 & 1u) << 2) | ((h1 >> 13) & 8u) | ((h2 & 1u) << 4) |
                       ((h2 >> 11) & 32u) | ((h3 & 1u) << 6) | ((h3 >> 9) & 128u);
    atomicOr(&bits[v >> 2], b << ((v & 3) * 8));
}

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
__device__ __noinline__ uint2 quant_masked_slow(uint4 x, uint32_t m, float s, int v, const uint32_t *bits,
                                                const int32_t *prefix, __half *xo) {
    uint2 q = quant_vec8(x, s);
    {
        const __half *e = reinterpret_cast<const __half *>(&x);
        uint32_t keep0 = 0, keep1 = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if ((m >> j) & 1u) {
                if (xo) {
                    const int col = v * 8 + j;
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

__device__ __forceinline__ uint2 quant_masked(uint4 x, uint32_t m, float s, int v, const uint32_t *bits,
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
// Phase B of one row held in registers (V > 0): masked absmax over the team,
// codes, scale and outlier activations. Every thread of the team calls it.
template <int T, int V>
__device__ __forceinline__ void quantize_row_regs(const QuantizeArgs &a, const uint32_t *bits, const int32_t *prefix,
                                                  int32_t n_out, const uint4 (&x)[V], int64_t r, bool valid,
                                                  uint32_t *red, int team, int tl) {
    const int nvec = (int)(a.K / 8);
    const int32_t n16 = (n_out + 15) & ~15;
    uint32_t m[V];
    uint32_t amax = 0;
#pragma unroll
    for (int i = 0; i < V; ++i) {
        const int v = tl + i * T;
        const bool in = valid && v < nvec;
        m[i] = in ? vec_mask(bits, v) : 0u;
        if (in) amax = max(amax, masked_absmax_bits(x[i], m[i]));
    }
    amax = team_max<T>(amax, red, team);
    if (!valid) return;
    const float sa = __half2float(__ushort_as_half((unsigned short)amax));
    const float s = sa > 0.f ? __fdiv_rn(127.f, sa) : 0.f;
    uint2 *ca2 = reinterpret_cast<uint2 *>(a.CA + r * a.K);
    __half *xo = a.Xo ? a.Xo + r * a.kcap : nullptr;
#pragma unroll
    for (int i = 0; i < V; ++i) {
        const int v = tl + i * T;
        if (v < nvec) ca2[v] = quant_masked(x[i], m[i], s, v, bits, prefix, xo);
    }
    if (xo)
        for (int32_t t = n_out + tl; t < n16; t += T) xo[t] = __float2half_rn(0.f);
    if (tl == 0) a.SCA[r] = sa;
}

// Load the V vectors of row r a team thread owns (zeros past the row end).
template <int T, int V>
__device__ __forceinline__ void load_row(const QuantizeArgs &a, int64_t r, int tl, uint4 (&x)[V]) {
    const int nvec = (int)(a.K / 8);
    const uint4 *x4 = reinterpret_cast<const uint4 *>(a.X + r * a.K);
#pragma unroll
    for (int i = 0; i < V; ++i) {
        const int v = tl + i * T;
        x[i] = v < nvec ? __ldg(x4 + v) : make_uint4(0, 0, 0, 0);
    }
}

// Phase B for the team's rows, re-read from memory (rows are not kept).
template <int T, int V>
__device__ void quantize_rows_team(const QuantizeArgs &a, const uint32_t *bits, const int32_t *prefix,
                                   int32_t n_out, int row_ctas, uint32_t *red) {
    const int teams = kThreads / T;
    const int team = threadIdx.x / T, tl = threadIdx.x & (T - 1);
    for (int64_t r = (int64_t)blockIdx.x * teams + team; r < a.M; r += (int64_t)row_ctas * teams) {
        if constexpr (V > 0) {
            uint4 x[V];
            load_row<T, V>(a, r, tl, x);
            quantize_row_regs<T, V>(a, bits, prefix, n_out, x, r, true, red, team, tl);
        } else {
            const int nvec = (int)(a.K / 8);
            const int32_t n16 = (n_out + 15) & ~15;
            const uint4 *x4 = reinterpret_cast<const uint4 *>(a.X + r * a.K);
            uint32_t amax = 0;
            for (int v = tl; v < nvec; v += T) amax = max(amax, masked_absmax_bits(__ldg(x4 + v), vec_mask(bits, v)));
            amax = team_max<T>(amax, red, team);
            const float sa = __half2float(__ushort_as_half((unsigned short)amax));
            const float s = sa > 0.f ? __fdiv_rn(127.f, sa) : 0.f;
            uint2 *ca2 = reinterpret_cast<uint2 *>(a.CA + r * a.K);
            __half *xo = a.Xo ? a.Xo + r * a.kcap : nullptr;
            for (int v = tl; v < nvec; v += T)
                ca2[v] = quant_masked(__ldg(x4 + v), vec_mask(bits, v), s, v, bits, prefix, xo);
            if (xo)
                for (int32_t t = n_out + tl; t < n16; t += T) xo[t] = __float2half_rn(0.f);
            if (tl == 0) a.SCA[r] = sa;
        }
    }
}

// Phase A for one team's rows: OR the rows' outlier bits into the CTA bitmap.
template <int T, int V>
__device__ void flag_rows_team(const QuantizeArgs &a, uint32_t *bits, int teams_total) {
    const int teams = kThreads / T;
    const int team = threadIdx.x / T, tl = threadIdx.x & (T - 1);
    const int nvec = (int)(a.K / 8);
    const uint32_t t2 = (uint32_t)a.tbits | ((uint32_t)a.tbits << 16);
    for (int64_t r = (int64_t)blockIdx.x * teams + team; r < a.M; r += teams_total) {
        if constexpr (V > 0) {
            uint4 x[V];
            load_row<T, V>(a, r, tl, x);
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int v = tl + i * T;
                if (v < nvec) flag_vec(x[i], t2, v, bits);
            }
        } else {
            const uint4 *x4 = reinterpret_cast<const uint4 *>(a.X + r * a.K);
            for (int v = tl; v < nvec; v += T) flag_vec(__ldg(x4 + v), t2, v, bits);
        }
    }
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Grid-wide barrier of the cooperative launch. The arrival count only grows:
// this launch's CTAs are all in once it reaches base + gridDim.x, which the
// waiters see directly in the count. The last CTA in publishes the next
// launch's base and generation (no CTA of this launch reads them any more;
// the next launch, behind this one in stream order, does). Every wait is
// bounded; after a timeout the count is off and the workspace header must be
// initialised again. Returns false (and records a timeout) if it ran out.
__device__ bool grid_barrier(WsHeader *h, uint32_t gen, uint32_t base) {
    __shared__ uint32_t s_ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t ok = 1;
        const uint32_t target = base + gridDim.x;
        __threadfence();
        const uint32_t old = atomicAdd(&h->bar_count, 1u);
        if (old == target - 1u) {
            *reinterpret_cast<volatile uint32_t *>(&h->qbase) = target;
            atomicExch(&h->qgen, gen + 1u);
        } else {
            const uint64_t t0 = globaltimer_ns();
            while ((int32_t)(ld_acquire_u32(&h->bar_count) - target) < 0) {
                if (globaltimer_ns() - t0 > kWaitLimitNs) {
                    ok = 0;
                    record_timeout(&h->status);
                    break;
                }
            }
        }
        __threadfence();
        s_ok = ok;
    }
    __syncthreads();
    return s_ok != 0;
}

// kOneRound: every row has its own team (M <= teams in the grid), which
// keeps its row in registers from phase A to phase B.
template <int T, int V, bool kOneRound>
__global__ void __launch_bounds__(kThreads, 2)
quantize_kernel(QuantizeArgs a, int64_t kwords) {
    extern __shared__ uint32_t smem[];
    __shared__ uint32_t red[kWarps];
    __shared__ uint32_t s_gen, s_base;
    uint32_t *bits = smem;                                         // [kwords]
    int32_t *prefix = reinterpret_cast<int32_t *>(smem + kwords);  // [kwords]
    const int teams_total = gridDim.x * (kThreads / T);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    // This launch's bitmap is bitmaps[gen & 1]; the previous launch zeroed it.
    if (threadIdx.x == 0) {
        s_gen = *reinterpret_cast<volatile uint32_t *>(&a.hdr->qgen);
        s_base = *reinterpret_cast<volatile uint32_t *>(&a.hdr->qbase);
    }
    for (int64_t w = threadIdx.x; w < kwords; w += kThreads) bits[w] = 0;
    __syncthreads();
    const uint32_t gen = s_gen;
    uint32_t *cur = a.bitmaps + (gen & 1u) * kMaxKwords;
    uint32_t *nxt = a.bitmaps + ((gen + 1u) & 1u) * kMaxKwords;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < kMaxKwords; i += (int64_t)gridDim.x * kThreads)
        nxt[i] = 0;

    constexpr int kTeams = kThreads / T;
    const int team = threadIdx.x / T, tl = threadIdx.x & (T - 1);
    const int64_t my_row = (int64_t)blockIdx.x * kTeams + team;
    uint4 xr[kOneRound ? V : 1];

    // Phase A: O = { h : some |X[i,h]| >= threshold } over every row.
    if constexpr (kOneRound) {
        if (my_row < a.M) {
            const int nvec = (int)(a.K / 8);
            const uint32_t t2 = (uint32_t)a.tbits | ((uint32_t)a.tbits << 16);
            load_row<T, V>(a, my_row, tl, xr);
#pragma unroll
            for (int i = 0; i < V; ++i) {
                const int v = tl + i * T;
                if (v < nvec) flag_vec(xr[i], t2, v, bits);
            }
        }
    } else {
        flag_rows_team<T, V>(a, bits, teams_total);
    }
    __syncthreads();
    for (int64_t w = threadIdx.x; w < kwords; w += kThreads)
        if (bits[w]) atomicOr(&cur[w], bits[w]);
    if (!grid_barrier(a.hdr, gen, s_base)) return;  // every CTA waits in the same barrier

    // Phase B: codes, scales, outlier activations; outlier-weight gather.
    for (int64_t w = threadIdx.x; w < kwords; w += kThreads) {
        uint32_t v = __ldcg(&cur[w]);
        if (w == kwords - 1 && (a.K & 31)) v &= (1u << (a.K & 31)) - 1u;
        bits[w] = v;
    }
    __syncthreads();
    const int32_t n_out = build_prefix(bits, prefix, kwords);
    const int32_t n16 = (n_out + 15) & ~15;
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
    if constexpr (kOneRound)
        quantize_row_regs<T, V>(a, bits, prefix, n_out, xr, my_row, my_row < a.M, red, team, tl);
    else
        quantize_rows_team<T, V>(a, bits, prefix, n_out, gridDim.x, red);
    if (a.Wo) {
        // Wo[j, t] = W[j, col_t]: half-warps over output channels, a lane per
        // outlier rank t, four channels' loads in flight before any store.
        const int hl = lane & 15;
        const int64_t hw = ((int64_t)blockIdx.x * kWarps + warp) * 2 + (lane >> 4);
        const int64_t nhw = (int64_t)gridDim.x * kWarps * 2;
        for (int32_t t0 = 0; t0 < n16; t0 += 16) {
            const int32_t t = t0 + hl;
            const bool real = t < n_out;
            const int64_t col = real ? outlier_column(bits, prefix, kwords, t) : 0;
            for (int64_t j0 = hw; j0 < a.N; j0 += 4 * nhw) {
                __half val[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int64_t j = j0 + u * nhw;
                    val[u] = __float2half_rn(0.f);
                    if (real && j < a.N) {
                        if (a.W_outlier) {
                            val[u] = a.W_outlier[j * a.K + col];
                        } else {
                            const float p = __fmul_rn((float)a.CB[j * a.K + col], a.SCB[j]);
                            val[u] = __float2half_rn(__fdiv_rn(p, 127.f));
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int64_t j = j0 + u * nhw;
                    if (j < a.N) a.Wo[j * a.kcap + t] = val[u];
                }
            }
        }
    }
    const int64_t tid = (int64_t)blockIdx.x * kThreads + threadIdx.x, nth = (int64_t)gridDim.x * kThreads;
    if (a.acc)
        for (int64_t i = tid; i < a.acc_words; i += nth) a.acc[i] = 0;
    if (a.cnt)
        for (int64_t i = tid; i < a.cnt_words; i += nth) a.cnt[i] = 0;
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

namespace {

// Resident CTAs of one kernel instance on the current device (for the
// cooperative grid size), computed once per device.
template <int T, int V, bool R>
cudaError_t resident_ctas(size_t smem, int *out) {
    static std::once_flag once[64];
    static int count[64];
    static cudaError_t err[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    dev &= 63;
    std::call_once(once[dev], [&] {
        int per_sm = 0, sms = 0;
        err[dev] = cudaFuncSetAttribute(quantize_kernel<T, V, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)(2 * kMaxKwords * 4));
        if (err[dev] == cudaSuccess)
            err[dev] = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quantize_kernel<T, V, R>, kThreads,
                                                                     2 * kMaxKwords * 4);
        if (err[dev] == cudaSuccess) err[dev] = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        count[dev] = per_sm * sms;
    });
    (void)smem;
    *out = count[dev];
    return err[dev];
}

template <int T, int V, bool R>
cudaError_t launch_quantize_tvr(const QuantizeArgs &a, int64_t kwords, int grid, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)kwords * 8;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, quantize_kernel<T, V, R>, a, kwords);
}

template <int T, int V>
cudaError_t launch_quantize_tv(const QuantizeArgs &a, int64_t kwords, cudaStream_t s) {
    const size_t smem = (size_t)kwords * 8;
    int max_ctas = 0;
    if (cudaError_t e = resident_ctas<T, V, false>(smem, &max_ctas)) return e;
    if (max_ctas <= 0) return cudaErrorInvalidConfiguration;
    const int teams = kThreads / T;
    // Enough teams for every row where possible; the grid barrier needs every
    // CTA resident at once, which the cooperative launch guarantees.
    int64_t want = ceil_div(a.M, teams);
    if (a.Wo) want = std::max<int64_t>(want, std::min<int64_t>(ceil_div(a.N, kWarps), 148));
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(want, max_ctas));
    if constexpr (V > 0) {
        // One round (each row its own team) needs a grid that covers every row.
        int max_r = 0;
        if (cudaError_t e = resident_ctas<T, V, true>(smem, &max_r)) return e;
        const int64_t need = ceil_div(a.M, teams);
        if (need <= max_r)
            return launch_quantize_tvr<T, V, true>(a, kwords, (int)std::max<int64_t>(need, grid > max_r ? max_r : grid),
                                                   s);
    }
    return launch_quantize_tvr<T, V, false>(a, kwords, grid, s);
}

}  // namespace

cudaError_t launch_quantize(const QuantizeArgs &a, cudaStream_t s) {
    const int64_t kwords = ceil_div(a.K, 32);
    const int64_t nvec = a.K / 8;
    // Row team: one warp per row up to K = 4096 (up to 16 loads in flight per
    // lane, and every row of a 2048-token batch in flight at once), four warps
    // per row up to K = 16384 (the row stays in registers); longer rows are
    // read twice.
    const int T = nvec <= 32 * 16 ? 32 : 128;
    const int64_t v = ceil_div(nvec, T);
    if (T == 32) {
        if (v <= 4) return launch_quantize_tv<32, 4>(a, kwords, s);
        if (v <= 8) return launch_quantize_tv<32, 8>(a, kwords, s);
        return launch_quantize_tv<32, 16>(a, kwords, s);
    }
    if (v <= 8) return launch_quantize_tv<128, 8>(a, kwords, s);
    if (v <= 16) return launch_quantize_tv<128, 16>(a, kwords, s);
    return launch_quantize_tv<128, 0>(a, kwords, s);
}

}  // namespace int8lt
