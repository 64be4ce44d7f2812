// Outlier detection and vector-wise absmax quantization (sm_100a).
//
// Method: "LLM.int8() paper summary" (kurtkim.github.io), "8-bit Data Types
// and Quantization" (absmax equation), "Vector-wise Quantization" and "The
// Core of LLM.int8(): Mixed-precision Decomposition"; "Hugging Face LLM.int8()
// integration" (agentlenshq.com), three-step recipe and CB/SCB weights.
//
// Kernels (the first four are HBM-bound streaming passes):
//   prepare_weight_kernel  W [N,K] -> CB, SCB          (one warp per row)
//   quantize_kernel        one cooperative launch: the CTA's rows of X are
//                          staged in shared memory; phase A ORs the outlier
//                          columns of every row into a bitmap, a grid
//                          barrier, then phase B writes O, CA, SCA, Xo from
//                          the staged rows and gathers Wo
//   quantize_stream_kernel prefill rows of 8192..16384 columns: X streamed
//                          once, each row quantized with its own outliers
//                          masked before the barrier and finished after it
//   quantize_decode_kernel decode batches of up to 8 rows: one cluster owns
//                          column slices of every row and exchanges the row
//                          maxima and outlier counts through distributed
//                          shared memory; no grid-wide step
//   barrier_timeout_kernel a deliberately short-counted grid barrier that runs
//                          out (failure-detection test of the bounded wait)
//
// Exactness: |x| >= threshold is decided on the fp16 bit pattern against the
// smallest fp16 pattern whose value reaches the fp32 threshold (the map from
// non-negative fp16 patterns to values is monotonic, so this is the fp32
// comparison). The absmax is a max of fp16 magnitudes (exact). The code is
// rint(x * fp32(127 / absmax)) with __fdiv_rn / __fmul_rn and a rounding
// add: one IEEE rounding per step, ties to even, never contracted into an FMA.
#include <algorithm>
#include <mutex>

#include "int8lt_internal.cuh"

namespace int8lt {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kBatch = 16;  // 16-byte loads in flight per thread in phase A
// CB up to this size is pulled into L2 for the GEMM during the quantize pass.
constexpr int64_t kPrefetchMaxBytes = 48ll << 20;

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
    const int64_t KB = wblocks_k(K), Kp = KB * kWBlockCols;
    // Rows past N inside the last row block are written as zero codes.
    for (int64_t j = warp; j < round_up(N, kWBlockRows); j += nwarps) {
        int64_t kz = 0;  // first column written as zero padding
        if (j < N) {
            const __half *w = W + j * K;
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
                for (int64_t v = lane; v < K / 8; v += 32)
                    *reinterpret_cast<uint2 *>(CB + cb_offset(j, v * 8, KB)) = quant_vec8(__ldg(w4 + v), s);
            } else {
                for (int64_t k = lane; k < K; k += 32)
                    CB[cb_offset(j, k, KB)] = (int8_t)(code_bits(__half2float(w[k]), s) & 0xffu);
            }
            if (lane == 0) SCB[j] = a;
            kz = K;
        }
        for (int64_t k = kz + lane; k < Kp; k += 32) CB[cb_offset(j, k, KB)] = 0;
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

// Bit k set for the elements k of the vector whose magnitude bits equal m.
__device__ __forceinline__ uint32_t elem_eq_mask(uint4 x, uint32_t m) {
    const uint32_t w[4] = {x.x & 0x7fff7fffu, x.y & 0x7fff7fffu, x.z & 0x7fff7fffu, x.w & 0x7fff7fffu};
    uint32_t b = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        b |= ((w[i] & 0xffffu) == m ? 1u : 0u) << (2 * i);
        b |= ((w[i] >> 16) == m ? 1u : 0u) << (2 * i + 1);
    }
    return b;
}

// The vector with its outlier elements (bits of m) replaced by +0: their
// code is then 0 and they do not count in the absmax.
__device__ __forceinline__ uint4 clear_masked(uint4 x, uint32_t m) {
    uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t lo = ((m >> (2 * j)) & 1u) ? 0u : 0x0000ffffu;
        const uint32_t hi = ((m >> (2 * j + 1)) & 1u) ? 0u : 0xffff0000u;
        w[j] &= lo | hi;
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Xo[rank of column] = x for the outlier elements (bits of m) of vector v.
// `cap` is the row's capacity in Xo; `st` the status word of a checking build.
__device__ __forceinline__ void store_outliers(uint4 x, uint32_t m, int v, const uint32_t *bits,
                                               const int32_t *prefix, __half *xo, int64_t cap, uint32_t *st) {
    while (m) {
        const int j = __ffs(m) - 1;
        m &= m - 1;
        const uint32_t w = j < 4 ? (j < 2 ? x.x : x.y) : (j < 6 ? x.z : x.w);
        const unsigned short h = (unsigned short)((j & 1) ? (w >> 16) : (w & 0xffffu));
        const int col = v * 8 + j;
        const int64_t rank = prefix[col >> 5] + __popc(bits[col >> 5] & ((1u << (col & 31)) - 1u));
        if (IN_BOUNDS(rank >= 0 && rank < cap, st)) xo[rank] = __ushort_as_half(h);
    }
}

// One warp per row. `row` points at the row's nvec 16-byte vectors, in
// shared memory (kSmem) or in X. Loops are rolled (unroll 4): the kernel's
// code stays small enough for the instruction caches.
template <bool kSmem>
__device__ __forceinline__ uint4 ld_vec(const uint4 *p) {
    if constexpr (kSmem) return *p;
    else return __ldg(p);
}

// Phase B of row r: masked absmax, codes, scale and outlier activations.
// Vectors holding outlier columns (a handful per row) take a short branch.
template <bool kSmem>
__device__ __forceinline__ void quantize_row(const QuantizeArgs &a, const uint4 *row, int64_t r, const uint32_t *bits,
                                             const int32_t *prefix, int32_t n_out, int lane) {
    const int nvec = (int)(a.K / 8);
    uint32_t amax = 0;
#pragma unroll 4
    for (int v = lane; v < nvec; v += 32) {
        uint4 x = ld_vec<kSmem>(row + v);
        const uint32_t m = vec_mask(bits, v);
        if (m) x = clear_masked(x, m);
        amax = max(amax, vec_absmax_bits(x));
    }
    amax = warp_max_u32(amax);
    const float sa = __half2float(__ushort_as_half((unsigned short)amax));
    const float s = sa > 0.f ? __fdiv_rn(127.f, sa) : 0.f;
    uint2 *ca2 = reinterpret_cast<uint2 *>(a.CA + r * a.K);
    __half *xo = a.Xo ? a.Xo + r * a.kcap : nullptr;
#pragma unroll 4
    for (int v = lane; v < nvec; v += 32) {
        uint4 x = ld_vec<kSmem>(row + v);
        const uint32_t m = vec_mask(bits, v);
        if (m) {
            if (xo) store_outliers(x, m, v, bits, prefix, xo, a.kcap, &a.hdr->status);
            x = clear_masked(x, m);
        }
        ca2[v] = quant_vec8(x, s);
    }
    if (xo) {
        const int32_t n16 = (n_out + 15) & ~15;
        for (int32_t t = n_out + lane; t < n16; t += 32)
            if (IN_BOUNDS(t < a.kcap, &a.hdr->status)) xo[t] = __float2half_rn(0.f);
    }
    if (lane == 0) a.SCA[r] = sa;
}

// Phase B of a staged row whose outlier elements are already zero.
__device__ __forceinline__ void quantize_row_plain(const QuantizeArgs &a, const uint4 *row, int64_t r, int lane) {
    const int nvec = (int)(a.K / 8);
    uint32_t amax = 0;
#pragma unroll 4
    for (int v = lane; v < nvec; v += 32) amax = max(amax, vec_absmax_bits(row[v]));
    amax = warp_max_u32(amax);
    const float sa = __half2float(__ushort_as_half((unsigned short)amax));
    const float s = sa > 0.f ? __fdiv_rn(127.f, sa) : 0.f;
    uint2 *ca2 = reinterpret_cast<uint2 *>(a.CA + r * a.K);
#pragma unroll 4
    for (int v = lane; v < nvec; v += 32) ca2[v] = quant_vec8(row[v], s);
    if (lane == 0) a.SCA[r] = sa;
}

// Phase B of a long staged row (outlier elements already zero) by the whole
// CTA; every thread calls it. s_red holds one maximum per warp.
__device__ __forceinline__ void quantize_row_cta(const QuantizeArgs &a, const uint4 *row, int64_t r, uint32_t *s_red,
                                                 int lane, int warp) {
    const int nvec = (int)(a.K / 8);
    uint32_t m = 0;
#pragma unroll 4
    for (int v = threadIdx.x; v < nvec; v += kThreads) m = max(m, vec_absmax_bits(row[v]));
    m = warp_max_u32(m);
    if (lane == 0) s_red[warp] = m;
    __syncthreads();
    uint32_t amax = s_red[0];
#pragma unroll
    for (int i = 1; i < kWarps; ++i) amax = max(amax, s_red[i]);
    const float sa = __half2float(__ushort_as_half((unsigned short)amax));
    const float s = sa > 0.f ? __fdiv_rn(127.f, sa) : 0.f;
    uint2 *ca2 = reinterpret_cast<uint2 *>(a.CA + r * a.K);
#pragma unroll 4
    for (int v = threadIdx.x; v < nvec; v += kThreads) ca2[v] = quant_vec8(row[v], s);
    if (threadIdx.x == 0) a.SCA[r] = sa;
    __syncthreads();  // s_red is free again
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Grid-wide barrier of the cooperative launch. The arrival count only grows:
// this launch's `ctas` CTAs (its grid) are all in once it reaches base +
// ctas, which the waiters see directly in the count. The last CTA in
// publishes the next launch's base and generation (no CTA of this launch
// reads them any more; the next launch, behind this one in stream order,
// does). Every wait is bounded by limit_ns; after a timeout the count is off
// and the workspace header must be initialised again. Returns false (and
// records a timeout) if it ran out.
__device__ bool grid_barrier(WsHeader *h, uint32_t gen, uint32_t base, uint32_t ctas,
                             uint64_t limit_ns = kWaitLimitNs) {
    __shared__ uint32_t s_ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t ok = 1;
        const uint32_t target = base + ctas;
        __threadfence();
        const uint32_t old = atomicAdd(&h->bar_count, 1u);
        if (old == target - 1u) {
            *reinterpret_cast<volatile uint32_t *>(&h->qbase) = target;
            atomicExch(&h->qgen, gen + 1u);
        } else {
            const uint64_t t0 = globaltimer_ns();
            while ((int32_t)(ld_acquire_u32(&h->bar_count) - target) < 0) {
                if (globaltimer_ns() - t0 > limit_ns) {
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

// Phase A walks the CTA's rows in rounds of R rows (rows of a round are
// contiguous in X): every thread keeps 16 16-byte loads in flight, tests
// them and, in the last round, also keeps them in shared memory. Phase B
// quantizes the last round from shared memory, then brings each earlier
// round back into shared memory (from L2 when X fits) and does the same; with
// a single round X is read from HBM exactly once. R = 0 (rows too long to
// keep): phase B reads every row from X, a warp per row.
__global__ void __launch_bounds__(kThreads, 2)
quantize_kernel(QuantizeArgs a, int64_t kwords, int R, int rounds) {
    extern __shared__ __align__(128) uint32_t smem[];
    __shared__ uint32_t s_gen, s_base, s_red[kWarps];
    uint32_t *bits = smem;                                         // [kwords]
    int32_t *prefix = reinterpret_cast<int32_t *>(smem + kwords);  // [kwords]
    uint4 *rows = reinterpret_cast<uint4 *>(smem + ((2 * kwords + 31) & ~int64_t(31)));  // [R][nvec]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nvec = (int)(a.K / 8);
    const int rows_per_round = R > 0 ? R : kWarps;
    const bool long_rows = nvec >= 4 * kThreads;  // K >= 8192: a CTA per staged row
    const uint32_t t2 = (uint32_t)a.tbits | ((uint32_t)a.tbits << 16);
    const uint4 *X4 = reinterpret_cast<const uint4 *>(a.X);
    // The GEMM behind this pass may start its prologue on SMs this grid frees;
    // it waits for the whole pass before it reads anything.
    grid_dep_launch();

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
    // A single CTA sees every row itself: its shared bitmap is the whole
    // outlier set, and the global bitmaps, the barrier and the launch counter
    // are left as they are (bitmaps[gen & 1] stays zero for the next launch).
    const bool alone = gridDim.x == 1;
    if (!alone)
        for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < kMaxKwords;
             i += (int64_t)gridDim.x * kThreads)
            nxt[i] = 0;

    // Phase A: O = { h : some |X[i,h]| >= threshold } over every row.
    for (int rd = 0; rd < rounds; ++rd) {
        const int64_t r0 = ((int64_t)rd * gridDim.x + blockIdx.x) * rows_per_round;
        const int64_t left = a.M - r0;
        const int nr = left <= 0 ? 0 : (left < rows_per_round ? (int)left : rows_per_round);
        const bool keep = R > 0 && rd == rounds - 1;
        const int64_t total = (int64_t)nr * nvec;          // this round's vectors
        const uint4 *src = X4 + r0 * nvec;
        int v = threadIdx.x % nvec;                          // column vector of `flat`
        for (int64_t flat = threadIdx.x; flat < total; flat += kBatch * kThreads) {
            uint4 x[kBatch];
            int vs[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int64_t f = flat + u * kThreads;
                vs[u] = v;
                x[u] = f < total ? __ldg(src + f) : make_uint4(0, 0, 0, 0);
                v += kThreads;
                if (v >= nvec) v = nvec >= kThreads ? v - nvec : v % nvec;
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int64_t f = flat + u * kThreads;
                if (f < total) {
                    flag_vec(x[u], t2, vs[u], bits);
                    if (keep) rows[f] = x[u];
                }
            }
        }
    }
    __syncthreads();
    // The prefill GEMM behind this pass streams CB; while this grid waits at
    // its barrier and quantizes, HBM is mostly idle, so start pulling CB into
    // L2 now (each CTA a slice; only when CB fits L2 comfortably).
    if (a.Wo && a.CB && a.N * a.K <= kPrefetchMaxBytes && threadIdx.x < 32) {
        const int64_t bytes = a.N * a.K;  // a multiple of 128: N % 8 == 0, K % 16 == 0
        const int64_t slice = round_up(ceil_div(bytes, gridDim.x), 4096);
        const int64_t b0 = (int64_t)blockIdx.x * slice, b1 = min(bytes, b0 + slice);
        for (int64_t off = b0 + (int64_t)threadIdx.x * 4096; off < b1; off += 32 * 4096) {
            const uint32_t n = (uint32_t)(b1 - off < 4096 ? b1 - off : 4096);
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.CB + off), "r"(n) : "memory");
        }
    }
    // Decode path: zero the GEMV's partial sums and k-block counters here,
    // before the barrier, where the stores overlap the wait (nothing in this
    // pass reads them, and the GEMV reads them only after the whole pass).
    {
        const int64_t tid = (int64_t)blockIdx.x * kThreads + threadIdx.x, nth = (int64_t)gridDim.x * kThreads;
        if (a.acc)
            for (int64_t i = tid; i < a.acc_words / 4; i += nth) reinterpret_cast<int4 *>(a.acc)[i] = make_int4(0, 0, 0, 0);
        if (a.cnt)
            for (int64_t i = tid; i < a.cnt_words / 4; i += nth) reinterpret_cast<uint4 *>(a.cnt)[i] = make_uint4(0, 0, 0, 0);
    }
    if (!alone) {
        for (int64_t w = threadIdx.x; w < kwords; w += kThreads)
            if (bits[w]) atomicOr(&cur[w], bits[w]);
        if (!grid_barrier(a.hdr, gen, s_base, gridDim.x)) return;  // every CTA waits in the same barrier
    }

    // Phase B: codes, scales, outlier activations; outlier-weight gather.
    for (int64_t w = threadIdx.x; w < kwords; w += kThreads) {
        uint32_t v = alone ? bits[w] : __ldcg(&cur[w]);
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
                    if (IN_BOUNDS(r >= 0 && r < a.K, &a.hdr->status)) a.outlier_idx[r] = (int32_t)(w * 32 + __ffs(v) - 1);
                    ++r;
                    v &= v - 1;
                }
            }
        }
    }
    // Outlier-weight gather Wo[j, t] = W[j, col_t] (or CB[j, col_t] * SCB[j]
    // / 127): half-warps over output channels, a lane per outlier rank t,
    // four channels per pass. The first pass's loads are issued before phase
    // B and stored after it, so their latency hides behind the quantization.
    const int hl = lane & 15;
    const int64_t hw = ((int64_t)blockIdx.x * kWarps + warp) * 2 + (lane >> 4);
    const int64_t nhw = (int64_t)gridDim.x * kWarps * 2;
    __half gv[4];
    auto gather_load = [&](int32_t t0, int64_t j0) {
        const int32_t t = t0 + hl;
        const bool real = t < n_out;
        const int64_t col = real ? outlier_column(bits, prefix, kwords, t) : 0;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int64_t j = j0 + u * nhw;
            gv[u] = __float2half_rn(0.f);
            if (real && j < a.N && IN_BOUNDS(col >= 0 && col < a.K, &a.hdr->status)) {
                if (a.W_outlier) {
                    gv[u] = a.W_outlier[j * a.K + col];
                } else {
                    const float p = __fmul_rn((float)a.CB[cb_offset(j, col, wblocks_k(a.K))], a.SCB[j]);
                    gv[u] = __float2half_rn(__fdiv_rn(p, 127.f));
                }
            }
        }
    };
    auto gather_store = [&](int32_t t0, int64_t j0) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int64_t j = j0 + u * nhw;
            if (j < a.N && IN_BOUNDS(t0 + hl < a.kcap, &a.hdr->status)) a.Wo[j * a.kcap + t0 + hl] = gv[u];
        }
    };
    const bool gather = a.Wo && n16 > 0;
    if (gather) gather_load(0, hw);

    for (int rd = rounds - 1; rd >= 0; --rd) {
        const int64_t r0 = ((int64_t)rd * gridDim.x + blockIdx.x) * rows_per_round;
        const int64_t left = a.M - r0;
        const int nr = left <= 0 ? 0 : (left < rows_per_round ? (int)left : rows_per_round);
        if (R == 0) {
            for (int r = warp; r < nr; r += kWarps)
                quantize_row<false>(a, X4 + (r0 + r) * nvec, r0 + r, bits, prefix, n_out, lane);
            continue;
        }
        if (rd != rounds - 1) {
            // An earlier round: bring its rows back into shared memory.
            __syncthreads();  // the previous round's rows are done with
            const int64_t total = (int64_t)nr * nvec;
            const uint4 *src = X4 + r0 * nvec;
            for (int64_t flat = threadIdx.x; flat < total; flat += kBatch * kThreads) {
                uint4 x[kBatch];
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int64_t f = flat + u * kThreads;
                    x[u] = f < total ? __ldg(src + f) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int64_t f = flat + u * kThreads;
                    if (f < total) rows[f] = x[u];
                }
            }
            __syncthreads();
        }
        // Staged rows: copy their outlier elements to Xo and zero them in
        // place (a warp per row), then quantize them without masks: a warp
        // per row, or the whole CTA per row when rows are long.
        for (int r = warp; r < nr; r += kWarps) {
            __half *rh = reinterpret_cast<__half *>(rows + (size_t)r * nvec);
            __half *xo = a.Xo ? a.Xo + (r0 + r) * a.kcap : nullptr;
            for (int32_t t = lane; t < n16; t += 32) {
                __half val = __float2half_rn(0.f);
                if (t < n_out) {
                    const int64_t col = outlier_column(bits, prefix, kwords, t);
                    val = rh[col];
                    rh[col] = __ushort_as_half((unsigned short)0);
                }
                if (xo && IN_BOUNDS(t < a.kcap, &a.hdr->status)) xo[t] = val;
            }
            __syncwarp();
            if (!long_rows) quantize_row_plain(a, rows + (size_t)r * nvec, r0 + r, lane);
        }
        if (long_rows) {
            __syncthreads();
            for (int r = 0; r < nr; ++r) quantize_row_cta(a, rows + (size_t)r * nvec, r0 + r, s_red, lane, warp);
        }
    }
    if (gather) {
        gather_store(0, hw);
        for (int32_t t0 = 0; t0 < n16; t0 += 16)
            for (int64_t j0 = hw + (t0 == 0 ? 4 * nhw : 0); j0 < a.N; j0 += 4 * nhw) {
                gather_load(t0, j0);
                gather_store(t0, j0);
            }
    }
}

// ------------------------------------------------ streaming, row per CTA --
//
// For batches with long rows (see launch_quantize) X is read from HBM once:
// each CTA streams rows, one row at a time across its 256 threads (three
// CTAs per SM, so one CTA's loads are in flight while the others quantize);
// after its first row a CTA takes the next untaken row from a counter in the
// workspace header, so the rows spread by speed, not by count. A row's
// elements with |x| >= threshold are outliers whatever the other rows hold,
// so they are zeroed and the row's absmax and codes are taken over the rest
// before the batch's outlier set O is known. After the grid barrier, with O
// known, each row is finished: the columns of O it did not flag itself get
// code 0 and their values go to Xo; the absmax stands unless every element
// attaining it lies in O (the row's maximum falls in another row's outlier
// column), in which case the row is quantized again from X with O masked.
// Which elements of one vector attain the absmax is recorded while the row is
// in registers, so that check needs no second read of X.
// Same results as quantize_kernel, bit for bit.
constexpr int kStreamVpt = 8;                                  // 16-byte vectors per thread and row
constexpr int64_t kStreamMaxK = (int64_t)kStreamVpt * kThreads * 8;  // 16384
constexpr int kStreamMaxRows = 64;                             // rows per CTA
constexpr int64_t kStreamMinK = 8192;                          // shorter rows: quantize_kernel

// Outlier lanes of two fp16 values: bit 15 (low) / 31 (high) set where
// |x| >= threshold. Exact integer arithmetic on the magnitude bits: 0x8000
// above each 15-bit magnitude keeps the lanes' subtractions apart.
__device__ __forceinline__ uint32_t ge_bits(uint32_t w, uint32_t t2) {
    return (((w & 0x7fff7fffu) | 0x80008000u) - t2) & 0x80008000u;
}

// The 8 outlier flags of a vector as bits 0..7 (from ge_bits of its words).
__device__ __forceinline__ uint32_t flags8(uint32_t g0, uint32_t g1, uint32_t g2, uint32_t g3) {
    return ((g0 >> 15) & 1u) | ((g0 >> 30) & 2u) | ((g1 >> 13) & 4u) | ((g1 >> 28) & 8u) | ((g2 >> 11) & 16u) |
           ((g2 >> 26) & 32u) | ((g3 >> 9) & 64u) | ((g3 >> 24) & 128u);
}

// Zero the flagged lanes of a word (g = its ge_bits).
__device__ __forceinline__ uint32_t clear_flagged(uint32_t w, uint32_t g) { return w & ~((g >> 15) * 0xffffu); }

__device__ __forceinline__ void stream_load(uint4 (&x)[kStreamVpt], const uint4 *row, int nvec, bool live) {
#pragma unroll
    for (int i = 0; i < kStreamVpt; ++i) {
        const int v = threadIdx.x + kThreads * i;
        x[i] = (live && v < nvec) ? __ldg(row + v) : make_uint4(0, 0, 0, 0);
    }
}

// Quantize one row held in x (one CTA): own outliers zeroed, absmax over the
// rest, codes to CA. Records the absmax and a vector attaining it.
__device__ __forceinline__ void stream_row(const QuantizeArgs &a, uint4 (&x)[kStreamVpt], int64_t r, int j, int nvec,
                                           uint32_t t2, uint32_t *bits, uint32_t (*s_wmax)[kWarps],
                                           int (*s_wv)[kWarps], uint32_t *s_amax, int32_t *s_vmax, uint32_t *s_eqm) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t mx = 0;
    int mv = 0;
#pragma unroll
    for (int i = 0; i < kStreamVpt; ++i) {
        const int v = threadIdx.x + kThreads * i;
        if (v < nvec) {
            const uint32_t g0 = ge_bits(x[i].x, t2), g1 = ge_bits(x[i].y, t2);
            const uint32_t g2 = ge_bits(x[i].z, t2), g3 = ge_bits(x[i].w, t2);
            if (g0 | g1 | g2 | g3) {
                atomicOr(&bits[v >> 2], flags8(g0, g1, g2, g3) << ((v & 3) * 8));
                x[i] = make_uint4(clear_flagged(x[i].x, g0), clear_flagged(x[i].y, g1), clear_flagged(x[i].z, g2),
                                  clear_flagged(x[i].w, g3));
            }
            const uint32_t vm = vec_absmax_bits(x[i]);
            if (vm > mx) {
                mx = vm;
                mv = v;
            }
        }
    }
    const uint32_t wm = warp_max_u32(mx);
    const uint32_t who = __ballot_sync(0xffffffffu, mx == wm);
    const int wv = __shfl_sync(0xffffffffu, mv, __ffs(who) - 1);
    uint32_t(&cm)[kWarps] = s_wmax[j & 1];
    int(&cv)[kWarps] = s_wv[j & 1];
    if (lane == 0) {
        cm[warp] = wm;
        cv[warp] = wv;
    }
    __syncthreads();
    uint32_t amax = cm[0];
    int vmax = cv[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w)
        if (cm[w] > amax) {
            amax = cm[w];
            vmax = cv[w];
        }
    const float sa = __half2float(__ushort_as_half((unsigned short)amax));
    const float sc = sa > 0.f ? __fdiv_rn(127.f, sa) : 0.f;
    uint2 *ca2 = reinterpret_cast<uint2 *>(a.CA + r * a.K);
#pragma unroll
    for (int i = 0; i < kStreamVpt; ++i) {
        const int v = threadIdx.x + kThreads * i;
        if (v < nvec) ca2[v] = quant_vec8(x[i], sc);
    }
    // The elements of vector vmax that attain the absmax (its own outliers are
    // zero here, so they never match a nonzero absmax), from the thread that
    // holds that vector.
    if ((vmax & (kThreads - 1)) == (int)threadIdx.x) {
        const int idx = vmax / kThreads;
        uint4 xv = x[0];
#pragma unroll
        for (int i = 1; i < kStreamVpt; ++i)
            if (i == idx) xv = x[i];
        s_eqm[j] = elem_eq_mask(xv, amax);
    }
    if (threadIdx.x == 0) {
        s_amax[j] = amax;
        s_vmax[j] = vmax;
    }
}

__global__ void __launch_bounds__(kThreads, 3) quantize_stream_kernel(QuantizeArgs a) {
    extern __shared__ __align__(128) uint32_t smem[];
    __shared__ uint32_t s_wmax[2][kWarps];
    __shared__ int s_wv[2][kWarps];
    __shared__ uint32_t s_amax[kStreamMaxRows];
    __shared__ int32_t s_vmax[kStreamMaxRows];
    __shared__ uint32_t s_eqm[kStreamMaxRows];
    __shared__ uint32_t s_gen, s_base;
    __shared__ int32_t s_row[kStreamMaxRows];  // the rows this CTA took, in order
    __shared__ int32_t s_next;
    uint32_t *row_next = &a.hdr->row_next;
    const int64_t kwords = ceil_div(a.K, 32);
    uint32_t *bits = smem;                                         // [kwords]
    int32_t *prefix = reinterpret_cast<int32_t *>(smem + kwords);  // [kwords]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nvec = (int)(a.K / 8);
    const uint32_t t2 = (uint32_t)a.tbits | ((uint32_t)a.tbits << 16);
    const uint4 *X4 = reinterpret_cast<const uint4 *>(a.X);
    grid_dep_launch();

    uint4 xa[kStreamVpt];
    stream_load(xa, X4 + (int64_t)blockIdx.x * nvec, nvec, blockIdx.x < a.M);
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

    // Row blockIdx.x first, then rows taken one at a time from a shared
    // counter (the next one is taken while the current one is quantized), so
    // that CTAs which run faster do more rows. At most kStreamMaxRows per CTA;
    // the launch gives every CTA room for ceil(M / grid) rows, so the others
    // take what one CTA leaves.
    int nrows = 0;
    {
        int64_t r0 = blockIdx.x;
        for (int j = 0; r0 < a.M; ++j) {
            if (j > 0) stream_load(xa, X4 + r0 * nvec, nvec, true);
            const bool more = j + 1 < kStreamMaxRows;
            uint32_t taken = 0;
            if (threadIdx.x == 0 && more) taken = atomicAdd(row_next, 1u);
            stream_row(a, xa, r0, j, nvec, t2, bits, s_wmax, s_wv, s_amax, s_vmax, s_eqm);
            if (threadIdx.x == 0) {
                s_row[j] = (int32_t)r0;
                s_next = more ? (int32_t)min((int64_t)gridDim.x + (int64_t)taken, a.M) : (int32_t)a.M;
            }
            __syncthreads();
            r0 = s_next;
            nrows = j + 1;
        }
    }
    __syncthreads();

    // CB into L2 for the GEMM (as quantize_kernel), then the batch's O.
    if (a.Wo && a.CB && a.N * a.K <= kPrefetchMaxBytes && threadIdx.x < 32) {
        const int64_t bytes = weight_bytes(a.N, a.K);
        const int64_t slice = round_up(ceil_div(bytes, gridDim.x), 4096);
        const int64_t b0 = (int64_t)blockIdx.x * slice, b1 = min(bytes, b0 + slice);
        for (int64_t off = b0 + (int64_t)threadIdx.x * 4096; off < b1; off += 32 * 4096) {
            const uint32_t n = (uint32_t)(b1 - off < 4096 ? b1 - off : 4096);
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.CB + off), "r"(n) : "memory");
        }
    }
    for (int64_t w = threadIdx.x; w < kwords; w += kThreads)
        if (bits[w]) atomicOr(&cur[w], bits[w]);
    if (!grid_barrier(a.hdr, gen, s_base, gridDim.x)) return;  // every CTA waits in the same barrier
    if (blockIdx.x == 0 && threadIdx.x == 0) *row_next = 0u;  // every row has been taken
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
                int32_t rk = prefix[w];
                while (v) {
                    if (IN_BOUNDS(rk >= 0 && rk < a.K, &a.hdr->status)) a.outlier_idx[rk] = (int32_t)(w * 32 + __ffs(v) - 1);
                    ++rk;
                    v &= v - 1;
                }
            }
        }
    }

    // Outlier-weight gather Wo[j, t] (as quantize_kernel): half-warps over
    // output channels, a lane per outlier rank, kGatherBatch channels' loads in
    // flight per lane; the first batch's loads are issued here and stored
    // after the rows are finished.
    constexpr int kGatherBatch = 8;
    const int hl = lane & 15;
    const int64_t hw = ((int64_t)blockIdx.x * kWarps + warp) * 2 + (lane >> 4);
    const int64_t nhw = (int64_t)gridDim.x * kWarps * 2;
    const int64_t KB = wblocks_k(a.K);
    __half gv[kGatherBatch];
    auto gather_load = [&](int32_t t0, int64_t j0) {
        const int32_t t = t0 + hl;
        const bool real = t < n_out;
        const int64_t col = real ? outlier_column(bits, prefix, kwords, t) : 0;
#pragma unroll
        for (int u = 0; u < kGatherBatch; ++u) {
            const int64_t jj = j0 + u * nhw;
            gv[u] = __float2half_rn(0.f);
            if (real && jj < a.N && IN_BOUNDS(col >= 0 && col < a.K, &a.hdr->status)) {
                if (a.W_outlier) {
                    gv[u] = a.W_outlier[jj * a.K + col];
                } else {
                    const float p = __fmul_rn((float)a.CB[cb_offset(jj, col, KB)], a.SCB[jj]);
                    gv[u] = __float2half_rn(__fdiv_rn(p, 127.f));
                }
            }
        }
    };
    auto gather_store = [&](int32_t t0, int64_t j0) {
#pragma unroll
        for (int u = 0; u < kGatherBatch; ++u) {
            const int64_t jj = j0 + u * nhw;
            if (jj < a.N && IN_BOUNDS(t0 + hl < a.kcap, &a.hdr->status)) a.Wo[jj * a.kcap + t0 + hl] = gv[u];
        }
    };
    const bool gather = a.Wo && n16 > 0;
    if (gather) gather_load(0, hw);

    // Finish the rows, a warp per row (rows warp, warp + 8, ...). Lane l first
    // checks whether row warp + 8 l keeps its absmax: some element outside O
    // attains it (else the row's maximum lies in O and the row is redone).
    __shared__ int32_t s_redo[kStreamMaxRows];
    __shared__ int32_t s_nredo;
    if (threadIdx.x == 0) s_nredo = 0;
    __syncthreads();
    constexpr int kRowsPerWarp = kStreamMaxRows / kWarps;
    uint32_t keep = 1;
    {
        const int j = warp + kWarps * lane;
        if (lane < kRowsPerWarp && j < nrows && s_amax[j] != 0u)
            keep = (s_eqm[j] & ~vec_mask(bits, s_vmax[j])) != 0u;
    }
    const uint32_t keep_mask = __ballot_sync(0xffffffffu, keep);
    // Columns of O: code 0 and the fp16 value into Xo (zero-padded to 16). With
    // |O| <= 32 lane t owns rank t in every row, its loads issued together.
    if (n16 <= 32) {
        const int64_t col = lane < n_out ? outlier_column(bits, prefix, kwords, lane) : 0;
        __half vals[kRowsPerWarp];
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i) {
            const int j = warp + kWarps * i;
            const int64_t r = (int64_t)s_row[j];
            vals[i] = (j < nrows && lane < n_out) ? a.X[r * a.K + col] : __float2half_rn(0.f);
        }
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i) {
            const int j = warp + kWarps * i;
            if (j >= nrows) break;
            const int64_t r = (int64_t)s_row[j];
            if (lane < n_out) a.CA[r * a.K + col] = 0;
            if (a.Xo && lane < n16 && IN_BOUNDS(lane < a.kcap, &a.hdr->status)) a.Xo[r * a.kcap + lane] = vals[i];
        }
    } else {
        for (int j = warp; j < nrows; j += kWarps) {
            const int64_t r = (int64_t)s_row[j];
            for (int32_t t = lane; t < n16; t += 32) {
                __half val = __float2half_rn(0.f);
                if (t < n_out) {
                    const int64_t col = outlier_column(bits, prefix, kwords, t);
                    val = a.X[r * a.K + col];
                    a.CA[r * a.K + col] = 0;
                }
                if (a.Xo && IN_BOUNDS(t < a.kcap, &a.hdr->status)) a.Xo[r * a.kcap + t] = val;
            }
        }
    }
    for (int i = 0, j = warp; j < nrows; ++i, j += kWarps) {
        if ((keep_mask >> i) & 1u) {
            if (lane == 0) a.SCA[(int64_t)s_row[j]] = __half2float(__ushort_as_half((unsigned short)s_amax[j]));
        } else if (lane == 0) {
            s_redo[atomicAdd(&s_nredo, 1)] = j;
            // its row is read again below: start pulling it into L2 now
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(X4 + (int64_t)s_row[j] * nvec),
                         "r"((uint32_t)(nvec * 16)) : "memory");
        }
    }
    __syncthreads();
    // Rows whose maximum lies in O: the whole CTA quantizes them again from X
    // with O masked (rare: a row's maximum in another row's outlier column).
    // Rolled loops that read the row again (from L2) rather than registers:
    // this code runs about once per launch, in one CTA, and with its loops
    // unrolled most of its time went to fetching its instructions.
    const int nredo = s_nredo;
    for (int k = 0; k < nredo; ++k) {
        const int j = s_redo[k];
        const int64_t r = (int64_t)s_row[j];
        const uint4 *row = X4 + r * nvec;
        uint32_t mx = 0;
#pragma unroll 1
        for (int v = threadIdx.x; v < nvec; v += kThreads) {
            uint4 x = __ldg(row + v);
            const uint32_t m = vec_mask(bits, v);  // O holds every element at or above the threshold
            if (m) x = clear_masked(x, m);
            mx = max(mx, vec_absmax_bits(x));
        }
        mx = warp_max_u32(mx);
        if (lane == 0) s_wmax[k & 1][warp] = mx;
        __syncthreads();
        uint32_t amax = s_wmax[k & 1][0];
#pragma unroll 1
        for (int w = 1; w < kWarps; ++w) amax = max(amax, s_wmax[k & 1][w]);
        const float sa = __half2float(__ushort_as_half((unsigned short)amax));
        const float sc = sa > 0.f ? __fdiv_rn(127.f, sa) : 0.f;
        uint2 *ca2 = reinterpret_cast<uint2 *>(a.CA + r * a.K);
#pragma unroll 1
        for (int v = threadIdx.x; v < nvec; v += kThreads) {
            uint4 x = __ldg(row + v);
            const uint32_t m = vec_mask(bits, v);
            if (m) x = clear_masked(x, m);
            ca2[v] = quant_vec8(x, sc);
        }
        if (threadIdx.x == 0) a.SCA[r] = sa;
    }

    if (gather) {
        gather_store(0, hw);
        for (int32_t t0 = 0; t0 < n16; t0 += 16)
            for (int64_t j0 = hw + (t0 == 0 ? kGatherBatch * nhw : 0); j0 < a.N; j0 += kGatherBatch * nhw) {
                gather_load(t0, j0);
                gather_store(t0, j0);
            }
    }
}

// ----------------------------------------------- decode batches (M <= 8) ----
//
// With at most 8 rows, every CTA of one cluster owns a slice of the columns
// for all rows. A CTA then sees every value of its columns and finds their
// outliers alone; what crosses CTAs is only the rows' partial maxima and the
// CTAs' outlier counts, exchanged through distributed shared memory at one
// cluster barrier. No grid-wide barrier and no global atomics: the kernel
// needs no cooperative launch and may start while the kernel before it
// drains. Further clusters of the same grid (and every CTA, for its share)
// zero the decode GEMV's partial sums and arrival counters.
constexpr int kDecClusterMaxM = 8;      // batches up to this many rows take this pass
constexpr int kDecSmemMax = 160 * 1024;  // staged slice (rows x slice vectors), at most
constexpr int kDecMinCtas = 8;           // CTAs per cluster: 8, or 16 where the device allows it
constexpr int kDecWordsMax = (int)((kMaxKwords + kDecMinCtas - 1) / kDecMinCtas + 3) & ~3;

__device__ __forceinline__ uint32_t ld_shared_cluster_u32(uint32_t cluster_addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
    return v;
}
__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_id_x() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_nctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

// kStage: the CTA's slice of every row is kept in shared memory between the
// passes (else the later passes read it again from X, through L1/L2).
template <bool kStage>
__global__ void __launch_bounds__(kThreads) quantize_decode_kernel(QuantizeArgs a, int64_t wpc) {
    extern __shared__ __align__(128) uint4 s_rows[];              // [M][vs] when staged
    __shared__ uint32_t s_bits[kDecWordsMax];                       // the slice's column bitmap
    __shared__ int32_t s_prefix[kDecWordsMax];                      // exclusive popcount prefix
    __shared__ uint32_t s_rowmax[kDecodeMaxM];                      // the slice's partial row maxima
    __shared__ uint32_t s_final[kDecodeMaxM];                       // the rows' maxima (bit patterns)
    __shared__ int32_t s_count, s_before, s_total;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t C = cluster_nctarank(), c = cluster_ctarank();
    const bool quantizer = cluster_id_x() == 0;
    const int64_t nvec = a.K / 8, kwords = ceil_div(a.K, 32);
    const int64_t w0 = min(kwords, (int64_t)c * wpc), w1 = min(kwords, w0 + wpc);
    const int64_t v0 = w0 * 4, v1 = min(nvec, w1 * 4), vs = v1 - v0;
    const int nw = (int)(w1 - w0);
    const uint32_t t2 = (uint32_t)a.tbits | ((uint32_t)a.tbits << 16);
    const int M = (int)a.M;

    // Let the GEMV behind this pass launch now and pull its first weight
    // blocks into L2 while this pass runs; read nothing until the kernel
    // before this one has finished.
    grid_dep_launch();
    grid_dep_wait();

    // Every CTA of the grid zeroes its share of the GEMV's partial sums: the
    // other clusters at once, the quantizing one after its passes, which are
    // the critical path.
    auto zero_share = [&]() {
        const int64_t b = (int64_t)blockIdx.x, nb = gridDim.x;
        const uint4 z = make_uint4(0, 0, 0, 0);
        if (a.acc) {
            uint4 *acc4 = reinterpret_cast<uint4 *>(a.acc);
            const int64_t n4 = a.acc_words / 4, per = ceil_div(n4, nb);
            for (int64_t i = b * per + threadIdx.x; i < min(n4, (b + 1) * per); i += kThreads) acc4[i] = z;
        }
        if (a.cnt) {
            uint4 *cnt4 = reinterpret_cast<uint4 *>(a.cnt);
            const int64_t n4 = a.cnt_words / 4, per = ceil_div(n4, nb);
            for (int64_t i = b * per + threadIdx.x; i < min(n4, (b + 1) * per); i += kThreads) cnt4[i] = z;
        }
    };
    if (!quantizer) {
        zero_share();
        return;
    }

    // Pass 1: outlier columns of the slice (every row of X is here).
    for (int i = threadIdx.x; i < nw; i += kThreads) s_bits[i] = 0;
    if (threadIdx.x < kDecodeMaxM) s_rowmax[threadIdx.x] = 0;
    __syncthreads();
    const uint4 *X4 = reinterpret_cast<const uint4 *>(a.X);
    for (int t = warp; t < M; t += kWarps) {
        const uint4 *src = X4 + (int64_t)t * nvec + v0;
        for (int64_t v = lane; v < vs; v += 32) {
            const uint4 x = __ldg(src + v);
            if constexpr (kStage) s_rows[(int64_t)t * vs + v] = x;
            flag_vec(x, t2, (int)v, s_bits);
        }
    }
    __syncthreads();

    // Pass 2: each row's maximum over the slice's other columns; the slice's
    // outlier count and the exclusive prefix of its bitmap words.
    for (int t = warp; t < M; t += kWarps) {
        const uint4 *src = kStage ? s_rows + (int64_t)t * vs : X4 + (int64_t)t * nvec + v0;
        uint32_t m = 0;
        for (int64_t v = lane; v < vs; v += 32) {
            uint4 x = kStage ? src[v] : __ldg(src + v);
            const uint32_t mk = vec_mask(s_bits, (int)v);
            if (mk) x = clear_masked(x, mk);
            m = max(m, vec_absmax_bits(x));
        }
        m = warp_max_u32(m);
        if (lane == 0) s_rowmax[t] = m;
    }
    if (warp == 0) {
        // single-warp scan: lane l takes words [l * per, (l + 1) * per)
        const int per = (nw + 31) / 32;
        const int i0 = min(nw, lane * per), i1 = min(nw, i0 + per);
        int32_t mine = 0;
        for (int i = i0; i < i1; ++i) mine += __popc(s_bits[i]);
        int32_t incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
        }
        int32_t run = incl - mine;
        for (int i = i0; i < i1; ++i) {
            s_prefix[i] = run;
            run += __popc(s_bits[i]);
        }
        if (lane == 31) s_count = incl;
    }
    // Publish the partial maxima and the count to the cluster.
    cluster_arrive();
    cluster_wait();
    if (threadIdx.x < (unsigned)M) {
        uint32_t m = 0;
        for (uint32_t r = 0; r < C; ++r)
            m = max(m, ld_shared_cluster_u32(mapa_shared(smem_u32(&s_rowmax[threadIdx.x]), r)));
        s_final[threadIdx.x] = m;
    } else if (threadIdx.x == 32) {
        int32_t before = 0, total = 0;
        for (uint32_t r = 0; r < C; ++r) {
            const int32_t n = (int32_t)ld_shared_cluster_u32(mapa_shared(smem_u32(&s_count), r));
            if (r < c) before += n;
            total += n;
        }
        s_before = before;
        s_total = total;
    }
    // This CTA no longer reads the others' shared memory; each waits for all
    // before it exits, so none leaves while another still reads its values.
    __syncthreads();
    cluster_arrive();

    // Pass 3: codes, scales, the outlier list and the outlier activations.
    const int32_t before = s_before, n_out = s_total;
    if (c == 0) {
        if (threadIdx.x < (unsigned)M)
            a.SCA[threadIdx.x] = __half2float(__ushort_as_half((unsigned short)s_final[threadIdx.x]));
        if (threadIdx.x == 0 && a.n_outliers) *a.n_outliers = n_out;
        if (a.Xo) {
            const int32_t n16 = (n_out + 15) & ~15;
            for (int i = threadIdx.x; i < M * (n16 - n_out); i += kThreads) {
                const int t = i / (n16 - n_out), j = n_out + i % (n16 - n_out);
                if (IN_BOUNDS(j < a.kcap, &a.hdr->status)) a.Xo[(int64_t)t * a.kcap + j] = __float2half_rn(0.f);
            }
        }
    }
    if (a.outlier_idx)
        for (int i = threadIdx.x; i < nw; i += kThreads) {
            uint32_t b = s_bits[i];
            int32_t r = before + s_prefix[i];
            while (b) {
                if (IN_BOUNDS(r >= 0 && r < a.K, &a.hdr->status)) a.outlier_idx[r] = (int32_t)((w0 + i) * 32 + __ffs(b) - 1);
                ++r;
                b &= b - 1;
            }
        }
    for (int t = warp; t < M; t += kWarps) {
        const uint4 *src = kStage ? s_rows + (int64_t)t * vs : X4 + (int64_t)t * nvec + v0;
        const float sa = __half2float(__ushort_as_half((unsigned short)s_final[t]));
        const float sc = sa > 0.f ? __fdiv_rn(127.f, sa) : 0.f;
        uint2 *ca2 = reinterpret_cast<uint2 *>(a.CA + (int64_t)t * a.K) + v0;
        __half *xo = a.Xo ? a.Xo + (int64_t)t * a.kcap + before : nullptr;
        for (int64_t v = lane; v < vs; v += 32) {
            uint4 x = kStage ? src[v] : __ldg(src + v);
            const uint32_t mk = vec_mask(s_bits, (int)v);
            if (mk) {
                if (xo) store_outliers(x, mk, (int)v, s_bits, s_prefix, xo, a.kcap - before, &a.hdr->status);
                x = clear_masked(x, mk);
            }
            ca2[v] = quant_vec8(x, sc);
        }
    }
    zero_share();
    cluster_wait();
}

// Test kernel: the quantize pass's grid barrier, entered by a grid that
// counts one CTA more than it has, so the wait cannot end before limit_ns.
// It reads the launch generation and base as quantize_kernel does, records
// the timeout in the status word and returns; the header's counts are then
// off until the workspace is initialised again.
__global__ void barrier_timeout_kernel(WsHeader *h, uint64_t limit_ns) {
    __shared__ uint32_t s_gen, s_base;
    if (threadIdx.x == 0) {
        s_gen = *reinterpret_cast<volatile uint32_t *>(&h->qgen);
        s_base = *reinterpret_cast<volatile uint32_t *>(&h->qbase);
    }
    __syncthreads();
    grid_barrier(h, s_gen, s_base, gridDim.x + 1u, limit_ns);
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
    int64_t blocks = ceil_div(round_up(N, kWBlockRows), kWarps);
    if (blocks > 148 * 16) blocks = 148 * 16;
    prepare_weight_kernel<<<(unsigned)blocks, kThreads, 0, s>>>(W, N, K, CB, SCB);
    return cudaGetLastError();
}

namespace {

// Largest dynamic shared memory a CTA may ask for while two still fit on an SM.
constexpr int kQuantDynMax = 113 * 1024 - 512;
// Batches up to this many elements (and no outlier-weight gather to spread)
// are quantized by a single CTA.
constexpr int64_t kAloneElems = 64 * 1024;
constexpr int64_t kAloneClearWords = 64 * 1024;  // and at most this many decode sums to zero
constexpr int64_t kClearWordsPerCta = 8 * 1024;  // decode sums zeroed per CTA otherwise

struct QuantOcc {
    std::mutex mu;
    bool init = false;
    cudaError_t err = cudaSuccess;
    int sms = 0;
    int cached_dyn[8] = {}, cached_per_sm[8] = {}, n_cached = 0;
};

// Resident CTAs per SM of quantize_kernel with `dyn` bytes of dynamic shared
// memory on the current device (cached per device and size).
cudaError_t quant_resident(int dyn, int *ctas) {
    static QuantOcc occ[64];
    int dev = 0;
    if (cudaError_t e = cudaGetDevice(&dev)) return e;
    QuantOcc &o = occ[dev & 63];
    std::lock_guard<std::mutex> lock(o.mu);
    if (!o.init) {
        o.init = true;
        o.err = cudaFuncSetAttribute(quantize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kQuantDynMax);
        if (o.err == cudaSuccess) o.err = cudaDeviceGetAttribute(&o.sms, cudaDevAttrMultiProcessorCount, dev);
    }
    if (o.err != cudaSuccess) return o.err;
    for (int i = 0; i < o.n_cached; ++i)
        if (o.cached_dyn[i] == dyn) {
            *ctas = o.cached_per_sm[i] * o.sms;
            return cudaSuccess;
        }
    int per_sm = 0;
    if (cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quantize_kernel, kThreads, dyn)) return e;
    const int slot = o.n_cached < 8 ? o.n_cached++ : (dyn & 7);
    o.cached_dyn[slot] = dyn;
    o.cached_per_sm[slot] = per_sm;
    *ctas = per_sm * o.sms;
    return cudaSuccess;
}

}  // namespace

// Resident CTAs of quantize_stream_kernel on the current device (cached;
// its shared memory is at most 4 KB of bitmap and prefix, whatever K).
cudaError_t stream_resident(int *ctas) {
    static int cached[64];
    static std::once_flag once[64];
    static cudaError_t err[64];
    int dev = 0;
    if (cudaError_t e = cudaGetDevice(&dev)) return e;
    std::call_once(once[dev & 63], [dev] {
        int sms = 0, per_sm = 0;
        err[dev & 63] = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (err[dev & 63] == cudaSuccess)
            err[dev & 63] = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                &per_sm, quantize_stream_kernel, kThreads, (size_t)2 * (kStreamMaxK / 32) * 4);
        cached[dev & 63] = sms * per_sm;
    });
    *ctas = cached[dev & 63];
    return err[dev & 63];
}

// CTAs per cluster of quantize_decode_kernel on the current device: 16 where
// a cluster of that size (non-portable) fits with the largest staging buffer,
// else 8. Cached per device; the kernels' attributes are set on first use.
cudaError_t decode_cluster_size(int *C) {
    static std::once_flag once[64];
    static int size[64];
    static cudaError_t err[64];
    int dev = 0;
    if (cudaError_t e = cudaGetDevice(&dev)) return e;
    std::call_once(once[dev & 63], [dev] {
        cudaError_t e = cudaFuncSetAttribute(quantize_decode_kernel<true>,
                                             cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(quantize_decode_kernel<false>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(quantize_decode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kDecSmemMax);
        int n = 0;
        if (e == cudaSuccess) {
            cudaLaunchConfig_t cfg = {};
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 16;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.gridDim = dim3(16, 1, 1);
            cfg.blockDim = dim3(kThreads, 1, 1);
            cfg.dynamicSmemBytes = kDecSmemMax;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (cudaOccupancyMaxActiveClusters(&n, quantize_decode_kernel<true>, &cfg) != cudaSuccess) {
                (void)cudaGetLastError();  // not supported here: use the portable size
                n = 0;
            }
        }
        err[dev & 63] = e;
        size[dev & 63] = n >= 1 ? 16 : kDecMinCtas;
    });
    *C = size[dev & 63];
    return err[dev & 63];
}

// Decode batches: one cluster quantizes (column slices of whole bitmap words
// per CTA), and the grid has enough clusters to zero the GEMV's partial sums
// at about 32 KB per CTA.
cudaError_t launch_quantize_decode(const QuantizeArgs &a, cudaStream_t s) {
    int C = kDecMinCtas;
    if (cudaError_t e = decode_cluster_size(&C)) return e;
    int sms = 0, dev = 0;
    if (cudaError_t e = cudaGetDevice(&dev)) return e;
    if (cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) return e;
    const int64_t kwords = ceil_div(a.K, 32);
    const int64_t wpc = ceil_div(kwords, C);
    const int64_t stage = a.M * 4 * wpc * 16;
    const int64_t zero_bytes = 4 * ((a.acc ? a.acc_words : 0) + (a.cnt ? a.cnt_words : 0));
    const int64_t clusters = std::max<int64_t>(1, std::min<int64_t>(std::max(1, sms / C),
                                                                     ceil_div(zero_bytes, (int64_t)C * 32768)));
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)(clusters * C), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (stage <= kDecSmemMax) {
        cfg.dynamicSmemBytes = (size_t)stage;
        return cudaLaunchKernelEx(&cfg, quantize_decode_kernel<true>, a, wpc);
    }
    return cudaLaunchKernelEx(&cfg, quantize_decode_kernel<false>, a, wpc);
}

cudaError_t launch_quantize(const QuantizeArgs &a, cudaStream_t s) {
    // Decode batches of up to 8 rows: a cluster-local pass, no grid barrier.
    // (For 9 to 16 rows it measured no faster per decode step than the
    // cooperative pass below, and up to 60% slower at 14 to 16 rows when the
    // GEMV behind it was let launch early.)
    if (a.M <= kDecClusterMaxM && !a.Wo) return launch_quantize_decode(a, s);
    // Prefill batches with long rows: X streamed once, a row per CTA at a time.
    if (a.M > kDecodeMaxM && a.K >= kStreamMinK && a.K <= kStreamMaxK && !a.acc && !a.cnt) {
        int resident = 0;
        if (cudaError_t e = stream_resident(&resident)) return e;
        if (resident > 0 && ceil_div(a.M, resident) <= kStreamMaxRows) {
            cudaLaunchConfig_t cfg = {};
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeCooperative;
            attr[0].val.cooperative = 1;
            cfg.gridDim = dim3((unsigned)std::min<int64_t>(resident, a.M), 1, 1);
            cfg.blockDim = dim3(kThreads, 1, 1);
            cfg.dynamicSmemBytes = (size_t)2 * ceil_div(a.K, 32) * 4;
            cfg.stream = s;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            return cudaLaunchKernelEx(&cfg, quantize_stream_kernel, a);
        }
    }
    const int64_t kwords = ceil_div(a.K, 32);
    const int64_t bits_bytes = round_up(2 * kwords * 4, 128);
    const int64_t row_bytes = 2 * a.K;
    // Rows kept per CTA and round (0: rows too long to keep; phase B reads X).
    const int64_t r_max = std::min<int64_t>(64, (kQuantDynMax - bits_bytes) / row_bytes);
    int R = 0, rounds = 1, grid = 0, resident = 0;
    if (r_max > 0) {
        if (cudaError_t e = quant_resident((int)(bits_bytes + r_max * row_bytes), &resident)) return e;
        if (resident <= 0) return cudaErrorInvalidConfiguration;
        if (a.M <= r_max && a.M * a.K <= kAloneElems && !a.Wo && a.acc_words <= kAloneClearWords) {
            // A small batch: one CTA, no grid-wide step at all.
            R = (int)a.M;
            grid = 1;
        } else if (a.M <= r_max * resident) {
            // One round: spread the rows over every resident CTA.
            R = (int)ceil_div(a.M, resident);
            grid = (int)ceil_div(a.M, R);
        } else {
            // Several rounds of equal size; the last one stays staged.
            grid = resident;
            rounds = (int)ceil_div(a.M, r_max * resident);
            R = (int)ceil_div(a.M, (int64_t)resident * rounds);
        }
    } else {
        if (cudaError_t e = quant_resident((int)bits_bytes, &resident)) return e;
        if (resident <= 0) return cudaErrorInvalidConfiguration;
        grid = (int)std::min<int64_t>(resident, std::max<int64_t>(1, ceil_div(a.M, kWarps)));
    }
    // The outlier-weight gather runs over all N output channels: give it
    // enough CTAs even when there are few rows.
    if (a.Wo) grid = (int)std::max<int64_t>(grid, std::min<int64_t>(resident, ceil_div(a.N, 32)));
    // The decode GEMV's partial sums are zeroed 32 KB per CTA (a grid of a
    // dozen CTAs for 3 MB took 2.5 µs longer per decode step).
    if (a.acc) grid = (int)std::max<int64_t>(grid, std::min<int64_t>(resident, ceil_div(a.acc_words, kClearWordsPerCta)));
    if (R == 0) rounds = (int)ceil_div(a.M, (int64_t)kWarps * grid);  // kWarps rows per CTA and round
    // The grid barrier needs every CTA resident at once: a cooperative launch.
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.gridDim = dim3((unsigned)std::max(grid, 1), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = (size_t)(bits_bytes + (int64_t)R * row_bytes);
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, quantize_kernel, a, kwords, R, rounds);
}

cudaError_t launch_barrier_timeout(WsHeader *h, uint64_t limit_ns, cudaStream_t s) {
    barrier_timeout_kernel<<<1, kThreads, 0, s>>>(h, limit_ns);
    return cudaGetLastError();
}

}  // namespace int8lt
