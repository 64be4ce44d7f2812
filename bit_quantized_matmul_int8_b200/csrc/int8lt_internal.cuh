// Internal declarations of libint8lt: workspace layout, kernel launchers and
// the sm_100a PTX wrappers (mbarrier, TMA, tcgen05) the kernels share.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/int8lt.h"

namespace int8lt {

constexpr int64_t kMaxK = 133144;       // 127^2 * K < 2^31
constexpr int kDecodeMaxM = 16;         // M <= 16 takes the GEMV path
constexpr int64_t kMaxKwords = (kMaxK + 31) / 32;  // words of the largest column bitmap
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s bound on every in-kernel wait

// Device status bits (workspace header word 0).
constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusBounds = 2u;  // checking builds: an index failed its bounds check

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

// Weight codes (CB) are stored in blocks of 32 output channels x 128 bytes of
// K, each block 4 KB contiguous, blocks ordered by row block, then k-block:
//   CB[j, k] at ((j / 32) * ceil(K / 128) + k / 128) * 4096 + (j % 32) * 128 + k % 128.
// Codes past N rows or K columns inside the last blocks are zero. A decode
// GEMV then streams one contiguous range of CB per warp, and the GEMM's TMA
// reads a 128-row tile as four 4 KB blocks.
constexpr int64_t kWBlockRows = 32, kWBlockCols = 128, kWBlockBytes = kWBlockRows * kWBlockCols;
__host__ __device__ __forceinline__ int64_t wblocks_k(int64_t K) { return ceil_div(K, kWBlockCols); }
__host__ __device__ __forceinline__ int64_t cb_offset(int64_t j, int64_t k, int64_t KB) {
    return ((j >> 5) * KB + (k >> 7)) * kWBlockBytes + (j & 31) * kWBlockCols + (k & 127);
}
__host__ __device__ __forceinline__ int64_t weight_bytes(int64_t N, int64_t K) {
    return ceil_div(N, kWBlockRows) * wblocks_k(K) * kWBlockBytes;
}

// Byte offsets of the workspace sections (every section 1024-byte aligned).
// The header and the two column bitmaps sit at fixed offsets whatever the
// shape, so one zeroing of the first kWsInitBytes prepares any workspace.
struct WsLayout {
    int64_t M, N, K;
    int64_t kwords;        // ceil(K / 32): words of one column bitmap
    int64_t kcap;          // round_up(K, 64): row pitch (elements) of Xo / Wo
    size_t hdr, bitmaps, idx, sca, ca, xo, wo, acc, cnt, sk;
    size_t zpa;            // zeropoint forward: zp_a [M] then the code sums [M] (int32)
    size_t total;
};
WsLayout ws_layout(int64_t M, int64_t N, int64_t K);

// Workspace header (first 256 bytes).
struct WsHeader {
    uint32_t status;       // kStatus* bits, sticky until read
    int32_t n_outliers;    // |O| of the last quantize pass
    uint32_t qgen;         // quantize launches so far: selects this launch's bitmap
    uint32_t bar_count;    // arrivals at the quantize grid barrier, all launches (wraps)
    uint32_t qbase;        // bar_count when the next quantize launch starts
    uint32_t row_next;     // streaming quantize: rows handed out past the first one per CTA (0 between launches)
    uint32_t pad[58];
};
static_assert(sizeof(WsHeader) == 256, "workspace header");
constexpr size_t kWsBitmapOffset = 1024;
// Stream-K of the prefill GEMM: one ready flag per (CTA pair, rank) in the
// zeroed region, and one int32 partial tile (128 x 256) per (pair, rank).
constexpr int kSkMaxPairs = 80;
constexpr size_t kSkPartialBytes = (size_t)128 * 256 * 4;
constexpr size_t kWsSkFlagOffset = kWsBitmapOffset + ((2 * (size_t)kMaxKwords * 4 + 1023) & ~size_t(1023));
constexpr size_t kWsInitBytes = kWsSkFlagOffset + 1024;
static_assert(2 * kSkMaxPairs * 4 <= 1024, "stream-K flags");

// ------------------------------------------------------------- launchers --

// fp16 bit pattern T: |x| >= threshold  <=>  (bits(x) & 0x7fff) >= T.
uint16_t threshold_bits(float threshold);

// Row-major int8 codes [N, K] <-> the blocked weight layout (pack: rows -> blocked).
cudaError_t launch_convert_weight(bool pack, int8_t *blocked, int8_t *rows, int64_t N, int64_t K, cudaStream_t s);

cudaError_t launch_prepare_weight(const __half *W, int64_t N, int64_t K, int8_t *CB, float *SCB,
                                  cudaStream_t s);

struct QuantizeArgs {
    const __half *X;
    int64_t M, K;
    WsHeader *hdr;            // generation counter and grid-barrier count
    uint32_t *bitmaps;        // 2 x kMaxKwords words, one per launch parity
    uint16_t tbits;
    int8_t *CA;
    float *SCA;
    int32_t *outlier_idx;     // may be null
    int32_t *n_outliers;      // may be null
    __half *Xo;               // [M][kcap] or null
    int64_t kcap;
    // Outlier weight gather (M > 16 path): Wo[j][t] for t < round_up(|O|, 16).
    const __half *W_outlier;  // null -> from CB/SCB
    const int8_t *CB;
    const float *SCB;
    __half *Wo;               // [N][kcap] or null (no gather)
    int64_t N;
    // Decode path: partial-sum buffers to zero for the GEMV, or null.
    int32_t *acc;
    int64_t acc_words;        // a multiple of 4
    uint32_t *cnt;
    int64_t cnt_words;
};
// Outlier detection and row quantization in one cooperative launch: column
// flags of every row, a grid barrier, then codes/scales/outlier gathers.
cudaError_t launch_quantize(const QuantizeArgs &a, cudaStream_t s);

// Zeropoint quantization of the rows of an fp16 matrix [R, K] (K % 8 == 0).
struct ZpQuantArgs {
    const __half *X;
    int64_t R, K;
    int8_t *Q;                // [R, K] codes, row-major (or the blocked weight layout)
    bool blocked;             // Q in the blocked weight layout, padding zeroed
    float *ND;                // [R]
    int32_t *ZP;              // [R]
    int32_t *SUM;             // [R]
    // Decode path: partial-sum buffers to zero for the GEMV, or null.
    int32_t *acc;
    int64_t acc_words;        // a multiple of 4
    uint32_t *cnt;
    int64_t cnt_words;        // a multiple of 4
};
cudaError_t launch_zp_quantize(const ZpQuantArgs &a, cudaStream_t s);

struct GemmArgs {
    const int8_t *CA;
    const int8_t *CB;
    const float *SCA;
    const float *SCB;
    const __half *Xo;         // [M][kcap]
    const __half *Wo;         // [N][kcap]
    int64_t kcap;
    const int32_t *n_outliers;  // device; null -> no outlier term
    const __half *bias;
    __half *Y;
    int32_t *C32;             // debug: raw int32 output instead of Y
    int64_t M, N, K;
    uint32_t *status;
    // Stream-K of the last wave (both null: whole tiles only).
    int32_t *sk_partial;      // [kSkMaxPairs][2][128][256]
    uint32_t *sk_flags;       // [kSkMaxPairs][2], zero between launches
    // Zeropoint mode (ZB non-null): SCA / SCB hold nd_a / nd_b, no outlier term.
    const int32_t *ZA, *SA;   // [M] zeropoints and code sums of the rows of CA
    const int32_t *ZB, *SB;   // [N] zeropoints and code sums of the rows of CB
};
cudaError_t launch_gemm_tc(const GemmArgs &a, cudaStream_t s);

struct GemvArgs {
    const int8_t *CA;
    const int8_t *CB;
    const float *SCA;
    const float *SCB;
    const __half *Xo;           // [M][kcap]
    int64_t kcap;
    const int32_t *outlier_idx;
    const int32_t *n_outliers;  // null -> no outlier term
    const __half *W_outlier;    // null -> CB/SCB recovery
    const __half *bias;
    __half *Y;
    int32_t *C32;               // debug: raw int32 output instead of Y
    int32_t *acc;               // partial sums of split row groups [N][M], zero on entry
    uint32_t *cnt;              // K segments summed per group of 8 rows [ceil(N/8)], zero on entry
    uint32_t *status;           // workspace status word (timeouts), may be null
    int64_t M, N, K;
    // Zeropoint mode (ZB non-null): SCA / SCB hold nd_a / nd_b, no outlier term.
    const int32_t *ZA, *SA;     // [M]
    const int32_t *ZB, *SB;     // [N]
};
cudaError_t launch_gemv(const GemvArgs &a, cudaStream_t s);

// 2-D row-major TMA map: `inner` elements per row (contiguous), `outer` rows,
// row pitch `pitch_bytes`; box of box_inner x box_outer; out-of-range
// elements read as zero. False if the driver rejects it.
bool make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
              uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer,
              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B);

cudaError_t launch_wait_timeout(uint32_t *status, uint64_t limit_ns, cudaStream_t s);
// One CTA at the quantize pass's grid barrier, waiting for a CTA that does not exist.
cudaError_t launch_barrier_timeout(WsHeader *h, uint64_t limit_ns, cudaStream_t s);

// The two halves of int8lt_forward on an already validated call; `ws` holds
// at least ws_layout(M, N, K).total bytes. Return an int8lt_status.
int forward_quantize(const void *X, int64_t M, int64_t N, int64_t K, const int8_t *CB, const float *SCB,
                     const void *W_outlier, float threshold, void *ws, cudaStream_t s);
int forward_matmul(int64_t M, int64_t N, int64_t K, const int8_t *CB, const float *SCB, const void *W_outlier,
                   const void *bias, void *Y, void *ws, cudaStream_t s);

// ------------------------------------------------------- device helpers --
#ifdef __CUDACC__

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait until the barrier phase with parity `parity` has completed, for at
// most limit_ns. Returns false on timeout (the caller records it and stops).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > limit_ns) return false;
    }
}

__device__ __forceinline__ void record_timeout(uint32_t *status) {
    if (status) atomicOr(status, kStatusTimeout);
}

// Bounds checks of the checking build (compiled with -DINT8LT_DEBUG): every
// computed global access of the kernels goes through IN_BOUNDS(index <
// extent, status word); a failed check records kStatusBounds and the access
// is skipped, so a wrong index is reported instead of touching memory that is
// not the buffer's. The regular build compiles the checks away.
__device__ __forceinline__ bool bounds_ok(bool ok, uint32_t *status) {
    if (!ok && status) atomicOr(status, kStatusBounds);
    return ok;
}
#ifdef INT8LT_DEBUG
#define IN_BOUNDS(cond, status) (::int8lt::bounds_ok((cond), (status)))
#else
#define IN_BOUNDS(cond, status) true
#endif

__device__ __forceinline__ void tma_prefetch(const CUtensorMap *m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 2-D tiled TMA load global -> shared, completion counted on `bar`.
// x is the innermost (contiguous) coordinate in elements.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *m, uint32_t bar,
                                            int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

// --- tcgen05 (5th-generation tensor core, accumulators in tensor memory) ---

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, int8 x int8 -> int32.
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, fp16 x fp16 -> fp32.
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every tcgen05.mma issued so far by this thread is done.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp gets lane
// (base lane + t), columns [col, col + 32).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the previous kernel in the stream is still
// running; grid_dep_wait() blocks until that kernel has completed and its
// memory is visible. grid_dep_launch() lets the dependent kernel start early.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Store 32 consecutive 32-bit TMEM columns of this warp's 32 lanes (one
// lane per thread), the inverse of tmem_ld_32x32b_x32.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// L2 policy that marks every line it touches evict-first: such lines are
// replaced before normal ones.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
// 2-D tiled TMA store shared -> global (bulk-group completion) with an L2
// cache policy for the written lines. Elements of the box outside the tensor
// are not written.
__device__ __forceinline__ void tma_store_2d_hint(const CUtensorMap *m, uint32_t src, int32_t x, int32_t y,
                                                  uint64_t policy) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%2, %3}], [%1], %4;" ::"l"(
                     reinterpret_cast<uint64_t>(m)),
                 "r"(src), "r"(x), "r"(y), "l"(policy)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// At most one committed store group may still be reading shared memory.
__device__ __forceinline__ void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Every committed store group has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// --- CTA pairs (cluster of 2) and the 2-SM tensor-core instructions -------

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address of the same shared variable in cluster CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

// Arrive on an mbarrier of any CTA of the cluster (shared::cluster address).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// 4-D tiled TMA load (coordinates innermost first) into this CTA's shared
// memory, completion counted on the mbarrier at `bar_cluster` as for
// tma_load_2d_pair. No multicast.
__device__ __forceinline__ void tma_load_4d_pair(uint32_t dst, const CUtensorMap *m, uint32_t bar_cluster,
                                                 int32_t c0, int32_t c1, int32_t c2, int32_t c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

// 2-D tiled TMA load into this CTA's shared memory whose completion is
// counted on the mbarrier at `bar_cluster` (shared::cluster address, here
// the pair leader's barrier). No multicast.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *m, uint32_t bar_cluster,
                                                 int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Pair MMA issued by the leader CTA: A rows split across the two CTAs (128
// each), B split by N (half each), D rows of each CTA in its own TMEM.
__device__ __forceinline__ void mma_i8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_f16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on the mbarrier at the same offset in every CTA of `cta_mask` once
// all pair MMAs issued so far by this thread are done.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            bar),
        "h"(cta_mask)
        : "memory");
}

// Shared-memory matrix descriptor for a K-major tile written by TMA with
// 128-byte swizzling: rows of 128 bytes, 8-row (1024-byte) swizzle atoms
// stacked along M/N (stride byte offset 1024). Tile base 1024-byte aligned.
__device__ __forceinline__ uint64_t sdesc_k_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);  // start address, 16-byte units
    d |= (uint64_t)1 << 16;                    // leading byte offset (unused here)
    d |= (uint64_t)(1024 >> 4) << 32;          // stride byte offset
    d |= (uint64_t)1 << 46;                    // descriptor version for tcgen05
    d |= (uint64_t)2 << 61;                    // 128-byte swizzle
    return d;
}

// Same for a K-major tile with 64-byte swizzling: rows of 64 bytes, 8-row
// (512-byte) swizzle atoms stacked along M/N (stride byte offset 512).
__device__ __forceinline__ uint64_t sdesc_k_sw64(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(512 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)4 << 61;                    // 64-byte swizzle
    return d;
}

#endif  // __CUDACC__

}  // namespace int8lt
