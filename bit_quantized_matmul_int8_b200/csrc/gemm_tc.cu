// Prefill path of the LLM.int8() forward on sm_100a tensor cores.
//
// Computes, per 256 x 256 output tile,
//     Y = fp16( C * SCA[i] * SCB[j] / 127^2 + bias[j] + P )
//     C = CA . CB^T    int8 x int8 -> int32   ("Int8 Matrix Multiplication with
//                      16-bit Float Inputs and Outputs" and "Vector-wise
//                      Quantization", LLM.int8() paper summary)
//     P = Xo . Wo^T    fp16 x fp16 -> fp32    (the outlier columns, "The Core
//                      of LLM.int8(): Mixed-precision Decomposition")
// in one persistent kernel run by CTA pairs (clusters of 2 SMs). Each tile
// is computed by one pair with 2-SM tensor-core MMAs (tcgen05 cta_group::2):
// each CTA stages its own 128 rows of A and its own half (128 rows) of B,
// so per SM a 128 x 256 x 128 k-block needs 32 KB of operands instead of
// 48 KB, and a 5-deep ring of stages fits in shared memory.
//   warp 0     (both CTAs) TMA producer: the int8 k-blocks into the ring, and
//              the tile's outlier columns (Xo, Wo: 32 fp16 per row, 64-byte
//              swizzle) into a slot of their own; the loads of both CTAs
//              complete on the leader CTA's barriers;
//   warp 1     (both CTAs) allocates the 512 tensor-memory columns: two int32
//              accumulators of 256 columns, so the epilogue of one tile
//              overlaps the mainloop of the next; in the leader it issues the
//              pair MMAs and multicasts the commits;
//   warps 2-9  (both CTAs) epilogue on the CTA's 128 rows.
// With outlier columns (|O| > 0) the epilogue runs in two passes over the
// tile's accumulator: it dequantizes the int32 sums to fp32 (plus bias) and
// writes them back into the same tensor-memory columns; the MMA warp then
// adds P there with kind::f16 MMAs (fp32 accumulate, K = 16 per MMA) while
// the next tile's int8 MMAs run; the second pass converts to fp16 and stores
// through shared memory with TMA (32 x 32 boxes, double buffered per warp).
// Without outliers the epilogue is a single pass.
// Every wait is bounded (kWaitLimitNs); a wait that runs out sets the
// workspace status word and the kernel winds down without touching Y.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "int8lt_internal.cuh"

namespace int8lt {

// Work of one CTA pair. Whole tiles round-robin over the pairs ("data
// parallel"), and, when the tile count is not a multiple of the pair count,
// the last one to two waves' worth of tiles are cut into k-block ranges of
// equal length, one per pair ("stream-K"), so every pair gets the same
// number of k-blocks. A range covers at least one tile, so a tile is split
// at most once: its first k-blocks end pair p's range (the "head", which
// finishes the tile) and its last k-blocks start pair p + 1's range (the
// "tail", which hands its int32 partial sums over through global memory).
struct Seg {
    int tile, kb0, kb1;
    bool head, tail;
};

struct TileSched {
    int num_tiles, nkb, total_kb, num_pairs, pair, dp_tiles;
    int64_t r, r_end;   // stream-K k-block cursor of this pair
    int dp_next;

    __host__ __device__ TileSched(int tiles, int nkb_, int total_kb_, int pairs, int p, bool sk_on)
        : num_tiles(tiles), nkb(nkb_), total_kb(total_kb_), num_pairs(pairs), pair(p) {
        dp_tiles = tiles;
        r = r_end = 0;
        if (sk_on && tiles > pairs && tiles % pairs != 0) {
            const int full = tiles / pairs;
            dp_tiles = (full - 1) * pairs;
            const int64_t iters = (int64_t)(tiles - dp_tiles) * nkb;
            r = iters * p / pairs;
            r_end = iters * (p + 1) / pairs;
        }
        dp_next = p;
    }
    __host__ __device__ bool next(Seg &g) {
        if (dp_next < dp_tiles) {
            g.tile = dp_next;
            g.kb0 = 0;
            g.kb1 = total_kb;
            g.head = g.tail = false;
            dp_next += num_pairs;
            return true;
        }
        if (r >= r_end) return false;
        g.tile = dp_tiles + (int)(r / nkb);
        g.kb0 = (int)(r % nkb);
        const int64_t left = r_end - r;
        g.kb1 = left < (int64_t)(nkb - g.kb0) ? g.kb0 + (int)left : nkb;
        g.head = g.kb0 == 0 && g.kb1 < nkb;
        g.tail = g.kb0 > 0;
        r += g.kb1 - g.kb0;
        return true;
    }
};

// Output tile t -> (tile row m, tile column n). The tiles go in groups of
// kGroupM tile rows, tile column by tile column inside a group, so the pairs
// working at the same time (one wave of consecutive tiles) share a few row
// panels of A and column panels of B; the next wave reuses the same A panels
// from L2. (With the tile row as the fast index a wave touched every row panel
// of A, and on a 8192 x 12288 x 36864 product the kernel read 8.1 GB from DRAM
// for 0.55 GB of operands.)
constexpr int kGroupM = 8;
__host__ __device__ __forceinline__ void tile_mn(int t, int num_m, int num_tiles, int &m, int &n) {
    const int num_n = num_tiles / num_m;
    const int per_group = kGroupM * num_n;
    const int g = t / per_group;
    const int first_m = g * kGroupM;
    const int gm = min(num_m - first_m, kGroupM);
    const int r = t - g * per_group;
    m = first_m + r % gm;
    n = r / gm;
}

// Split policy (INT8LT_SPLIT_*): process-wide, read at each launch.
std::atomic<int> g_split_mode{0};

// Whether the tiles after the last full wave are split between pairs. Auto:
// only when it saves the busiest pair at least 32 k-blocks, roughly the
// measured cost of handing the tails' int32 sums over.
bool split_wanted(int64_t tiles, int nkb, int pairs, int mode) {
    if (pairs > kSkMaxPairs || tiles <= pairs || tiles % pairs == 0 || mode == 2) return false;
    if (mode == 1) return true;
    const int64_t waves = (tiles + pairs - 1) / pairs;
    const int64_t saved = (waves * pairs - tiles) * (int64_t)nkb / pairs;  // k-blocks per pair
    return saved >= 32;
}

namespace {

constexpr int BM = 256, BN = 256;         // pair tile
constexpr int kCtaRows = 128;             // rows of A (and of B) staged per CTA
constexpr int kStages = 5;
constexpr int kStageA = kCtaRows * 128;   // bytes: 128 rows x 128 B
constexpr int kStageB = kCtaRows * 128;   // bytes: 128 rows x 128 B (half of N)
constexpr uint32_t kTxBytes = 2 * (kStageA + kStageB);  // both CTAs, counted by the leader
constexpr int kOkb = 32;                  // outlier columns per k-block (64-byte rows)
constexpr int kOStage = kCtaRows * kOkb * 2;            // bytes of Xo (or Wo) per CTA: 8 KB
constexpr uint32_t kOTxBytes = 2 * 2 * kOStage;         // Xo + Wo of both CTAs
constexpr int kEpiWarps = 8;                      // 2 per TMEM lane quadrant
constexpr int kEpiCols = BN * 4 / kEpiWarps;      // accumulator columns per epilogue warp
constexpr int kEpiChunks = kEpiCols / 32;         // tcgen05.ld chunks of 32 columns per warp
constexpr int kBoxes = 2;                         // fp16 store boxes per epilogue warp
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kThreads = 64 + kEpiThreads;
constexpr uint32_t kTmemCols = 512;
constexpr int kEpiBarrier = 1;            // named barrier of the epilogue warps
constexpr uint16_t kPairMask = 0x3;       // both CTAs of the cluster

// Instruction descriptors (tcgen05 .kind::i8 / .kind::f16): dense, K-major
// A and B, N = 256 (bits 17-22 hold N/8), M = 256 (bits 24-28 hold M/16).
constexpr uint32_t kIdescI8 = (2u << 4)      // D = s32
                              | (1u << 7)    // A = signed int8
                              | (1u << 10)   // B = signed int8
                              | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
constexpr uint32_t kIdescF16 = (1u << 4)     // D = f32, A = B = f16 (0)
                               | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

struct __align__(8) Ctrl {
    uint64_t full[kStages];     // leader: both CTAs' stage bytes landed
    uint64_t empty[kStages];    // each CTA: the pair MMAs are done with the stage
    uint64_t ofull;             // leader: both CTAs' outlier k-block landed
    uint64_t oempty;            // each CTA: the P MMAs are done with the outlier slot
    uint64_t acc_full[2];       // each CTA: the buffer holds the tile's int32 sums
    uint64_t acc_mid[2];        // leader: both CTAs' epilogues wrote fp32 into the buffer
    uint64_t acc_p[2];          // each CTA: P has been added to the buffer
    uint64_t acc_empty[2];      // leader: both CTAs' epilogues have read the buffer
    uint64_t drain;             // each CTA: every pair MMA has finished
    uint32_t tmem_base;
    uint32_t abort;
    uint32_t epi_abort[2];      // epilogue votes, one slot per tile parity
};

constexpr int kStoreBox = 32;                                    // Y staged in 32 x 32 fp16 boxes
constexpr size_t kStoreBufBytes = kStoreBox * kStoreBox * 2;     // 2 KB
constexpr size_t kSmemTiles = (size_t)kStages * (kStageA + kStageB);
constexpr size_t kOffOut = kSmemTiles;                           // Xo slot, then Wo slot
constexpr size_t kOffStage = kOffOut + 2 * (size_t)kOStage;      // [kEpiWarps][kBoxes] store boxes
constexpr size_t kOffCtrl = kOffStage + (size_t)kEpiWarps * kBoxes * kStoreBufBytes;
constexpr size_t kOffScb = kOffCtrl + 256;
constexpr size_t kOffBias = kOffScb + BN * 4;
constexpr size_t kOffZb = kOffBias + BN * 4;   // zeropoint mode: zp_b of the tile's columns
constexpr size_t kOffSb = kOffZb + BN * 4;     // zeropoint mode: code sums of the tile's columns
constexpr size_t kSmemUsed = kOffSb + BN * 4;
constexpr size_t kSmemBytes = 1024 /*align slack*/ + kSmemUsed;
static_assert(sizeof(Ctrl) <= 256, "control block");
static_assert(kOffOut % 1024 == 0 && kOStage % 1024 == 0, "swizzle atoms need aligned slots");
static_assert(kSmemBytes <= 232448, "shared memory budget");

__device__ __forceinline__ void epi_sync() {
    asm volatile("bar.sync %0, %1;" ::"r"(kEpiBarrier), "r"(kEpiThreads) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_flag(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Hand a TMEM buffer back to the leader's MMA warp (or signal the leader's
// acc_mid barrier): one arrival per epilogue warp of each CTA.
__device__ __forceinline__ void arrive_leader(Ctrl *ctrl, uint64_t *bar, uint32_t rank) {
    const uint32_t b = smem_u32(bar);
    if (rank == 0) mbar_arrive(b); else mbar_arrive_cluster(mapa_shared(b, 0));
}

// Partial sums of a split tile's tail, written so that each store of a
// warp covers 512 contiguous bytes: int4 (v) of chunk cc of lane l of
// epilogue warp ew sits at slot[((ew * kEpiChunks + cc / 32) * 8 + v) * 32 + l]. The
// head reads them back with the same warp and lane, which own the same rows
// and columns in both CTAs' epilogues.
__device__ __forceinline__ void epilogue_store_partial(uint32_t tmem, uint32_t lane_base, int buf, int hcol, int ew,
                                                       int lane, uint32_t rank, Ctrl *ctrl, int4 *slot) {
    const uint32_t col0 = (uint32_t)(buf * 256 + hcol * kEpiCols);
    int4 *dst = slot + (size_t)ew * kEpiChunks * 8 * 32 + lane;
    for (int cc = 0; cc < kEpiCols; cc += 32) {
        uint32_t acc[32];
        tmem_ld_32x32b_x32(tmem + lane_base + col0 + cc, acc);
        tmem_ld_wait();
        if (cc == kEpiCols - 32) {
            tc_fence_before();
            if (lane == 0) arrive_leader(ctrl, &ctrl->acc_empty[buf], rank);
        }
#pragma unroll
        for (int v = 0; v < 8; ++v)
            __stcg(dst + ((cc >> 5) * 8 + v) * 32,
                   make_int4((int)acc[4 * v], (int)acc[4 * v + 1], (int)acc[4 * v + 2], (int)acc[4 * v + 3]));
    }
}

// Head of a split tile: add the tail's int32 sums of this warp's chunk cc
// (exact), read in the layout epilogue_store_partial wrote.
__device__ __forceinline__ void add_partial(uint32_t (&acc)[32], const int4 *part, int cc) {
    if (!part) return;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
        const int4 t = __ldcg(part + ((cc >> 5) * 8 + v) * 32);
        acc[4 * v] += (uint32_t)t.x;
        acc[4 * v + 1] += (uint32_t)t.y;
        acc[4 * v + 2] += (uint32_t)t.z;
        acc[4 * v + 3] += (uint32_t)t.w;
    }
}

// acc (int32 sums of 32 columns, plus the tail's partial sums if any) ->
// fp32 C * rs * SCB[j] + bias[j], in place as bit patterns, two columns per
// packed fp32x2 operation (each lane rounds like fmaf/fmul).
__device__ __forceinline__ void dequant32(uint32_t (&acc)[32], float rs, const float *s_scb, const float *s_bias,
                                          const int4 *part, int cc) {
    add_partial(acc, part, cc);
    const float2 rs2 = make_float2(rs, rs);
    const float4 *sc4 = reinterpret_cast<const float4 *>(s_scb);
    const float4 *bi4 = reinterpret_cast<const float4 *>(s_bias);
#pragma unroll
    for (int v = 0; v < 8; ++v) {
        const float4 sc = sc4[v], bi = bi4[v];
        const float2 c01 = __fmul2_rn(make_float2((float)(int32_t)acc[4 * v], (float)(int32_t)acc[4 * v + 1]), rs2);
        const float2 c23 = __fmul2_rn(make_float2((float)(int32_t)acc[4 * v + 2], (float)(int32_t)acc[4 * v + 3]), rs2);
        const float2 y01 = __ffma2_rn(c01, make_float2(sc.x, sc.y), make_float2(bi.x, bi.y));
        const float2 y23 = __ffma2_rn(c23, make_float2(sc.z, sc.w), make_float2(bi.z, bi.w));
        acc[4 * v] = __float_as_uint(y01.x);
        acc[4 * v + 1] = __float_as_uint(y01.y);
        acc[4 * v + 2] = __float_as_uint(y23.x);
        acc[4 * v + 3] = __float_as_uint(y23.y);
    }
}

// Zeropoint mode: acc (int32 sums A.B of 32 columns, plus the tail's partial
// sums if any) -> fp32 (C + zb_j * ta + za * sb_j) * inv_a * inv_b_j + bias_j,
// the unrolled (A + zp_a)(B + zp_b) product of "8-bit Data Types and
// Quantization" (zeropoint quantization) with ta = sa + K * za. The
// correction is added in int64 (exact), then converted to fp32 once.
__device__ __forceinline__ void dequant32_zp(uint32_t (&acc)[32], float inv_a, int64_t ta, int32_t za,
                                             const float *s_invb, const float *s_bias, const int32_t *s_zb,
                                             const int32_t *s_sb, const int4 *part, int cc) {
    add_partial(acc, part, cc);
    const float4 *ib4 = reinterpret_cast<const float4 *>(s_invb);
    const float4 *bi4 = reinterpret_cast<const float4 *>(s_bias);
    const int4 *zb4 = reinterpret_cast<const int4 *>(s_zb);
    const int4 *sb4 = reinterpret_cast<const int4 *>(s_sb);
#pragma unroll
    for (int v = 0; v < 8; ++v) {
        const float4 ib = ib4[v], bi = bi4[v];
        const int4 zb = zb4[v], sb = sb4[v];
        const float ibv[4] = {ib.x, ib.y, ib.z, ib.w}, biv[4] = {bi.x, bi.y, bi.z, bi.w};
        const int32_t zbv[4] = {zb.x, zb.y, zb.z, zb.w}, sbv[4] = {sb.x, sb.y, sb.z, sb.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int64_t c = (int64_t)(int32_t)acc[4 * v + e] + (int64_t)zbv[e] * ta + (int64_t)za * sbv[e];
            acc[4 * v + e] = __float_as_uint(__fmaf_rn(__fmul_rn(__ll2float_rn(c), inv_a), ibv[e], biv[e]));
        }
    }
}

// fp32 (bit patterns) -> fp16, staged in the warp's next 32 x 32 box in shared
// memory (64-byte swizzle: 16-byte chunk i of row r sits at chunk
// i ^ ((r >> 1) & 3), which keeps the four stores of each row conflict-free)
// and handed to the TMA engine. Rows and columns past M and N are clipped by it.
// Y is written once and never read here, so its lines go into L2 as
// evict-first: on the 8192 x 12288 x 36864 product this kept more of the A
// and B panels that later tiles read again, and DRAM reads per launch fell
// from 3.2 to 2.6 GB.
__device__ __forceinline__ void store32(const uint32_t (&y)[32], uint8_t *s_stage, int ew, int &sbuf, int lane,
                                        const CUtensorMap *tmY, int32_t x, int32_t yrow) {
    uint32_t packed[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        __half2 h = __float22half2_rn(make_float2(__uint_as_float(y[2 * k]), __uint_as_float(y[2 * k + 1])));
        packed[k] = *reinterpret_cast<uint32_t *>(&h);
    }
    if (lane == 0) {  // this box's previous store has read it
        if constexpr (kBoxes == 2) bulk_wait_read_1();
        else bulk_wait_read_0();
    }
    __syncwarp();
    uint8_t *box = s_stage + (size_t)(ew * kBoxes + sbuf) * kStoreBufBytes;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        *reinterpret_cast<uint4 *>(box + lane * 64 + ((i ^ ((lane >> 1) & 3)) * 16)) =
            make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d_hint(tmY, smem_u32(box), x, yrow, l2_policy_evict_first());
        bulk_commit_group();
    }
    sbuf = kBoxes == 2 ? sbuf ^ 1 : 0;
}

template <bool kZp>
__global__ void __launch_bounds__(kThreads, 1)
gemm_i8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmXo, const __grid_constant__ CUtensorMap tmWo,
               const __grid_constant__ CUtensorMap tmY, const GemmArgs a, const int num_m_tiles,
               const int num_tiles) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + kStages * kStageA;
    uint8_t *sXo = smem + kOffOut;
    uint8_t *sWo = smem + kOffOut + kOStage;
    Ctrl *ctrl = reinterpret_cast<Ctrl *>(smem + kOffCtrl);
    float *s_scb = reinterpret_cast<float *>(smem + kOffScb);
    float *s_bias = reinterpret_cast<float *>(smem + kOffBias);
    int32_t *s_zb = reinterpret_cast<int32_t *>(smem + kOffZb);
    int32_t *s_sb = reinterpret_cast<int32_t *>(smem + kOffSb);
    uint8_t *s_stage = smem + kOffStage;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();          // 0: leader, 1: follower
    const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
    const int nkb = (int)ceil_div(a.K, 128);
    const bool sk_on = a.sk_partial && a.sk_flags && num_pairs <= kSkMaxPairs;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&ctrl->full[s]), 1);
            mbar_init(smem_u32(&ctrl->empty[s]), 1);
        }
        mbar_init(smem_u32(&ctrl->ofull), 1);
        mbar_init(smem_u32(&ctrl->oempty), 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&ctrl->acc_full[b]), 1);
            mbar_init(smem_u32(&ctrl->acc_mid[b]), 2 * kEpiWarps);
            mbar_init(smem_u32(&ctrl->acc_p[b]), 1);
            mbar_init(smem_u32(&ctrl->acc_empty[b]), 2 * kEpiWarps);
        }
        mbar_init(smem_u32(&ctrl->drain), 1);
        ctrl->abort = 0;
        ctrl->epi_abort[0] = ctrl->epi_abort[1] = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (threadIdx.x == 32) {
        tma_prefetch(&tmA);
        tma_prefetch(&tmB);
        if (!a.C32) tma_prefetch(&tmY);
        tma_prefetch(&tmXo);
        tma_prefetch(&tmWo);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(&ctrl->tmem_base), kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers exist before any cross-CTA signal
    tc_fence_after();
    // Everything above touches only this CTA pair; from here on the kernel
    // reads what the quantize pass wrote (launched with programmatic stream
    // serialization, the prologue overlaps the end of that pass).
    grid_dep_wait();
    int n_out = (!kZp && a.n_outliers && a.Xo && a.Wo && !a.C32) ? *a.n_outliers : 0;
    if (!IN_BOUNDS(n_out >= 0 && n_out <= a.kcap, a.status)) n_out = 0;
    const int n_okb = (n_out + kOkb - 1) / kOkb;       // outlier k-blocks per tile
    const int n_mma_o = (n_out + 15) >> 4;             // fp16 MMAs of K = 16 per tile
    const uint32_t tmem = ctrl->tmem_base;
    volatile uint32_t *abort_flag = &ctrl->abort;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------- TMA producer --
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            // Outlier k-blocks go out in schedule order, for every segment
            // that finishes a tile (not for tails), once the segment's int8
            // k-blocks are all issued and the slot is free; waiting for a
            // ring stage never blocks them.
            TileSched tsp(num_tiles, nkb, nkb, num_pairs, pair, sk_on);
            Seg gp;
            int p_avail = 0, p_done = 0, okb = 0;
            bool have_gp = false;
            uint32_t o_issued = 0;
            auto pump = [&](bool block) {
                while (p_done < p_avail && !*abort_flag) {
                    if (!have_gp) {
                        do { have_gp = tsp.next(gp); } while (have_gp && gp.tail);
                        if (!have_gp) return;
                    }
                    const uint32_t eb = smem_u32(&ctrl->oempty);
                    const uint32_t par = (o_issued & 1u) ^ 1u;
                    if (block) {
                        if (!mbar_wait_bounded(eb, par, kWaitLimitNs)) {
                            *abort_flag = 1;
                            record_timeout(a.status);
                            return;
                        }
                    } else if (!mbar_try_wait(eb, par)) {
                        return;
                    }
                    const uint32_t fb = smem_u32(&ctrl->ofull);
                    if (rank == 0) mbar_arrive_expect_tx(fb, kOTxBytes);
                    const uint32_t fb_leader = mapa_shared(fb, 0);
                    int tm, tn;
                    tile_mn(gp.tile, num_m_tiles, num_tiles, tm, tn);
                    const int32_t m0 = tm * BM + (int32_t)rank * kCtaRows;
                    const int32_t n0 = tn * BN + (int32_t)rank * kCtaRows;
                    tma_load_2d_pair(smem_u32(sXo), &tmXo, fb_leader, okb * kOkb, m0);
                    tma_load_2d_pair(smem_u32(sWo), &tmWo, fb_leader, okb * kOkb, n0);
                    ++o_issued;
                    if (++okb == n_okb) {
                        okb = 0;
                        ++p_done;
                        have_gp = false;
                    }
                }
            };
            TileSched ts(num_tiles, nkb, nkb, num_pairs, pair, sk_on);
            Seg g;
            while (!*abort_flag && ts.next(g)) {
                int tm, tn;
                tile_mn(g.tile, num_m_tiles, num_tiles, tm, tn);
                const int32_t m0 = tm * BM + (int32_t)rank * kCtaRows;
                const int32_t n0 = tn * BN + (int32_t)rank * kCtaRows;
                for (int kb = g.kb0; kb < g.kb1; ++kb) {
                    if (*abort_flag) break;
                    const uint32_t eb = smem_u32(&ctrl->empty[stage]);
                    if (!mbar_try_wait(eb, phase ^ 1u)) {
                        const uint64_t t0 = globaltimer_ns();
                        bool ok = true;
                        while (!mbar_try_wait(eb, phase ^ 1u)) {
                            if (n_okb) pump(false);
                            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                                ok = false;
                                break;
                            }
                        }
                        if (!ok) {
                            *abort_flag = 1;
                            record_timeout(a.status);
                            break;
                        }
                    }
                    const uint32_t fb = smem_u32(&ctrl->full[stage]);
                    if (rank == 0) mbar_arrive_expect_tx(fb, kTxBytes);
                    const uint32_t fb_leader = mapa_shared(fb, 0);
                    tma_load_2d_pair(smem_u32(sA + stage * kStageA), &tmA, fb_leader, kb * 128, m0);
                    tma_load_4d_pair(smem_u32(sB + stage * kStageB), &tmB, fb_leader, 0, 0, kb,
                                     (int32_t)(n0 / kWBlockRows));
                    ++issued;
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
                if (n_okb && !g.tail) {
                    ++p_avail;
                    pump(false);
                }
            }
            if (n_okb) pump(true);
            // Do not leave while copies this thread started are in flight:
            // a stage (or the outlier slot) is free again once the pair MMAs
            // have consumed it.
            for (int u = max(0, issued - kStages); u < issued; ++u) {
                const int s = u % kStages;
                if (!mbar_wait_bounded(smem_u32(&ctrl->empty[s]), (uint32_t)((u / kStages) & 1), kWaitLimitNs)) {
                    record_timeout(a.status);
                    break;
                }
            }
            if (o_issued && !mbar_wait_bounded(smem_u32(&ctrl->oempty), (o_issued - 1u) & 1u, kWaitLimitNs))
                record_timeout(a.status);
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ----------------------------------------- MMA issuer (leader) --
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;  // local segment count
            uint32_t p_uses[2] = {0u, 0u};  // P passes per buffer so far
            uint32_t o_used = 0;            // outlier k-blocks consumed so far
            bool pend = false;              // a finished tile still waits for its P
            int pbuf = 0;
            // P of the pending tile: once both epilogues have written its fp32
            // values into the buffer, accumulate Xo . Wo^T onto them.
            auto issue_p = [&](bool block) {
                const uint32_t mb = smem_u32(&ctrl->acc_mid[pbuf]);
                const uint32_t par = p_uses[pbuf] & 1u;
                if (block) {
                    if (!mbar_wait_bounded(mb, par, kWaitLimitNs)) {
                        *abort_flag = 1;
                        record_timeout(a.status);
                        pend = false;
                        return;
                    }
                } else if (!mbar_try_wait(mb, par)) {
                    return;
                }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(pbuf * 256);
                for (int j = 0; j < n_okb; ++j) {
                    if (!mbar_wait_bounded(smem_u32(&ctrl->ofull), o_used & 1u, kWaitLimitNs)) {
                        *abort_flag = 1;
                        record_timeout(a.status);
                        pend = false;
                        return;
                    }
                    tc_fence_after();
                    const uint64_t da = sdesc_k_sw64(smem_u32(sXo));
                    const uint64_t db = sdesc_k_sw64(smem_u32(sWo));
                    for (int k = 0; k < 2 && 2 * j + k < n_mma_o; ++k)  // K = 16 fp16 = 32 bytes each
                        mma_f16_pair(d, da + 2 * k, db + 2 * k, kIdescF16, 1u);
                    mma_commit_pair(smem_u32(&ctrl->oempty), kPairMask);
                    ++o_used;
                }
                mma_commit_pair(smem_u32(&ctrl->acc_p[pbuf]), kPairMask);
                ++p_uses[pbuf];
                pend = false;
            };
            TileSched ts(num_tiles, nkb, nkb, num_pairs, pair, sk_on);
            Seg g;
            for (; !*abort_flag && ts.next(g); ++it) {
                const int buf = it & 1;
                const uint32_t use = (uint32_t)(it >> 1);
                if (!mbar_wait_bounded(smem_u32(&ctrl->acc_empty[buf]), (use & 1u) ^ 1u, kWaitLimitNs)) {
                    *abort_flag = 1;
                    record_timeout(a.status);
                    break;
                }
                tc_fence_after();
                const uint32_t d_i32 = tmem + (uint32_t)(buf * 256);
                for (int kb = g.kb0; kb < g.kb1; ++kb) {
                    if (*abort_flag) break;
                    if (!mbar_wait_bounded(smem_u32(&ctrl->full[stage]), phase, kWaitLimitNs)) {
                        *abort_flag = 1;
                        record_timeout(a.status);
                        break;
                    }
                    tc_fence_after();
                    const uint64_t da = sdesc_k_sw128(smem_u32(sA + stage * kStageA));
                    const uint64_t db = sdesc_k_sw128(smem_u32(sB + stage * kStageB));
#pragma unroll
                    for (int k = 0; k < 4; ++k)  // 4 x (K = 32 int8 = 32 bytes)
                        mma_i8_pair(d_i32, da + 2 * k, db + 2 * k, kIdescI8, (kb != g.kb0) || (k != 0));
                    mma_commit_pair(smem_u32(&ctrl->empty[stage]), kPairMask);
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                    if (pend) issue_p(false);
                }
                // lands in both CTAs when this segment's MMAs are done
                mma_commit_pair(smem_u32(&ctrl->acc_full[buf]), kPairMask);
                if (pend && !*abort_flag) issue_p(true);
                if (n_okb && !g.tail) {
                    pend = true;
                    pbuf = buf;
                }
            }
            if (pend && !*abort_flag) issue_p(true);
            // Nothing may still write either CTA's TMEM when it is freed.
            mma_commit_pair(smem_u32(&ctrl->drain), kPairMask);
        }
        if (lane == 0) {
            if (!mbar_wait_bounded(smem_u32(&ctrl->drain), 0, kWaitLimitNs)) record_timeout(a.status);
        }
    } else {
        // ---------------------------------------------------- epilogue --
        const int ew = warp - 2;                 // 0..7
        const int q = warp & 3;                  // TMEM lanes [32q, 32q + 32) are this warp's
        const int hcol = ew >> 2;                // columns [kEpiCols hcol, kEpiCols (hcol + 1))
        const int et = threadIdx.x - 64;         // 0 .. kEpiThreads - 1; thread et < BN stages column et
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        int sbuf = 0;  // which of the warp's two store boxes is next
        int it = 0;
        uint32_t p_uses[2] = {0u, 0u};
        TileSched ts(num_tiles, nkb, nkb, num_pairs, pair, sk_on);
        Seg g;
        for (; ts.next(g); ++it) {
            int tm, tn;
            tile_mn(g.tile, num_m_tiles, num_tiles, tm, tn);
            const int64_t m0 = (int64_t)tm * BM + rank * kCtaRows;
            const int64_t n0 = (int64_t)tn * BN;
            const int buf = it & 1;
            const uint32_t use = (uint32_t)(it >> 1);
            // Fetch this tile's column data (thread et owns column n0 + et)
            // and this thread's row scale while the MMAs are still running.
            const int64_t col = n0 + et;
            const bool col_ok = !a.C32 && et < BN && col < a.N;
            // (Zeropoint mode: 1 / nd_b, zp_b and the code sums per column;
            // 1 / nd_a, zp_a and sa + K zp_a for the row.)
            const float scb_v = col_ok ? (kZp ? 1.0f / a.SCB[col] : a.SCB[col]) : 0.f;
            const float bias_v = (col_ok && a.bias) ? __half2float(a.bias[col]) : 0.f;
            const int64_t row = m0 + q * 32 + lane;
            const bool row_ok = row < a.M;
            const float sca_v = (row_ok && a.SCA) ? (kZp ? 1.0f / a.SCA[row] : a.SCA[row]) : 0.f;
            int32_t zb_v = 0, sb_v = 0, za_v = 0;
            int64_t ta_v = 0;
            if constexpr (kZp) {
                if (col_ok) {
                    zb_v = a.ZB[col];
                    sb_v = a.SB[col];
                }
                if (row_ok) {
                    za_v = a.ZA[row];
                    ta_v = (int64_t)a.SA[row] + a.K * (int64_t)za_v;
                }
            }
            // Wait for the accumulator, then decide together whether to go
            // on: every epilogue warp votes before the barrier and reads the
            // same slot after it, so all of them leave the loop together.
            bool ok = mbar_wait_bounded(smem_u32(&ctrl->acc_full[buf]), use & 1u, kWaitLimitNs);
            if (!ok) record_timeout(a.status);
            ok = __all_sync(0xffffffffu, ok);
            volatile uint32_t *vote = &ctrl->epi_abort[it & 1];
            if (lane == 0 && (!ok || *abort_flag)) *vote = 1;
            // Stage this tile's column data (the previous tile's readers are done).
            epi_sync();
            if (*vote) {
                *abort_flag = 1;
                break;
            }
            if (!a.C32 && et < BN) {
                s_scb[et] = scb_v;
                s_bias[et] = bias_v;
                if constexpr (kZp) {
                    s_zb[et] = zb_v;
                    s_sb[et] = sb_v;
                }
            }
            epi_sync();
            tc_fence_after();
            const uint32_t col0 = (uint32_t)(buf * 256 + hcol * kEpiCols);
            if (g.tail) {
                // Tail of a split tile: hand the int32 sums to the head's pair.
                int4 *slot = reinterpret_cast<int4 *>(a.sk_partial) + (size_t)(pair * 2 + rank) * (kSkPartialBytes / 16);
                epilogue_store_partial(tmem, lane_base, buf, hcol, ew, lane, rank, ctrl, slot);
                __threadfence();
                epi_sync();
                if (et == 0) atomicExch(&a.sk_flags[pair * 2 + rank], 1u);
                continue;
            }
            const int4 *part = nullptr;
            if (g.head) {
                // Head of a split tile: the next pair wrote the tail's sums at
                // the start of its range; wait (bounded) until they are visible.
                const uint32_t *flag = &a.sk_flags[(pair + 1) * 2 + rank];
                if (et == 0) {
                    const uint64_t t0 = globaltimer_ns();
                    while (ld_acquire_flag(flag) == 0) {
                        if (globaltimer_ns() - t0 > kWaitLimitNs) {
                            record_timeout(a.status);
                            break;
                        }
                    }
                }
                epi_sync();
                part = reinterpret_cast<const int4 *>(a.sk_partial) +
                       (size_t)((pair + 1) * 2 + rank) * (kSkPartialBytes / 16) + (size_t)ew * kEpiChunks * 8 * 32 + lane;
            }
            const float rs = sca_v * (1.0f / 16129.0f);
            if (a.C32) {
                // Raw int32 sums (test entry): no scales, no outliers.
                for (int cc = 0; cc < kEpiCols; cc += 32) {
                    uint32_t acc[32];
                    tmem_ld_32x32b_x32(tmem + lane_base + col0 + cc, acc);
                    tmem_ld_wait();
                    if (cc == kEpiCols - 32) {
                        tc_fence_before();
                        if (lane == 0) arrive_leader(ctrl, &ctrl->acc_empty[buf], rank);
                    }
                    add_partial(acc, part, cc);
                    const int64_t c0 = n0 + hcol * kEpiCols + cc;
                    if (!row_ok || c0 >= a.N) continue;
                    int32_t *dst = a.C32 + row * a.N + c0;
#pragma unroll
                    for (int v = 0; v < 8; ++v)
                        if (c0 + 4 * v < a.N && IN_BOUNDS(row * a.N + c0 + 4 * v + 3 < a.M * a.N, a.status))
                            reinterpret_cast<int4 *>(dst)[v] = make_int4((int)acc[4 * v], (int)acc[4 * v + 1],
                                                                         (int)acc[4 * v + 2], (int)acc[4 * v + 3]);
                }
            } else if (n_okb) {
                // Pass 1: fp32 C * rs * SCB + bias back into the buffer.
                for (int cc = 0; cc < kEpiCols; cc += 32) {
                    uint32_t acc[32];
                    tmem_ld_32x32b_x32(tmem + lane_base + col0 + cc, acc);
                    tmem_ld_wait();
                    dequant32(acc, rs, s_scb + hcol * kEpiCols + cc, s_bias + hcol * kEpiCols + cc, part, cc);
                    tmem_st_32x32b_x32(tmem + lane_base + col0 + cc, acc);
                }
                tmem_st_wait();
                tc_fence_before();
                if (lane == 0) arrive_leader(ctrl, &ctrl->acc_mid[buf], rank);
                // The MMA warp adds P; all warps vote on the outcome together.
                bool pok = mbar_wait_bounded(smem_u32(&ctrl->acc_p[buf]), p_uses[buf] & 1u, kWaitLimitNs);
                if (!pok) record_timeout(a.status);
                ++p_uses[buf];
                pok = __all_sync(0xffffffffu, pok);
                if (lane == 0 && !pok) *vote = 1;
                epi_sync();
                if (*vote) {
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                // Pass 2: fp16 out.
                for (int cc = 0; cc < kEpiCols; cc += 32) {
                    uint32_t y[32];
                    tmem_ld_32x32b_x32(tmem + lane_base + col0 + cc, y);
                    tmem_ld_wait();
                    if (cc == kEpiCols - 32) {
                        tc_fence_before();
                        if (lane == 0) arrive_leader(ctrl, &ctrl->acc_empty[buf], rank);
                    }
                    if (n0 + hcol * kEpiCols + cc < a.N)
                        store32(y, s_stage, ew, sbuf, lane, &tmY, (int32_t)(n0 + hcol * kEpiCols + cc),
                                (int32_t)(m0 + q * 32));
                }
            } else {
                // No outliers: one pass.
                for (int cc = 0; cc < kEpiCols; cc += 32) {
                    uint32_t acc[32];
                    tmem_ld_32x32b_x32(tmem + lane_base + col0 + cc, acc);
                    tmem_ld_wait();
                    if (cc == kEpiCols - 32) {
                        tc_fence_before();
                        if (lane == 0) arrive_leader(ctrl, &ctrl->acc_empty[buf], rank);
                    }
                    if (n0 + hcol * kEpiCols + cc >= a.N) continue;  // whole chunk past the last column
                    const int sc = hcol * kEpiCols + cc;
                    if constexpr (kZp)
                        dequant32_zp(acc, sca_v, ta_v, za_v, s_scb + sc, s_bias + sc, s_zb + sc, s_sb + sc, part, cc);
                    else
                        dequant32(acc, rs, s_scb + sc, s_bias + sc, part, cc);
                    store32(acc, s_stage, ew, sbuf, lane, &tmY, (int32_t)(n0 + hcol * kEpiCols + cc),
                            (int32_t)(m0 + q * 32));
                }
            }
            if (g.head) {
                epi_sync();  // every warp has read the tail's sums
                if (et == 0) a.sk_flags[(pair + 1) * 2 + rank] = 0u;
            }
        }
        if (lane == 0) bulk_wait_all();  // every store of this warp has finished
    }

    // Teardown: the pair's peer must be done signalling this CTA's barriers
    // and its MMAs done with this CTA's TMEM before TMEM is freed and the CTA exits.
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

}  // namespace

// ----------------------------------------------------------- tensor maps --

namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}
}  // namespace

bool make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
              uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {pitch_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {
// CB in the blocked weight layout as a 4-D tensor (128 bytes, 32 rows,
// k-blocks, row blocks); a box of (128, 32, 1, 4) is one k-block of 128
// consecutive output channels, landing in shared memory exactly as a 128-row
// x 128-byte box of a row-major matrix would (same 128-byte swizzle).
bool make_map_wblocks(CUtensorMap *m, const int8_t *CB, int64_t N, int64_t K) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    const int64_t KB = wblocks_k(K), NB = ceil_div(N, kWBlockRows);
    cuuint64_t dims[4] = {(cuuint64_t)kWBlockCols, (cuuint64_t)kWBlockRows, (cuuint64_t)KB, (cuuint64_t)NB};
    cuuint64_t strides[3] = {(cuuint64_t)kWBlockCols, (cuuint64_t)kWBlockBytes, (cuuint64_t)(KB * kWBlockBytes)};
    cuuint32_t box[4] = {(cuuint32_t)kWBlockCols, (cuuint32_t)kWBlockRows, 1, kCtaRows / kWBlockRows};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<int8_t *>(CB), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int g_num_sms[64];  // resident CTA pairs per device

}  // namespace

cudaError_t launch_gemm_tc(const GemmArgs &a, cudaStream_t s) {
    CUtensorMap mA, mB, mXo, mWo;
    if (!make_map(&mA, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.CA, a.K, a.M, a.K, 128, kCtaRows) ||
        !make_map_wblocks(&mB, a.CB, a.N, a.K))
        return cudaErrorInvalidValue;
    if (a.Xo && a.Wo && a.n_outliers) {
        if (!make_map(&mXo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.Xo, a.kcap, a.M, a.kcap * 2, kOkb, kCtaRows,
                      CU_TENSOR_MAP_SWIZZLE_64B) ||
            !make_map(&mWo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.Wo, a.kcap, a.N, a.kcap * 2, kOkb, kCtaRows,
                      CU_TENSOR_MAP_SWIZZLE_64B))
            return cudaErrorInvalidValue;
    } else {
        mXo = mA;  // never read: |O| = 0 without outlier buffers
        mWo = mB;
    }
    CUtensorMap mY = mA;  // never read when the raw int32 sums are stored instead
    if (!a.C32 && !make_map(&mY, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.Y, a.N, a.M, a.N * 2, kStoreBox, kStoreBox,
                            CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    static std::once_flag attr_once[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    cudaError_t attr_err = cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;  // CTA pairs
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    std::call_once(attr_once[dev & 63], [&] {
        attr_err = cudaFuncSetAttribute(gemm_i8_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)kSmemBytes);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(gemm_i8_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            (int)kSmemBytes);
        if (attr_err != cudaSuccess) return;
        // How many CTA pairs can be resident at once (a pair needs two SMs of one GPC).
        cudaLaunchConfig_t q = cfg;
        q.gridDim = dim3(2, 1, 1);
        int clusters = 0;
        attr_err = cudaOccupancyMaxActiveClusters(&clusters, (void *)gemm_i8_kernel<false>, &q);
        g_num_sms[dev & 63] = clusters;
    });
    if (attr_err != cudaSuccess) return attr_err;
    const int num_m_tiles = (int)ceil_div(a.M, BM);
    const int64_t tiles = (int64_t)num_m_tiles * ceil_div(a.N, BN);
    const int pairs = g_num_sms[dev & 63] > 0 ? g_num_sms[dev & 63] : 74;
    const int grid_pairs = (int)std::min<int64_t>(tiles, pairs);
    GemmArgs b = a;
    if (!split_wanted(tiles, (int)ceil_div(a.K, 128), grid_pairs, g_split_mode.load(std::memory_order_relaxed))) {
        b.sk_partial = nullptr;
        b.sk_flags = nullptr;
    }
    cfg.gridDim = dim3(2 * (unsigned)grid_pairs, 1, 1);
    cfg.numAttrs = 2;  // and programmatic stream serialization
    if (a.ZB) {  // zeropoint mode: no outlier term
        if (!a.ZA || !a.SA || !a.SB || !a.SCA || !a.SCB || a.C32) return cudaErrorInvalidValue;
        b.n_outliers = nullptr;
        return cudaLaunchKernelEx(&cfg, gemm_i8_kernel<true>, mA, mB, mXo, mWo, mY, b, num_m_tiles, (int)tiles);
    }
    return cudaLaunchKernelEx(&cfg, gemm_i8_kernel<false>, mA, mB, mXo, mWo, mY, b, num_m_tiles, (int)tiles);
}

}  // namespace int8lt

// Test entry: the schedule as the GEMM walks it, enumerated on the host.
// Rows of 6 int32: pair, tile, kb0, kb1, head, tail.
extern "C" int int8lt_debug_gemm_schedule(int tiles, int nkb, int pairs, int mode, int32_t *out, int cap_rows) {
    if (tiles < 0 || nkb < 1 || pairs < 1 || mode < 0 || mode > 2 || (!out && cap_rows > 0)) return -1;
    const bool sk = int8lt::split_wanted(tiles, nkb, pairs, mode);
    int n = 0;
    for (int p = 0; p < pairs; ++p) {
        int8lt::TileSched ts(tiles, nkb, nkb, pairs, p, sk);
        int8lt::Seg g;
        while (ts.next(g)) {
            if (n < cap_rows) {
                int32_t *r = out + 6 * n;
                r[0] = p; r[1] = g.tile; r[2] = g.kb0; r[3] = g.kb1; r[4] = g.head; r[5] = g.tail;
            }
            ++n;
        }
    }
    return n;
}

extern "C" int int8lt_debug_tile_order(int num_m, int num_n, int32_t *out) {
    if (num_m < 1 || num_n < 1 || !out || (int64_t)num_m * num_n > (1 << 30)) return -1;
    const int tiles = num_m * num_n;
    for (int t = 0; t < tiles; ++t) {
        int m, n;
        int8lt::tile_mn(t, num_m, tiles, m, n);
        out[2 * t] = m;
        out[2 * t + 1] = n;
    }
    return tiles;
}

extern "C" int int8lt_set_gemm_split(int mode) {
    if (mode < 0 || mode > 2) return -1;
    return int8lt::g_split_mode.exchange(mode);
}
