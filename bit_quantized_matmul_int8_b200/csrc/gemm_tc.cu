// Prefill path of the LLM.int8() forward on sm_100a tensor cores.
//
// Computes, per 256 x 256 output tile,
//     Y = fp16( C * SCA[i] * SCB[j] / 127^2 + P + bias[j] )
//     C = CA . CB^T    int8 x int8 -> int32   ("Int8 Matrix Multiplication with
//                      16-bit Float Inputs and Outputs" and "Vector-wise
//                      Quantization", LLM.int8() paper summary)
//     P = Xo . Wo^T    fp16 x fp16 -> fp32    (the outlier columns, "The Core
//                      of LLM.int8(): Mixed-precision Decomposition")
// in one persistent kernel run by CTA pairs (clusters of 2 SMs). Each tile
// is computed by one pair with 2-SM tensor-core MMAs (tcgen05 cta_group::2):
// each CTA stages its own 128 rows of A and its own half (128 rows) of B,
// so per SM a 128 x 256 x 128 k-block needs 32 KB of operands instead of
// 48 KB, and a 6-deep ring of stages fits in shared memory.
//   warp 0     (both CTAs) TMA producer into a 6-stage ring; the loads of
//              both CTAs complete on the leader CTA's full barrier;
//   warp 1     (both CTAs) allocates the 512 tensor-memory columns; in the
//              leader it issues the pair MMAs and multicasts the commits;
//   warps 2-9  (both CTAs) epilogue on the CTA's 128 rows: tcgen05.ld the
//              accumulator, dequantize in fp32, add P and bias, and store fp16
//              through shared memory with TMA (32 x 32 boxes, double buffered
//              per warp), so the epilogue warps never wait on global stores.
// Outlier product, chosen on the device from |O| (no host sync):
//   |O| <= kEpiOutlierMax: two int32 accumulators of 256 columns (double
//       buffered: the epilogue of one tile overlaps the mainloop of the next)
//       and P on the CUDA cores in the epilogue, from the row's Xo values in
//       registers and the tile's Wo in shared memory; every fp16 x fp16
//       product is exact in fp32, as on the tensor cores;
//   |O| >  kEpiOutlierMax: one int32 accumulator (columns 0-255) and P as
//       tcgen05 kind::f16 MMAs into an fp32 accumulator (columns 256-511).
// Every wait is bounded (kWaitLimitNs); a wait that runs out sets the
// workspace status word and the kernel winds down without touching Y.
#include <algorithm>
#include <mutex>

#include "int8lt_internal.cuh"

namespace int8lt {

namespace {

constexpr int BM = 256, BN = 256;         // pair tile
constexpr int kCtaRows = 128;             // rows of A (and of B) staged per CTA
constexpr int kStages = 5;
constexpr int kStageA = kCtaRows * 128;   // bytes: 128 rows x 128 B
constexpr int kStageB = kCtaRows * 128;   // bytes: 128 rows x 128 B (half of N)
constexpr uint32_t kTxBytes = 2 * (kStageA + kStageB);  // both CTAs, counted by the leader
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kThreads = 64 + kEpiThreads;
constexpr uint32_t kTmemCols = 512;
constexpr int kEpiOutlierMax = 24;  // largest |O| whose product runs on the CUDA cores
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
    uint64_t acc_full[2];       // each CTA: the accumulator buffer is complete
    uint64_t acc_empty[2];      // leader: both CTAs' epilogues have read the buffer
    uint64_t drain;             // each CTA: every pair MMA has finished
    uint32_t tmem_base;
    uint32_t abort;
    uint32_t epi_abort[2];      // epilogue votes, one slot per tile parity
};

constexpr int kStoreBox = 32;                                    // Y staged in 32 x 32 fp16 boxes
constexpr size_t kStoreBufBytes = kStoreBox * kStoreBox * 2;     // 2 KB
constexpr size_t kSmemTiles = (size_t)kStages * (kStageA + kStageB);
constexpr size_t kOffStage = kSmemTiles;                         // [kEpiWarps][2] store boxes
constexpr size_t kOffCtrl = kOffStage + (size_t)kEpiWarps * 2 * kStoreBufBytes;
constexpr size_t kOffScb = kOffCtrl + 256;
constexpr size_t kOffBias = kOffScb + BN * 4;
constexpr size_t kOffWo = kOffBias + BN * 4;                     // fp32 [kEpiOutlierMax][BN]
constexpr size_t kSmemUsed = kOffWo + (size_t)kEpiOutlierMax * BN * 4;
constexpr size_t kSmemBytes = 1024 /*align slack*/ + kSmemUsed;
static_assert(sizeof(Ctrl) <= 256, "control block");
static_assert(kSmemBytes <= 232448, "shared memory budget");

__device__ __forceinline__ void epi_sync() {
    asm volatile("bar.sync %0, %1;" ::"r"(kEpiBarrier), "r"(kEpiThreads) : "memory");
}

// Epilogue of one tile for one warp: 32 rows (TMEM lanes) x 128 columns, in
// chunks of 32. kMmaOut: the outlier product P is in TMEM (fp32, 256 columns
// after the int32 sums); otherwise it is computed here from Xo and Wo.
template <bool kMmaOut>
__device__ __forceinline__ void epilogue_tile(const GemmArgs &a, uint32_t tmem, uint32_t lane_base, int buf, int hcol,
                                              int q, int lane, int ew, uint32_t rank, bool row_ok, int64_t row,
                                              float rs, int64_t n0, int64_t m0, int n_out, const float *s_scb,
                                              const float *s_bias, const float *s_wo, uint8_t *s_stage, int &sbuf,
                                              Ctrl *ctrl, const CUtensorMap *tmY,
                                              const uint4 (&xo_v)[kEpiOutlierMax / 8]) {
    const bool cuda_out = !kMmaOut && n_out > 0;
    // This row's outlier activations (CUDA-core outlier product), fp16.
    const __half *xo = reinterpret_cast<const __half *>(xo_v);
    const uint32_t col0 = (uint32_t)(buf * 256 + hcol * 128);
    for (int cc = 0; cc < 128; cc += 32) {
        const int c = hcol * 128 + cc;  // column within the tile
        uint32_t acc[32], po[32];
        tmem_ld_32x32b_x32(tmem + lane_base + col0 + cc, acc);
        if constexpr (kMmaOut) tmem_ld_32x32b_x32(tmem + lane_base + 256 + col0 + cc, po);
        tmem_ld_wait();
        if (cc == 96) {
            // Every TMEM read of this buffer is done: hand it back to
            // the leader's MMA warp.
            tc_fence_before();
            if (lane == 0) {
                const uint32_t eb = smem_u32(&ctrl->acc_empty[buf]);
                if (rank == 0) mbar_arrive(eb); else mbar_arrive_cluster(mapa_shared(eb, 0));
            }
        }
        if (n0 + c >= a.N) continue;  // whole chunk past the last column
        if (a.C32) {
            if (!row_ok) continue;
            int32_t *dst = a.C32 + row * a.N + n0 + c;
#pragma unroll
            for (int v = 0; v < 8; ++v)
                if (n0 + c + 4 * v < a.N)
                    reinterpret_cast<int4 *>(dst)[v] =
                        make_int4((int)acc[4 * v], (int)acc[4 * v + 1], (int)acc[4 * v + 2], (int)acc[4 * v + 3]);
            continue;
        }
        // y = C * SCA / 127^2 * SCB + bias (+ P), two columns per
        // packed fp32x2 operation (each lane rounds like fmaf/fmul).
        float2 y2[16];
        const float2 rs2 = make_float2(rs, rs);
        const float4 *sc4 = reinterpret_cast<const float4 *>(s_scb + c);
        const float4 *bi4 = reinterpret_cast<const float4 *>(s_bias + c);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const float4 sc = sc4[v], bi = bi4[v];
            const float2 c01 = __fmul2_rn(make_float2((float)(int32_t)acc[4 * v], (float)(int32_t)acc[4 * v + 1]), rs2);
            const float2 c23 =
                __fmul2_rn(make_float2((float)(int32_t)acc[4 * v + 2], (float)(int32_t)acc[4 * v + 3]), rs2);
            y2[2 * v] = __ffma2_rn(c01, make_float2(sc.x, sc.y), make_float2(bi.x, bi.y));
            y2[2 * v + 1] = __ffma2_rn(c23, make_float2(sc.z, sc.w), make_float2(bi.z, bi.w));
        }
        if constexpr (kMmaOut) {
#pragma unroll
            for (int k = 0; k < 16; ++k)
                y2[k] = __fadd2_rn(y2[k], make_float2(__uint_as_float(po[2 * k]), __uint_as_float(po[2 * k + 1])));
        }
        if (!kMmaOut && cuda_out) {
#pragma unroll
            for (int t = 0; t < (kMmaOut ? 1 : kEpiOutlierMax); ++t) {
                if (t >= n_out) break;  // uniform across the CTA
                const float xt = __half2float(xo[t]);
                const float2 xv = make_float2(xt, xt);
                const float4 *w4 = reinterpret_cast<const float4 *>(s_wo + t * BN + c);
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    const float4 wv = w4[v];
                    y2[2 * v] = __ffma2_rn(xv, make_float2(wv.x, wv.y), y2[2 * v]);
                    y2[2 * v + 1] = __ffma2_rn(xv, make_float2(wv.z, wv.w), y2[2 * v + 1]);
                }
            }
        }
        uint32_t packed[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            __half2 h = __float22half2_rn(y2[k]);
            packed[k] = *reinterpret_cast<uint32_t *>(&h);
        }
        // Stage the warp's 32 x 32 box in shared memory (64-byte swizzle:
        // 16-byte chunk i of row r sits at chunk i ^ ((r >> 1) & 3), which
        // keeps the four stores of each row conflict-free) and hand it to
        // the TMA engine. Rows and columns past M and N are clipped by it.
        if (lane == 0) bulk_wait_read_1();  // this buffer's previous store has read it
        __syncwarp();
        uint8_t *box = s_stage + (size_t)(ew * 2 + sbuf) * kStoreBufBytes;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *reinterpret_cast<uint4 *>(box + lane * 64 + ((i ^ ((lane >> 1) & 3)) * 16)) =
                make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(tmY, smem_u32(box), (int32_t)(n0 + c), (int32_t)(m0 + q * 32));
            bulk_commit_group();
        }
        sbuf ^= 1;
    }
}

__global__ void __launch_bounds__(kThreads, 1)
gemm_i8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmXo, const __grid_constant__ CUtensorMap tmWo,
               const __grid_constant__ CUtensorMap tmY, const GemmArgs a, const int num_m_tiles,
               const int num_tiles) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + kStages * kStageA;
    Ctrl *ctrl = reinterpret_cast<Ctrl *>(smem + kOffCtrl);
    float *s_scb = reinterpret_cast<float *>(smem + kOffScb);
    float *s_bias = reinterpret_cast<float *>(smem + kOffBias);
    float *s_wo = reinterpret_cast<float *>(smem + kOffWo);
    uint8_t *s_stage = smem + kOffStage;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();          // 0: leader, 1: follower
    const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
    const int nkb = (int)ceil_div(a.K, 128);
    const int n_out = a.n_outliers ? *a.n_outliers : 0;
    const bool mma_out = n_out > kEpiOutlierMax;       // outlier product on the tensor cores
    const int nbuf = mma_out ? 1 : 2;                  // accumulator buffers in TMEM
    const int n_mma_o = mma_out ? (n_out + 15) >> 4 : 0;   // fp16 MMAs of K = 16
    const int nkb_o = mma_out ? (n_out + 63) >> 6 : 0;     // fp16 k-blocks of 64
    const int total_kb = nkb + nkb_o;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&ctrl->full[s]), 1);
            mbar_init(smem_u32(&ctrl->empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&ctrl->acc_full[b]), 1);
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
        if (mma_out) {
            tma_prefetch(&tmXo);
            tma_prefetch(&tmWo);
        }
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(&ctrl->tmem_base), kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers exist before any cross-CTA signal
    tc_fence_after();
    const uint32_t tmem = ctrl->tmem_base;
    volatile uint32_t *abort_flag = &ctrl->abort;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------- TMA producer --
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            for (int tile = pair; tile < num_tiles && !*abort_flag; tile += num_pairs) {
                const int32_t m0 = (tile % num_m_tiles) * BM + (int32_t)rank * kCtaRows;
                const int32_t n0 = (tile / num_m_tiles) * BN + (int32_t)rank * kCtaRows;
                for (int kb = 0; kb < total_kb; ++kb) {
                    if (*abort_flag) break;
                    if (!mbar_wait_bounded(smem_u32(&ctrl->empty[stage]), phase ^ 1u, kWaitLimitNs)) {
                        *abort_flag = 1;
                        record_timeout(a.status);
                        break;
                    }
                    const uint32_t fb = smem_u32(&ctrl->full[stage]);
                    if (rank == 0) mbar_arrive_expect_tx(fb, kTxBytes);
                    const uint32_t fb_leader = mapa_shared(fb, 0);
                    if (kb < nkb) {
                        tma_load_2d_pair(smem_u32(sA + stage * kStageA), &tmA, fb_leader, kb * 128, m0);
                        tma_load_2d_pair(smem_u32(sB + stage * kStageB), &tmB, fb_leader, kb * 128, n0);
                    } else {
                        const int ko = (kb - nkb) * 64;
                        tma_load_2d_pair(smem_u32(sA + stage * kStageA), &tmXo, fb_leader, ko, m0);
                        tma_load_2d_pair(smem_u32(sB + stage * kStageB), &tmWo, fb_leader, ko, n0);
                    }
                    ++issued;
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
            }
            // Do not leave while copies this thread started are in flight:
            // a stage is free again once the pair MMAs have consumed it.
            for (int u = max(0, issued - kStages); u < issued; ++u) {
                const int s = u % kStages;
                if (!mbar_wait_bounded(smem_u32(&ctrl->empty[s]), (uint32_t)((u / kStages) & 1), kWaitLimitNs)) {
                    record_timeout(a.status);
                    break;
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ----------------------------------------- MMA issuer (leader) --
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;  // local tile count
            for (int tile = pair; tile < num_tiles && !*abort_flag; tile += num_pairs, ++it) {
                const int buf = it % nbuf;
                const uint32_t use = (uint32_t)(it / nbuf);
                if (!mbar_wait_bounded(smem_u32(&ctrl->acc_empty[buf]), (use & 1u) ^ 1u, kWaitLimitNs)) {
                    *abort_flag = 1;
                    record_timeout(a.status);
                    break;
                }
                tc_fence_after();
                const uint32_t d_i32 = tmem + (uint32_t)(buf * 256);
                const uint32_t d_f32 = tmem + 256;
                for (int kb = 0; kb < total_kb; ++kb) {
                    if (*abort_flag) break;
                    if (!mbar_wait_bounded(smem_u32(&ctrl->full[stage]), phase, kWaitLimitNs)) {
                        *abort_flag = 1;
                        record_timeout(a.status);
                        break;
                    }
                    tc_fence_after();
                    const uint64_t da = sdesc_k_sw128(smem_u32(sA + stage * kStageA));
                    const uint64_t db = sdesc_k_sw128(smem_u32(sB + stage * kStageB));
                    if (kb < nkb) {
#pragma unroll
                        for (int k = 0; k < 4; ++k)  // 4 x (K = 32 int8 = 32 bytes)
                            mma_i8_pair(d_i32, da + 2 * k, db + 2 * k, kIdescI8, (kb | k) != 0);
                    } else {
                        const int kbo = kb - nkb;
                        const int nk = min(4, n_mma_o - kbo * 4);
                        for (int k = 0; k < nk; ++k)  // K = 16 fp16 = 32 bytes each
                            mma_f16_pair(d_f32, da + 2 * k, db + 2 * k, kIdescF16, (kbo | k) != 0);
                    }
                    mma_commit_pair(smem_u32(&ctrl->empty[stage]), kPairMask);
                    if (++stage == kStages) { stage = 0; phase ^= 1u; }
                }
                // lands in both CTAs when this tile's MMAs are done
                mma_commit_pair(smem_u32(&ctrl->acc_full[buf]), kPairMask);
            }
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
        const int hcol = ew >> 2;                // columns [128 hcol, 128 hcol + 128)
        const int et = threadIdx.x - 64;         // 0..255
        const uint32_t lane_base = (uint32_t)(q * 32) << 16;
        const bool cuda_out = !mma_out && n_out > 0;
        int sbuf = 0;  // which of the warp's two store boxes is next
        int it = 0;
        for (int tile = pair; tile < num_tiles; tile += num_pairs, ++it) {
            const int64_t m0 = (int64_t)(tile % num_m_tiles) * BM + rank * kCtaRows;
            const int64_t n0 = (int64_t)(tile / num_m_tiles) * BN;
            const int buf = it % nbuf;
            const uint32_t use = (uint32_t)(it / nbuf);
            // Fetch this tile's column data (thread et owns column n0 + et)
            // and this thread's row data into registers while the MMAs are
            // still running: 16-byte loads, all issued before any wait.
            const int64_t col = n0 + et;
            const bool col_ok = !a.C32 && col < a.N;
            const float scb_v = col_ok ? a.SCB[col] : 0.f;
            const float bias_v = (col_ok && a.bias) ? __half2float(a.bias[col]) : 0.f;
            const int64_t row = m0 + q * 32 + lane;
            const bool row_ok = row < a.M;
            const float sca_v = (row_ok && a.SCA) ? a.SCA[row] : 0.f;
            uint4 wo_v[kEpiOutlierMax / 8], xo_v[kEpiOutlierMax / 8];
#pragma unroll
            for (int v = 0; v < kEpiOutlierMax / 8; ++v) {
                const bool need = cuda_out && 8 * v < n_out;
                wo_v[v] = (need && col_ok) ? *reinterpret_cast<const uint4 *>(a.Wo + col * a.kcap + 8 * v)
                                           : make_uint4(0, 0, 0, 0);
                xo_v[v] = (need && row_ok) ? *reinterpret_cast<const uint4 *>(a.Xo + row * a.kcap + 8 * v)
                                           : make_uint4(0, 0, 0, 0);
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
            if (!a.C32) {
                s_scb[et] = scb_v;
                s_bias[et] = bias_v;
                if (cuda_out) {
                    const __half *wh = reinterpret_cast<const __half *>(wo_v);
#pragma unroll
                    for (int t = 0; t < kEpiOutlierMax; ++t)
                        if (t < n_out) s_wo[t * BN + et] = __half2float(wh[t]);
                }
            }
            epi_sync();
            tc_fence_after();
            const float rs = sca_v * (1.0f / 16129.0f);
            if (mma_out)
                epilogue_tile<true>(a, tmem, lane_base, buf, hcol, q, lane, ew, rank, row_ok, row, rs, n0, m0, n_out,
                                    s_scb, s_bias, s_wo, s_stage, sbuf, ctrl, &tmY, xo_v);
            else
                epilogue_tile<false>(a, tmem, lane_base, buf, hcol, q, lane, ew, rank, row_ok, row, rs, n0, m0, n_out,
                                     s_scb, s_bias, s_wo, s_stage, sbuf, ctrl, &tmY, xo_v);
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

// ----------------------------------------------------------- tensor maps --

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

// 2-D row-major map: `inner` elements per row (contiguous), `outer` rows,
// row pitch `pitch_bytes`; box of box_inner x box_outer; 128-byte swizzle;
// out-of-range elements read as zero.
bool make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
              uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer,
              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
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

int g_num_sms[64];  // resident CTA pairs per device

}  // namespace

cudaError_t launch_gemm_tc(const GemmArgs &a, cudaStream_t s) {
    CUtensorMap mA, mB, mXo, mWo;
    if (!make_map(&mA, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.CA, a.K, a.M, a.K, 128, kCtaRows) ||
        !make_map(&mB, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.CB, a.K, a.N, a.K, 128, kCtaRows))
        return cudaErrorInvalidValue;
    if (a.Xo && a.Wo && a.n_outliers) {
        if (!make_map(&mXo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.Xo, a.kcap, a.M, a.kcap * 2, 64, kCtaRows) ||
            !make_map(&mWo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.Wo, a.kcap, a.N, a.kcap * 2, 64, kCtaRows))
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
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;  // CTA pairs
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    std::call_once(attr_once[dev & 63], [&] {
        attr_err = cudaFuncSetAttribute(gemm_i8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
        if (attr_err != cudaSuccess) return;
        // How many CTA pairs can be resident at once (a pair needs two SMs of one GPC).
        cudaLaunchConfig_t q = cfg;
        q.gridDim = dim3(2, 1, 1);
        int clusters = 0;
        attr_err = cudaOccupancyMaxActiveClusters(&clusters, (void *)gemm_i8_kernel, &q);
        g_num_sms[dev & 63] = clusters;
    });
    if (attr_err != cudaSuccess) return attr_err;
    const int num_m_tiles = (int)ceil_div(a.M, BM);
    const int64_t tiles = (int64_t)num_m_tiles * ceil_div(a.N, BN);
    const int pairs = g_num_sms[dev & 63] > 0 ? g_num_sms[dev & 63] : 74;
    cfg.gridDim = dim3(2 * (unsigned)std::min<int64_t>(tiles, pairs), 1, 1);
    return cudaLaunchKernelEx(&cfg, gemm_i8_kernel, mA, mB, mXo, mWo, mY, a, num_m_tiles, (int)tiles);
}

}  // namespace int8lt
