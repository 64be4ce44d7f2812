// Prefill path of the LLM.int8() forward on sm_100a tensor cores.
//
// Computes, per 128 x 256 output tile,
//     Y = fp16( C * SCA[i] * SCB[j] / 127^2 + P + bias[j] )
//     C = CA . CB^T    int8 x int8 -> int32   ("Int8 Matrix Multiplication with
//                      16-bit Float Inputs and Outputs" and "Vector-wise
//                      Quantization", LLM.int8() paper summary)
//     P = Xo . Wo^T    fp16 x fp16 -> fp32    (the outlier columns, "The Core
//                      of LLM.int8(): Mixed-precision Decomposition")
// in one kernel:
//   warp 0     TMA producer: 128-byte-swizzled K-major tiles of CA/CB (int8,
//              128 wide) then Xo/Wo (fp16, 64 wide) into a 4-stage ring;
//   warp 1     allocates tensor memory and issues tcgen05.mma (kind::i8 into
//              TMEM columns [0,256), then kind::f16 into [256,512));
//   warps 2-5  epilogue: tcgen05.ld both accumulators, dequantize in fp32,
//              add P and bias, store fp16.
// The outlier count |O| is read from device memory, so no host sync happens
// between the quantize pass and this kernel. Every wait is bounded
// (kWaitLimitNs); a wait that runs out sets the workspace status word and
// the kernel winds down without touching Y.
#include <algorithm>
#include <mutex>

#include "int8lt_internal.cuh"

namespace int8lt {

namespace {

constexpr int BM = 128, BN = 256;
constexpr int kStages = 4;
constexpr int kStageA = BM * 128;  // bytes: 128 rows x 128 B
constexpr int kStageB = BN * 128;  // bytes: 256 rows x 128 B
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccOutlierCol = 256;

// Instruction descriptors (tcgen05 .kind::i8 / .kind::f16): dense, K-major
// A and B, N = 256 (bits 17-22 hold N/8), M = 128 (bits 24-28 hold M/16).
constexpr uint32_t kIdescI8 = (2u << 4)      // D = s32
                              | (1u << 7)    // A = signed int8
                              | (1u << 10)   // B = signed int8
                              | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
constexpr uint32_t kIdescF16 = (1u << 4)     // D = f32, A = B = f16 (0)
                               | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

constexpr size_t kSmemTiles = (size_t)kStages * (kStageA + kStageB);
constexpr size_t kSmemBytes = 1024 /*align slack*/ + kSmemTiles + 256 /*barriers*/ + 2 * BN * 4;

struct __align__(8) Ctrl {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t acc;
    uint32_t tmem_base;
    uint32_t abort;
};

__global__ void __launch_bounds__(kThreads, 1)
gemm_i8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmXo, const __grid_constant__ CUtensorMap tmWo,
               const GemmArgs a, const int num_m_tiles) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + kStages * kStageA;
    Ctrl *ctrl = reinterpret_cast<Ctrl *>(smem + kSmemTiles);
    float *s_scb = reinterpret_cast<float *>(smem + kSmemTiles + 256);
    float *s_bias = s_scb + BN;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mt = blockIdx.x % num_m_tiles, nt = blockIdx.x / num_m_tiles;
    const int64_t m0 = (int64_t)mt * BM, n0 = (int64_t)nt * BN;
    const int nkb = (int)ceil_div(a.K, 128);
    const int n_out = a.n_outliers ? *a.n_outliers : 0;
    const int n_mma_o = (n_out + 15) >> 4;   // fp16 MMAs of K = 16
    const int nkb_o = (n_out + 63) >> 6;     // fp16 k-blocks of 64
    const int total_kb = nkb + nkb_o;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&ctrl->full[s]), 1);
            mbar_init(smem_u32(&ctrl->empty[s]), 1);
        }
        mbar_init(smem_u32(&ctrl->acc), 1);
        ctrl->abort = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (threadIdx.x == 32) {
        tma_prefetch(&tmA);
        tma_prefetch(&tmB);
        if (nkb_o) {
            tma_prefetch(&tmXo);
            tma_prefetch(&tmWo);
        }
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&ctrl->tmem_base), kTmemCols);
        tmem_relinquish();
    }
    if (warp >= 2) {
        for (int c = threadIdx.x - 64; c < BN; c += 128) {
            const int64_t j = n0 + c;
            s_scb[c] = (a.SCB && j < a.N) ? a.SCB[j] : 0.f;
            s_bias[c] = (a.bias && j < a.N) ? __half2float(a.bias[j]) : 0.f;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctrl->tmem_base;
    volatile uint32_t *abort_flag = &ctrl->abort;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------- TMA producer --
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            for (int kb = 0; kb < total_kb; ++kb) {
                if (*abort_flag) break;
                if (!mbar_wait_bounded(smem_u32(&ctrl->empty[stage]), phase ^ 1u, kWaitLimitNs)) {
                    *abort_flag = 1;
                    record_timeout(a.status);
                    break;
                }
                const uint32_t fb = smem_u32(&ctrl->full[stage]);
                mbar_arrive_expect_tx(fb, kStageA + kStageB);
                if (kb < nkb) {
                    tma_load_2d(smem_u32(sA + stage * kStageA), &tmA, fb, kb * 128, (int32_t)m0);
                    tma_load_2d(smem_u32(sB + stage * kStageB), &tmB, fb, kb * 128, (int32_t)n0);
                } else {
                    const int ko = (kb - nkb) * 64;
                    tma_load_2d(smem_u32(sA + stage * kStageA), &tmXo, fb, ko, (int32_t)m0);
                    tma_load_2d(smem_u32(sB + stage * kStageB), &tmWo, fb, ko, (int32_t)n0);
                }
                ++issued;
                if (++stage == kStages) { stage = 0; phase ^= 1u; }
            }
            // Do not leave while copies this thread started are in flight.
            for (int u = max(0, issued - kStages); u < issued; ++u) {
                const int s = u % kStages;
                if (!mbar_wait_bounded(smem_u32(&ctrl->full[s]), (uint32_t)((u / kStages) & 1), kWaitLimitNs)) {
                    record_timeout(a.status);
                    break;
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer --
            int stage = 0;
            uint32_t phase = 0;
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
                        mma_i8(tmem, da + 2 * k, db + 2 * k, kIdescI8, (kb | k) != 0);
                } else {
                    const int kbo = kb - nkb;
                    const int nk = min(4, n_mma_o - kbo * 4);
                    for (int k = 0; k < nk; ++k)  // K = 16 fp16 = 32 bytes each
                        mma_f16(tmem + kAccOutlierCol, da + 2 * k, db + 2 * k, kIdescF16, (kbo | k) != 0);
                }
                mma_commit(smem_u32(&ctrl->empty[stage]));
                if (++stage == kStages) { stage = 0; phase ^= 1u; }
            }
            // Always signal the epilogue; the arrive lands once every MMA
            // issued above has finished, so TMEM is safe to read (or free).
            mma_commit(smem_u32(&ctrl->acc));
            if (!mbar_wait_bounded(smem_u32(&ctrl->acc), 0, kWaitLimitNs)) record_timeout(a.status);
        }
    } else {
        // ---------------------------------------------------- epilogue --
        const int q = warp & 3;  // this warp may touch TMEM lanes [32q, 32q + 32)
        const int64_t row = m0 + q * 32 + lane;
        bool ok = mbar_wait_bounded(smem_u32(&ctrl->acc), 0, kWaitLimitNs);
        if (!ok) record_timeout(a.status);
        ok = __all_sync(0xffffffffu, ok) && !*abort_flag;
        tc_fence_after();
        if (ok) {
            const bool row_ok = row < a.M;
            const float rs = (row_ok && a.SCA) ? a.SCA[row] * (1.0f / 16129.0f) : 0.f;
            const uint32_t lane_base = (uint32_t)(q * 32) << 16;
            for (int c = 0; c < BN; c += 32) {
                uint32_t acc[32], po[32];
                tmem_ld_32x32b_x32(tmem + lane_base + c, acc);
                if (n_out > 0) tmem_ld_32x32b_x32(tmem + lane_base + kAccOutlierCol + c, po);
                tmem_ld_wait();
                if (!row_ok || n0 + c >= a.N) continue;
                if (a.C32) {
                    int32_t *dst = a.C32 + row * a.N + n0 + c;
#pragma unroll
                    for (int v = 0; v < 8; ++v)
                        if (n0 + c + 4 * v < a.N)
                            reinterpret_cast<int4 *>(dst)[v] =
                                make_int4((int)acc[4 * v], (int)acc[4 * v + 1], (int)acc[4 * v + 2], (int)acc[4 * v + 3]);
                    continue;
                }
                uint32_t packed[16];
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    float y0 = (float)(int32_t)acc[j] * (rs * s_scb[c + j]) + s_bias[c + j];
                    float y1 = (float)(int32_t)acc[j + 1] * (rs * s_scb[c + j + 1]) + s_bias[c + j + 1];
                    if (n_out > 0) {
                        y0 += __uint_as_float(po[j]);
                        y1 += __uint_as_float(po[j + 1]);
                    }
                    __half2 h = __floats2half2_rn(y0, y1);
                    packed[j >> 1] = *reinterpret_cast<uint32_t *>(&h);
                }
                __half *dst = a.Y + row * a.N + n0 + c;
#pragma unroll
                for (int v = 0; v < 4; ++v)
                    if (n0 + c + 8 * v < a.N)
                        reinterpret_cast<uint4 *>(dst)[v] =
                            make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
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
              uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {pitch_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_gemm_tc(const GemmArgs &a, cudaStream_t s) {
    CUtensorMap mA, mB, mXo, mWo;
    if (!make_map(&mA, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.CA, a.K, a.M, a.K, 128, BM) ||
        !make_map(&mB, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.CB, a.K, a.N, a.K, 128, BN))
        return cudaErrorInvalidValue;
    if (a.Xo && a.Wo && a.n_outliers) {
        if (!make_map(&mXo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.Xo, a.kcap, a.M, a.kcap * 2, 64, BM) ||
            !make_map(&mWo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.Wo, a.kcap, a.N, a.kcap * 2, 64, BN))
            return cudaErrorInvalidValue;
    } else {
        mXo = mA;  // never read: |O| = 0 without outlier buffers
        mWo = mB;
    }
    static std::once_flag attr_once[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once[dev & 63], [&] {
        attr_err = cudaFuncSetAttribute(gemm_i8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    });
    if (attr_err != cudaSuccess) return attr_err;
    const int num_m_tiles = (int)ceil_div(a.M, BM);
    const int64_t tiles = (int64_t)num_m_tiles * ceil_div(a.N, BN);
    gemm_i8_kernel<<<(unsigned)tiles, kThreads, kSmemBytes, s>>>(mA, mB, mXo, mWo, a, num_m_tiles);
    return cudaGetLastError();
}

}  // namespace int8lt
