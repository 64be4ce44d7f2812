/*
 * int8lt -- LLM.int8() mixed-precision linear layer for NVIDIA B200 (sm_100a).
 *
 * C ABI of libint8lt.so. Computes Y = X W^T + bias the LLM.int8() way:
 *
 *   1. O = feature columns of X holding any |x| >= threshold (outliers);
 *   2. the other columns of X are quantized row-wise (one absmax scale per
 *      token), the weights per output channel (one absmax scale per row of W);
 *   3. int8 x int8 GEMM with int32 accumulation on the tensor cores;
 *   4. dequantize with the outer product of row and column scales;
 *   5. add the fp16 product of the outlier columns (and the bias).
 *
 * Sources (web pages on LLM.int8(), cited by page title and section):
 *   [HF]  "Hugging Face LLM.int8() integration into transformers and
 *         accelerate" (agentlenshq.com): three-step recipe; absmax example;
 *         Linear8bitLt / CB / SCB with W ~= CB * SCB / 127.
 *   [P]   "LLM.int8() paper summary" (kurtkim.github.io/p/llm.int8/):
 *         "8-bit Data Types and Quantization" (absmax equation);
 *         "Int8 Matrix Multiplication with 16-bit Float Inputs and Outputs";
 *         "Vector-wise Quantization"; "The Core of LLM.int8(): Mixed-precision
 *         Decomposition" (threshold alpha = 6.0).
 *
 * Conventions for every entry point:
 *   - Matrices are dense row-major. X is [M, K] (tokens x features), W is
 *     [N, K] (nn.Linear layout: one row per output channel), Y is [M, N].
 *   - The int8 weight codes CB, logically [N, K], are stored in this
 *     library's blocked weight layout: 4096-byte blocks of 32 output channels
 *     x 128 bytes of K, ordered row block by row block (k-blocks inside),
 *     each block row-major; CB[j, k] sits at byte
 *       ((j / 32) * ceil(K / 128) + k / 128) * 4096 + (j % 32) * 128 + k % 128,
 *     and the codes past N or K inside the last blocks are zero. The buffer
 *     has int8lt_weight_bytes(N, K) bytes. int8lt_pack_weight and
 *     int8lt_unpack_weight convert from and to row-major codes.
 *   - "fp16" means IEEE binary16, passed as void pointers. Every tensor
 *     pointer is DEVICE memory owned by the caller; the library allocates
 *     nothing and keeps no per-call state. `stream` is a cudaStream_t (NULL =
 *     legacy default stream). All compute entry points are asynchronous and
 *     stream-ordered; they return after the launches are queued.
 *   - Host-side validation runs before any launch. A call whose output is
 *     empty (M == 0 or N == 0, with a valid K) returns INT8LT_OK without
 *     reading its pointers, which may then be NULL. On any error status no
 *     kernel has been launched (except INT8LT_ERR_CUDA, reported when a
 *     launch itself fails).
 *   - Codes are int8 in [-127, 127]; scales are the fp32 absmax of the
 *     quantized vector (not its reciprocal), so x ~= code * scale / 127.
 *   - Shapes: M, N >= 0 (0 is a no-op returning INT8LT_OK), 16 <= K <= 133144
 *     and K % 16 == 0 (int8 rows must be 16-byte multiples for the TMA
 *     engine; 133144 * 127^2 < 2^31 keeps every int32 sum exact), N % 8 == 0.
 *   - Alignment: X, W, W_outlier, CB, CA, Y and the workspace must be 16-byte
 *     aligned; scale arrays 4-byte, bias 2-byte. A 32-byte aligned CB (any
 *     cudaMalloc'd buffer is) lets the decode GEMV read it with 256-bit loads;
 *     a CB that is only 16-byte aligned gives the same results, more slowly.
 *   - NaN or infinite values inside X or W are outside the contract.
 */
#ifndef INT8LT_H
#define INT8LT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    INT8LT_OK = 0,
    INT8LT_ERR_NULL = 1,        /* a required pointer is NULL */
    INT8LT_ERR_SHAPE = 2,       /* M, N or K outside the limits above */
    INT8LT_ERR_ALIGN = 3,       /* a pointer is not aligned as required */
    INT8LT_ERR_VALUE = 4,       /* threshold is NaN or negative */
    INT8LT_ERR_WORKSPACE = 5,   /* ws_bytes < int8lt_workspace_size(...) */
    INT8LT_ERR_CUDA = 6,        /* a CUDA runtime call or launch failed */
    INT8LT_ERR_TIMEOUT = 7,     /* a kernel gave up a bounded wait (device status) */
    INT8LT_ERR_UNSUPPORTED = 8, /* current device is not compute capability 10.0 */
    INT8LT_ERR_TOO_LARGE = 9,   /* call exceeds the fixed scratch of
                                   int8lt_forward_static_scratch */
    INT8LT_ERR_BOUNDS = 10      /* checking build only (libint8lt_check.so): a
                                   kernel's index failed its bounds check and
                                   the access was skipped (device status) */
} int8lt_status;

/* Human-readable name of a status code (static string, never NULL). */
const char *int8lt_status_string(int status);

/* Library version, as major * 10000 + minor * 100 + patch. */
int int8lt_version(void);

/*
 * Workspace bytes that int8lt_forward needs for an [M, K] x [N, K]^T call.
 * Holds the outlier bitmap partials, the outlier list and count, the device
 * status word, CA/SCA, the gathered fp16 outlier activations, and either the
 * gathered fp16 outlier weights (M > 16) or the decode GEMV's int32 partial
 * sums of row blocks shared between warps (M <= 16).
 * The outlier buffers are sized for the worst case |O| = K, so any input fits.
 * Returns 0 for shapes the library rejects.
 */
size_t int8lt_workspace_size(int64_t M, int64_t N, int64_t K);

/*
 * Prepare a freshly allocated workspace (stream-ordered): zeroes all
 * ws_bytes of it, so that the device status word, the outlier count, the
 * quantize pass's launch, barrier and row counters, its column bitmaps and the
 * prefill GEMM's split-tile flags start at zero. Call once after allocating
 * a workspace, before its first use; later calls keep it consistent by
 * themselves. After a reported INT8LT_ERR_TIMEOUT call it again before the
 * next use. int8lt_read_device_status clears the status word alone.
 */
int int8lt_workspace_init(void *ws, size_t ws_bytes, void *stream);

/*
 * Synchronize `stream`, then read and clear the workspace's status word.
 * Returns INT8LT_OK, or INT8LT_ERR_TIMEOUT if any kernel that used this
 * workspace since the last read gave up a bounded wait (its outputs are then
 * undefined), INT8LT_ERR_BOUNDS (checking build only) if a kernel's index
 * failed its bounds check, or INT8LT_ERR_CUDA if the stream reported an error.
 */
int int8lt_read_device_status(void *ws, size_t ws_bytes, void *stream);

/*
 * Bytes of the blocked weight codes of an [N, K] weight:
 * ceil(N / 32) * ceil(K / 128) * 4096. Returns 0 for N < 0 or K < 1.
 */
size_t int8lt_weight_bytes(int64_t N, int64_t K);

/*
 * Layout conversions (stream-ordered): row-major int8 codes CB_rows [N, K]
 * -> the blocked weight layout CB (int8lt_weight_bytes(N, K) bytes, padding
 * written as zero), and back (only the N x K codes are written). CB must be
 * 16-byte aligned, CB_rows too when K % 16 == 0. Any N >= 0, K >= 1.
 */
int int8lt_pack_weight(const int8_t *CB_rows, int64_t N, int64_t K, int8_t *CB, void *stream);
int int8lt_unpack_weight(const int8_t *CB, int64_t N, int64_t K, int8_t *CB_rows, void *stream);

/*
 * Memory accounting of a prepared layer: the device bytes it keeps resident
 * between calls, CB (int8lt_weight_bytes(N, K)) + SCB (4 N), plus the fp16
 * weight (2 N K) when the caller keeps it to serve the outlier columns
 * (keep_fp16_weight != 0, W_outlier non-NULL). Against the 2 N K bytes of the
 * fp16 layer this is about 50% without the fp16 weight, the saving the
 * "LLM.int8() paper summary" states ("Int8 Matrix Multiplication at Scale");
 * the outlier term then costs no extra weight memory, because its fp16
 * weights are recovered from CB and SCB ([HF] has_fp16_weights=False). The
 * per-call workspace (int8lt_workspace_size) is transient and not counted.
 * Returns 0 for N < 0 or K < 1.
 */
size_t int8lt_layer_bytes(int64_t N, int64_t K, int keep_fp16_weight);

/*
 * Weight conversion: W fp16 [N, K] -> CB int8 [N, K] (blocked weight
 * layout, int8lt_weight_bytes(N, K) bytes) and SCB fp32 [N].
 * [HF] "transformers integration": weights become int8 in [-127, 127] with a
 * per-output-channel scale, recoverable as W ~= CB * SCB / 127; [P] absmax
 * equation, vector-wise (per output channel). SCB[j] = max_k |W[j,k]|,
 * CB[j,k] = clamp(rint(W[j,k] * fp32(127 / SCB[j])), -127, 127) with the
 * division and product rounded to fp32, ties to even; SCB[j] = 0 gives all
 * zero codes. Deterministic and idempotent: re-running it gives identical
 * bytes. K % 16 == 0 is not required here (K >= 1).
 */
int int8lt_prepare_weight(const void *W, int64_t N, int64_t K, int8_t *CB, float *SCB,
                          void *stream);

/*
 * Outlier detection and row-wise quantization of X fp16 [M, K].
 * [HF] recipe step 1 and [P] "Mixed-precision Decomposition": O = { h : some
 * |X[i,h]| >= threshold }, compared in fp32. [HF] step 2 and [P] absmax /
 * vector-wise equations: for every row i, SCA[i] = max over h not in O of
 * |X[i,h]|, CA[i,h] = clamp(rint(X[i,h] * fp32(127 / SCA[i])), -127, 127) for
 * h not in O and CA[i,h] = 0 for h in O. threshold = +inf gives O empty;
 * threshold = 0 puts every column in O.
 *   outlier_idx: int32 [K] capacity; receives O in ascending order.
 *   n_outliers : one int32 (device) receiving |O|.
 *   ws         : scratch of at least int8lt_workspace_size(M, 8, K) bytes.
 */
int int8lt_quantize_rows(const void *X, int64_t M, int64_t K, float threshold,
                         int8_t *CA, float *SCA, int32_t *outlier_idx, int32_t *n_outliers,
                         void *ws, size_t ws_bytes, void *stream);

/*
 * The LLM.int8() forward: Y fp16 [M, N] =
 *     fp16( C[i,j] * SCA[i] * SCB[j] / 127^2 + sum_{h in O} X[i,h] Wo[j,h] + bias[j] )
 * with C = CA CB^T accumulated exactly in int32 ([P] int8 matmul and
 * vector-wise equations), O and CA/SCA as in int8lt_quantize_rows, and the
 * outlier term of [P] "Mixed-precision Decomposition" / [HF] step 3.
 * The combination is computed in fp32 and rounded once to fp16.
 *   CB, SCB   : from int8lt_prepare_weight (CB in the blocked weight layout).
 *   W_outlier : fp16 [N, K] weights for the outlier columns (only the columns
 *               in O are read), or NULL to use fp16(fp32(CB * SCB) / 127).
 *   bias      : fp16 [N] or NULL.
 *   ws        : at least int8lt_workspace_size(M, N, K) bytes.
 * Dispatch: M <= 16 runs the memory-bound streaming GEMV; larger M runs the
 * tcgen05 int8 GEMM with the outlier MMA and the dequantization fused into it.
 */
int int8lt_forward(const void *X, int64_t M, int64_t N, int64_t K,
                   const int8_t *CB, const float *SCB, const void *W_outlier,
                   float threshold, const void *bias, void *Y,
                   void *ws, size_t ws_bytes, void *stream);

/*
 * The two halves of int8lt_forward, for callers that want to time or
 * schedule them apart; int8lt_forward is exactly _quantize then _matmul on
 * the same stream and workspace, with identical arguments.
 *   _quantize: outlier set O, CA/SCA and the fp16 outlier activations of X
 *              into the workspace, plus (M > 16) the fp16 outlier weights
 *              gathered from W_outlier (or CB/SCB).
 *   _matmul  : the int8 GEMM (M > 16) or GEMV (M <= 16) with the fused
 *              dequantization, outlier product and bias, writing Y. It reads
 *              only what the preceding _quantize left in `ws`.
 */
int int8lt_forward_quantize(const void *X, int64_t M, int64_t N, int64_t K,
                            const int8_t *CB, const float *SCB, const void *W_outlier,
                            float threshold, void *ws, size_t ws_bytes, void *stream);
int int8lt_forward_matmul(int64_t M, int64_t N, int64_t K, const int8_t *CB, const float *SCB,
                          const void *W_outlier, const void *bias, void *Y,
                          void *ws, size_t ws_bytes, void *stream);

/*
 * Allocation-free forward for decode shapes. The paper has no counterpart:
 * this is a deployment convenience of this library. It computes exactly what
 * int8lt_forward computes (same kernels, same results) for M <= 16 tokens,
 * but takes its scratch from a fixed 8 MiB array inside the library instead
 * of a caller workspace, for callers that cannot allocate device memory: a
 * plugin or engine that is handed only input and output buffers, a runtime
 * whose device memory is owned by its own pool, or a decode loop that must
 * not call cudaMalloc because it can synchronize the device.
 *   - Limits: M <= 16, and the call's scratch (int8lt_workspace_size(M, N, K))
 *     must fit the 8 MiB array (e.g. K = 12288 with N up to about 100k);
 *     larger calls return INT8LT_ERR_TOO_LARGE without launching anything.
 *   - The array lives on every GPU on which the library is loaded, until the
 *     process exits. The first call on a device (this one or
 *     int8lt_static_scratch_read_status) looks up the array's device address
 *     with that device current and zeroes the whole array with a synchronous
 *     cudaMemset; make that first call before any stream capture. If that
 *     set-up fails, the call returns INT8LT_ERR_CUDA and the next call tries
 *     again.
 *   - All calls on a device share the array. Each call re-initialises what
 *     it reads, but calls whose kernels overlap on the GPU (unordered streams
 *     or concurrent host threads) race on it and produce wrong results.
 *   - A bounded wait that runs out on the device is recorded in the array's
 *     own status word, not reported by this call's return value: read it
 *     with int8lt_static_scratch_read_status (the output of a call that timed
 *     out is undefined).
 * Other arguments and errors as int8lt_forward.
 */
int int8lt_forward_static_scratch(const void *X, int64_t M, int64_t N, int64_t K,
                                  const int8_t *CB, const float *SCB, const void *W_outlier,
                                  float threshold, const void *bias, void *Y, void *stream);

/*
 * Device status of int8lt_forward_static_scratch on the current device, as
 * int8lt_read_device_status is for a workspace: synchronizes `stream`, reads
 * and clears the fixed array's status word, and returns INT8LT_OK, or
 * INT8LT_ERR_TIMEOUT if a kernel of an earlier call gave up a bounded wait
 * (after which the array's header and bitmaps are zeroed again, so the next
 * call starts clean), or INT8LT_ERR_CUDA if the stream reported an error.
 * Allocates nothing.
 */
int int8lt_static_scratch_read_status(void *stream);

/* ------------------------------------------------- zeropoint quantization -- */

/*
 * Zeropoint (asymmetric) row quantization, [P] "8-bit Data Types and
 * Quantization", zeropoint quantization: every row x of X fp16 [R, K] (a
 * token of an activation matrix, or an output channel of W) gets
 *   ND[i]  = fp32(254 / fp32(max x - min x))   (1 when max x == min x),
 *   ZP[i]  = rint(fp32(ND[i] * min x)) + 127,
 *   Q[i,h] = clamp(rint(fp32(ND[i] * X[i,h])) - ZP[i], -127, 127),
 *   SUM[i] = sum over h of Q[i,h],
 * rint rounding ties to even, so that X[i,h] ~= (Q[i,h] + ZP[i]) / ND[i]. The
 * page's zeropoint formula is garbled; this is the reading whose shifted
 * codes the page's product (A + zp_a)(B + zp_b) takes. Unlike absmax codes,
 * the full [-127, 127] range is used by every row whatever its sign balance.
 *   Q   : int8 [R, K] row-major (16-byte aligned); ND fp32 [R]; ZP, SUM int32 [R].
 * K % 16 == 0, 16 <= K <= 133144 (as for int8lt_forward). Deterministic; no
 * workspace. int8lt_prepare_weight_zp is the same operation on W [N, K]
 * (N % 8 == 0), written CB / NDB / ZB / SB for int8lt_forward_zp, with CB in
 * the blocked weight layout (int8lt_weight_bytes(N, K) bytes).
 */
int int8lt_quantize_rows_zp(const void *X, int64_t R, int64_t K, int8_t *Q, float *ND,
                            int32_t *ZP, int32_t *SUM, void *stream);
int int8lt_prepare_weight_zp(const void *W, int64_t N, int64_t K, int8_t *CB, float *NDB,
                             int32_t *ZB, int32_t *SB, void *stream);

/*
 * Linear layer with zeropoint quantization on both sides and no outlier
 * split ([P] "8-bit Data Types and Quantization": the product of two
 * zeropoint-quantized operands, unrolled):
 *   C[i,j] = (A_i + za_i) . (B_j + zb_j)
 *          = A_i . B_j + zb_j SA_i + za_i SB_j + K za_i zb_j,
 *   Y[i,j] = fp16( C[i,j] / (NDA[i] NDB[j]) + bias[j] ),
 * where A, NDA, za, SA are the zeropoint codes of the rows of X (computed by
 * this call into the workspace) and CB, NDB, ZB, SB come from
 * int8lt_prepare_weight_zp. A_i . B_j runs on the int8 tensor cores (int32,
 * exact); the corrections are added in int64 (exact) and the sum is scaled
 * in fp32. Same dispatch, shapes, alignment and workspace
 * (int8lt_workspace_size) as int8lt_forward; ZB and SB 4-byte aligned.
 */
int int8lt_forward_zp(const void *X, int64_t M, int64_t N, int64_t K,
                      const int8_t *CB, const float *NDB, const int32_t *ZB, const int32_t *SB,
                      const void *bias, void *Y, void *ws, size_t ws_bytes, void *stream);

/*
 * The two halves of int8lt_forward_zp, as int8lt_forward_quantize /
 * int8lt_forward_matmul are of int8lt_forward: int8lt_forward_zp is exactly
 * _quantize then _matmul on the same stream and workspace.
 *   _quantize: zeropoint codes, nd, zeropoints and code sums of X's rows
 *              into the workspace (and, M <= 16, zeroes the GEMV's sums).
 *   _matmul  : the int8 GEMM (M > 16) or GEMV (M <= 16) on those codes with
 *              the zeropoint corrections, scales and bias fused, writing Y.
 */
int int8lt_forward_zp_quantize(const void *X, int64_t M, int64_t N, int64_t K,
                               void *ws, size_t ws_bytes, void *stream);
int int8lt_forward_zp_matmul(int64_t M, int64_t N, int64_t K, const int8_t *CB, const float *NDB,
                             const int32_t *ZB, const int32_t *SB, const void *bias, void *Y,
                             void *ws, size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------- tests -- */

/*
 * Test entry: the int8 GEMM alone, C int32 [M, N] = CA [M, K] . CB [N, K]^T
 * (CA row-major, CB in the blocked weight layout),
 * through the same kernels int8lt_forward dispatches to (M <= 16: the GEMV,
 * otherwise the tcgen05 GEMM) with the dequantizing epilogue replaced by an
 * int32 store, so the accumulators can be compared bit for bit. Same shape,
 * alignment and workspace rules as int8lt_forward.
 */
int int8lt_debug_gemm_i32(const int8_t *CA, const int8_t *CB, int64_t M, int64_t N, int64_t K,
                          int32_t *C, void *ws, size_t ws_bytes, void *stream);

/* Schedules of the prefill GEMM's last wave (int8lt_set_gemm_split). */
enum {
    INT8LT_SPLIT_AUTO = 0,    /* split when it saves enough (default) */
    INT8LT_SPLIT_ALWAYS = 1,  /* split whenever the tile count allows */
    INT8LT_SPLIT_NEVER = 2    /* whole tiles only */
};

/*
 * Tuning: how the prefill GEMM (M > 16) schedules its 256 x 256 output tiles
 * over its CTA pairs. Whole tiles go round-robin. When the tile count is not
 * a multiple of the pair count, the tiles after the last full wave may be
 * split into equal k-block ranges, one per pair ("stream-K"), at the price of
 * handing one tile's int32 sums per pair through the workspace (measured at
 * roughly 8 us per launch). INT8LT_SPLIT_AUTO splits only when that saves the
 * busiest pair at least 32 k-blocks of 128 bytes (one 256 x 256 x 4096 tile).
 * The setting is process-wide, thread-safe, and applies to launches made
 * after the call; the results do not depend on it (integer sums are exact).
 * Returns the previous mode, or -1 for an unknown mode.
 */
int int8lt_set_gemm_split(int mode);

/*
 * Test entry (host only, no GPU needed): the work schedule of the prefill
 * GEMM for `tiles` output tiles of `nkb` 128-byte k-blocks over `pairs` CTA
 * pairs under split mode `mode` (INT8LT_SPLIT_*), as the kernel walks it.
 * Writes up to cap_rows rows of 6 int32 (pair, tile, first k-block, end
 * k-block, head flag, tail flag) and returns the number of segments (or -1
 * for bad arguments). A split tile's head (its first k-blocks, which finishes
 * it) and tail (its last k-blocks, whose int32 sums are handed over) sit in
 * adjacent pairs.
 */
int int8lt_debug_gemm_schedule(int tiles, int nkb, int pairs, int mode, int32_t *out, int cap_rows);

/*
 * Test entry (host only, no GPU needed): the order in which the prefill GEMM
 * visits its output tiles, for num_m tile rows (256 rows of Y each) and
 * num_n tile columns (256 output channels each). Tile index t is the one the
 * schedule above names; out[2t], out[2t + 1] receive its tile row and tile
 * column (out holds 2 * num_m * num_n int32, caller-owned). Returns
 * num_m * num_n, or -1 for bad arguments (a null out, a dimension below 1,
 * more than 2^30 tiles).
 */
int int8lt_debug_tile_order(int num_m, int num_n, int32_t *out);

/*
 * Test entry: launch one block that waits on a barrier nothing ever arrives
 * at, with the same bounded-wait routine the GEMM pipeline uses, limited to
 * `limit_ns` nanoseconds (1e3 .. 1e9). The kernel records INT8LT_ERR_TIMEOUT
 * in the workspace status word and returns normally; no GPU fault, trap or
 * hang is involved.
 */
int int8lt_debug_wait_timeout(void *ws, size_t ws_bytes, int64_t limit_ns, void *stream);

/*
 * Test entry: one block enters the grid-wide barrier of the quantize pass
 * (the step between outlier detection and quantization) of a launch that
 * counts one block more than it has, so its bounded wait gives up after
 * `limit_ns` nanoseconds (1e3 .. 1e9). The kernel records INT8LT_ERR_TIMEOUT
 * in the workspace status word and returns normally. The barrier's counts in
 * the workspace header are then off, as after any such timeout: call
 * int8lt_workspace_init before the workspace's next use. ws_bytes must cover
 * the header and bitmaps (any int8lt_workspace_size of a valid shape does).
 */
int int8lt_debug_barrier_timeout(void *ws, size_t ws_bytes, int64_t limit_ns, void *stream);

/*
 * Test entry: as int8lt_debug_barrier_timeout, against the header of the
 * fixed array of int8lt_forward_static_scratch on the current device, so that
 * int8lt_static_scratch_read_status can be seen to report the timeout and
 * restore the array.
 */
int int8lt_debug_static_scratch_timeout(int64_t limit_ns, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* INT8LT_H */
