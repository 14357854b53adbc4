/*
 * qgmm.h -- C ABI of the B200 (sm_100a) fused int8 GroupedMatmul +
 * MoeFinalizeRouting library (libqgmm.so).
 *
 * The operation (pages: "aclnnGroupedMatmulFinalizeRoutingWeightNzV2",
 * function description and parameter constraints; "matmul支持pertoken量化模式",
 * 计算示例):
 *
 *   off[0] = 0; off[g+1] = group_list[g]            (group_list_type 0: cumulative ends)
 *               off[g+1] = off[g] + group_list[g]   (group_list_type 1: per-group counts)
 *   for every expert g and row i in [off[g], off[g+1]):
 *     acc[i][j] = sum_kk x1[i][kk] * W(g, kk, j)                      exact int32
 *     y[i][j]   = ((f32(acc) * scale[g][j]) * pertoken_scale[i] + bias[g][j]) * logit[i]
 *   out[r][j]  = (shared_offset <= r < shared_offset + shared_bs) ? f32(shared[r - shared_offset][j]) : 0
 *   out[row_index[i]][j] += y[i][j]    for every row i below the groups' total
 *
 * W(g, kk, j) is x2[g][kk][j] (int8, layout (e, k, n), n contiguous), or for
 * int4 weights the signed nibble j%8 (lowest nibble = lowest j) of the int32
 * word x2[g][kk][j/8] (layout (e, k, n/8)), or for E4M3 operands the value of
 * the FLOAT8 E4M3FN byte x2[g][kk][j] (x1 is then E4M3 too).  Every f32 step rounds to nearest
 * even; nothing is fused into an FMA.  Where the pages leave the formula open
 * (bias position, unweighted sharedInput, nibble order, summation order) the
 * library takes the readings written above.
 *
 * Conventions shared by every entry point:
 *  - Every pointer except those of qgmm_finalize_workspace, qgmm_device_status
 *    (flags) and qgmm_status_string is a DEVICE pointer on the current CUDA
 *    device.  The caller owns all memory, including the workspace; the library
 *    allocates nothing and keeps no state between calls (a per-device cache of
 *    the SM count and the driver's tensor-map entry point aside).
 *  - Every call is asynchronous on `cuda_stream` (a cudaStream_t; NULL = the
 *    legacy default stream) except qgmm_device_status, which synchronises it.
 *  - Host-side checks run before any launch; a failing check returns its code
 *    and launches nothing.
 *  - Problems the host cannot see (group_list values, row_index values) are
 *    checked on the device: offending rows are skipped, the remaining rows are
 *    still computed, and QGMM_DEV_* bits are set in the workspace status word,
 *    which qgmm_device_status returns.  No kernel traps or asserts.
 *  - Every wait inside a kernel is bounded (about one second); if one runs out
 *    the kernel sets QGMM_DEV_TIMEOUT and returns.
 */
#ifndef QGMM_H
#define QGMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QGMM_OK = 0,
    QGMM_ERR_NULL_PTR = 1,            /* a required pointer is NULL                          */
    QGMM_ERR_SHAPE = 2,               /* a size is out of range (limits below)                */
    QGMM_ERR_DTYPE = 3,               /* an unknown weight / index / group-list / scale type   */
    QGMM_ERR_WORKSPACE_TOO_SMALL = 4, /* ws_bytes below qgmm_finalize_workspace's answer      */
    QGMM_ERR_UNSUPPORTED = 5,         /* the device is not sm_100 or a feature is not built   */
    QGMM_ERR_CUDA = 6,                /* a CUDA runtime / driver call failed                  */
    QGMM_ERR_DEVICE_INPUT = 7,        /* qgmm_device_status found QGMM_DEV_* bits set         */
    QGMM_ERR_ALIGNMENT = 8,           /* a pointer is not suitably (16- or 32-byte) aligned   */
    QGMM_ERR_SCRATCH_LIMIT = 9        /* qgmm_finalize_static_scratch: scratch above its cap  */
} qgmm_status;

/* x2 (and x1) element type: int8 x2 (e,k,n) | int4 packed in int32 (e,k,n/8) |
 * FLOAT8 E4M3FN x1 and x2 (e,k,n), page 1's Atlas 350 per-token / per-channel mode |
 * MxA8W4: E4M3 x1, FP4 E2M1 x2 (e,n,k/2 bytes), E8M0 block scales (page 1, Atlas 350) */
enum { QGMM_W_INT8 = 0, QGMM_W_INT4_PACKED_INT32 = 1, QGMM_W_FP8_E4M3 = 2, QGMM_W_MXFP4 = 3 };
enum { QGMM_IDX_INT64 = 0, QGMM_IDX_INT32 = 1 };          /* row_index element type             */
enum { QGMM_GROUP_CUMSUM = 0, QGMM_GROUP_COUNTS = 1 };    /* group_list meaning                 */
enum { QGMM_SCALE_F32 = 0, QGMM_SCALE_BF16 = 1 };         /* scale element type                 */

/* Device-side status bits (qgmm_device_status). */
#define QGMM_DEV_GROUP_NEGATIVE     (1u << 0)  /* a type-1 count (or type-0 end) below zero    */
#define QGMM_DEV_GROUP_NOT_MONOTONE (1u << 1)  /* type 0: an end smaller than the previous one */
#define QGMM_DEV_GROUP_TOTAL_GT_M   (1u << 2)  /* the groups cover more than m rows           */
#define QGMM_DEV_ROW_INDEX_RANGE    (1u << 3)  /* a row_index value outside [0, output_bs)    */
#define QGMM_DEV_TIMEOUT            (1u << 4)  /* a bounded in-kernel wait ran out            */

/*
 * Problem description.
 *   m       rows of x1 (tokens x topK), 1 <= m <= 2^24 (page 1 allows [1, 16*1024*8])
 *   k       reduction size, 128 <= k <= 65536, k % 128 == 0 (page 1 fixes k = 2048)
 *   n       output columns, 256 <= n <= 65536, n % 256 == 0 (page 1 fixes n = 7168)
 *   e       experts, 1 <= e <= 1024 (page 1: [1, 256] on A2/A3, [1, 1024] on Atlas 350)
 *   output_bs   rows of out, >= 1
 *   weight_type     QGMM_W_INT8 | QGMM_W_INT4_PACKED_INT32 | QGMM_W_FP8_E4M3.  With
 *                   QGMM_W_FP8_E4M3 both x1 and x2 hold FLOAT8 E4M3FN bytes (page 1,
 *                   Atlas 350: x1 and x2 FLOAT8_E4M3FN with a per-channel scale and a
 *                   per-token pertokenScale); acc is then the tensor core's f32 sum
 *                   of the E4M3 products (not exact: rounded once per K = 32 step
 *                   at most), and the dequant below starts from that f32 value.
 *                   With QGMM_W_MXFP4 (page 1's Atlas 350 MxA8W4 mode, where x2 is
 *                   transposed and pertokenScale and scale hold one scale per 32
 *                   k-elements): x1 is E4M3 [m, k]; x2 holds FP4 E2M1 values
 *                   (e, n, k), two per byte with the lower k in the low nibble,
 *                   (e, n, k/2) bytes, and transpose_x2 must be 1; pertoken_scale
 *                   points to E8M0 bytes sfa [m, k/32] (as produced by
 *                   qgmm_per_token_quant_mxfp8) and scale to E8M0 bytes sfb
 *                   [e, n, k/32], both required; then
 *                     acc[i][j] = sum_b 2^(sfa[i][b]-127) 2^(sfb[g][j][b]-127)
 *                                       * sum_{kk in block b} x1[i][kk] W(g, j, kk)
 *                   summed by the tensor core in f32 (tcgen05.mma
 *                   kind::mxf8f6f4.block_scale), and y = (acc + bias) * logit.
 *                   ld_sb is then the n-stride of sfb and bias; ld_x2 that of x2.
 *   group_list_type QGMM_GROUP_CUMSUM (0) | QGMM_GROUP_COUNTS (1)
 *   row_index_type  QGMM_IDX_INT64 | QGMM_IDX_INT32
 *   shared_bs, shared_offset   sharedInput rows and where they land;
 *                   shared_bs == 0 means no sharedInput;
 *                   0 <= shared_offset and shared_offset + shared_bs <= output_bs (page 1)
 *   deterministic   0: combine with float atomics (order unspecified);
 *                   1: fixed per-element order -- shared value first, then the
 *                      source rows in ascending order -- through a
 *                      destination-sorted segmented reduce.  Bitwise
 *                      reproducible from run to run.  (Page 1, 确定性计算.)
 *   expected_m_per_expert   tiling hint, rows one expert is expected to get;
 *                   0 = use m / e.  Changes only the tile shape, never the
 *                   result.  (Page 1: tuningConfigOptional[0].)
 *   scale_type      QGMM_SCALE_F32 (0) | QGMM_SCALE_BF16 (1): element type of
 *                   `scale` (page 1: scaleOptional is FLOAT or BF16 on A2/A3).
 *                   A bf16 scale is widened to f32, which is exact, and then
 *                   enters the same f32 dequant.
 *   transpose_x2    0: int8 x2 is (e, k, n); 1: int8 x2 is (e, n, k) (page 1,
 *                   full-quant scenario: x2 may be transposed, (e, n, k), on
 *                   Atlas 350; A2/A3 take only the non-transposed layout).
 *                   Same result either way (int8 and E4M3).  int4 weights must
 *                   be non-transposed (QGMM_ERR_UNSUPPORTED otherwise).
 *   ld_x2, ld_sb, ld_out, ld_shared   row strides, 0 = n (no counterpart on the pages).
 *                   They let a call work on a block of n columns inside wider
 *                   tensors -- the column split across GPUs, where each GPU
 *                   owns columns [c0, c0 + n) of an N-column op and passes
 *                   pointers advanced to column c0:
 *                     ld_x2   columns of x2's rows: x2 element (g, kk, j) is at
 *                             (g*k + kk)*ld_x2 + j (int8), word (g*k + kk)*ld_x2/8 + j/8
 *                             (int4), or (g*ld_x2 + j)*k + kk (transpose_x2);
 *                             n <= ld_x2 <= 2^23, ld_x2 % 32 == 0
 *                     ld_sb   row stride of scale and bias: element (g, j) at
 *                             g*ld_sb + j; n <= ld_sb <= 2^32, ld_sb % 8 == 0
 *                     ld_out  row stride of out: element (r, j) at r*ld_out + j;
 *                             n <= ld_out <= 2^32, ld_out % 8 == 0
 *                     ld_shared   the same for shared_input
 *                   Columns outside [0, n) of each row are neither read nor
 *                   written, so calls on disjoint column blocks of the same
 *                   tensors may run at the same time.
 */
typedef struct {
    int64_t m, k, n, e, output_bs;
    int32_t weight_type, group_list_type, row_index_type;
    int64_t shared_bs, shared_offset;
    int32_t deterministic;
    int64_t expected_m_per_expert;
    int32_t scale_type;
    int32_t transpose_x2;
    int64_t ld_x2, ld_sb, ld_out, ld_shared;
} qgmm_problem;

/*
 * Stage 1 (page 1: the GetWorkspaceSize call, which validates the inputs).
 * Checks `p` and writes the workspace bytes qgmm_finalize needs with it to
 * *ws_bytes (host pointers).  Atomic mode: 256 bytes (the status word).
 * Deterministic mode, each part rounded up to 256 bytes:
 *   256                        status word
 *   + m*n*4                    f32 rows y
 *   + S*output_bs*4            per-segment destination histograms, where
 *                              S = min(1024, max(1, ceil(m/1024)),
 *                                      max(1, floor(max(2^24, m*n/16) / output_bs)))
 *   + (output_bs + 1)*4        bucket boundaries
 *   + m*4                      source rows grouped by destination
 * QGMM_W_MXFP4 adds, after the above, each part rounded up to 256 bytes:
 *   + (ceil(m/128) + e) * (k/128) * 512        x1's scale atoms
 *   + e * (n/128) * (k/128) * 512              the weights' scale atoms
 * (the scale words rearranged per call into the per-stage layout the MX kernel
 * bulk-copies; as many bytes as the scale arrays themselves, plus padding).
 * Errors: NULL_PTR, SHAPE, DTYPE, UNSUPPORTED (transpose_x2 with int4 weights, or
 * QGMM_W_MXFP4 without transpose_x2).
 */
qgmm_status qgmm_finalize_workspace(const qgmm_problem *p, size_t *ws_bytes);

/*
 * How many kernels one qgmm_finalize call with `p` launches on the current
 * device (host pointers; the plan depends on the device's SM count and on the
 * QGMM_PAIR / QGMM_PAIR_W4 / QGMM_PAIR_TAILS environment switches, read now).
 * Atomic mode: the output init plus the grouped GEMM launches (1, or 2 when
 * full-height tiles run on CTA pairs and odd tails on a single-CTA launch).
 * Deterministic mode adds the five bucketing kernels and the final reduce.
 * QGMM_W_MXFP4 adds the two kernels that write its scale atoms.
 * The per-token quant prologue is a separate call and is not counted.
 * Errors: NULL_PTR, SHAPE, DTYPE, UNSUPPORTED, CUDA (no usable device).
 */
qgmm_status qgmm_finalize_launches(const qgmm_problem *p, int32_t *launches);

/*
 * The grouped GEMM's plan for `p` on a device with `sms` SMs, without touching
 * any device (host pointers; no counterpart on the pages).  The same planner
 * qgmm_finalize runs, with the same QGMM_* environment switches read now, for
 * the call's combine mode (p->deterministic).  Lets a caller (or a test on a
 * machine without a GPU) see what a call would launch.
 *   tile_rows      x1 rows per tile: 16, 32, 64 or 128 (from
 *                  expected_m_per_expert, else m / e)
 *   pair           1: full-height int8 tiles on CTA pairs (256 rows per tile)
 *   tail_mode      pair path only: a group's odd last <= 128 rows run as a
 *                  padded pair tile (0), on a single-CTA launch after the pair
 *                  launch (1), or as an M = 128 pair tile (2)
 *   slab_ntiles    output slab width in 256-column tiles (atomic combine)
 *   grid           CTAs of the main GEMM launch (even on the pair path)
 *   gemm_launches  GEMM launches per call: 2 with a tail launch, else 1
 * Errors: NULL_PTR, SHAPE, DTYPE, UNSUPPORTED (as qgmm_finalize_workspace),
 * and SHAPE when sms < 2.
 */
typedef struct {
    int32_t tile_rows, pair, tail_mode, slab_ntiles, grid, gemm_launches;
} qgmm_plan_info;
qgmm_status qgmm_plan(const qgmm_problem *p, int32_t sms, qgmm_plan_info *info);

/*
 * Stage 2: run the operation on `cuda_stream`.
 *   x1              int8 [m, k] row-major, required
 *   x2              int8 [e, k, n] (or [e, n, k] with transpose_x2) or int32
 *                   [e, k, n/8], row-major, required
 *   scale           f32 or bf16 bits [e, n] (page 1's (e, 1, n)), by scale_type; NULL = all ones
 *   pertoken_scale  f32 [m]; NULL = all ones
 *   group_list      int64 [e], required
 *   logit           f32 [m]; NULL = all ones
 *   row_index       int64 or int32 [m]; NULL = identity (needs output_bs >= total).
 *                   With NULL and no shared_input, the atomic mode stores each row
 *                   directly (one contribution per output row: the same 0 + y) and
 *                   zeroes only the rows past the groups' total
 *   bias            f32 [e, n]; NULL = zeros
 *   shared_input    bf16 bits [shared_bs, n]; required iff shared_bs > 0
 *   out             f32 [output_bs, n], fully overwritten (no need to clear it)
 * (Rows of x2, scale and bias, out, and shared_input are ld_x2, ld_sb, ld_out
 * and ld_shared apart; the shapes above are for the default strides.)
 *   workspace       device memory of ws_bytes bytes, 256-byte aligned
 * x1, x2, out, shared_input, scale and bias must be 16-byte aligned (x2 32-byte
 * aligned with QGMM_W_MXFP4, the base its packed 4-bit tile copy needs).  Rows at
 * or past the groups' total are ignored.
 * Errors: NULL_PTR, SHAPE, DTYPE, ALIGNMENT, WORKSPACE_TOO_SMALL, UNSUPPORTED, CUDA.
 */
qgmm_status qgmm_finalize(const qgmm_problem *p, const int8_t *x1, const void *x2,
                          const void *scale, const float *pertoken_scale,
                          const int64_t *group_list, const float *logit, const void *row_index,
                          const float *bias, const uint16_t *shared_input, float *out,
                          void *workspace, size_t ws_bytes, void *cuda_stream);

/*
 * qgmm_finalize, plus two caller-owned cudaEvent_t handles recorded on
 * `cuda_stream` immediately before and after the grouped-GEMM launch, so a
 * caller can time that kernel alone inside a live call.  The result is the
 * same as qgmm_finalize's.  Errors: as qgmm_finalize, and NULL_PTR when
 * either event is NULL.
 */
qgmm_status qgmm_finalize_profiled(const qgmm_problem *p, const int8_t *x1, const void *x2,
                                   const void *scale, const float *pertoken_scale,
                                   const int64_t *group_list, const float *logit, const void *row_index,
                                   const float *bias, const uint16_t *shared_input, float *out,
                                   void *workspace, size_t ws_bytes, void *cuda_stream,
                                   void *gemm_begin_event, void *gemm_end_event);

/*
 * qgmm_finalize for callers that cannot allocate device memory.  (No
 * counterpart on the pages: this entry point exists for this library's users.)
 *
 * Some callers are handed only their inputs and outputs and cannot call
 * cudaMalloc for a workspace: a plugin slot in a host inference engine that
 * grants no workspace, or a serving loop that must not call cudaMalloc or
 * cudaFree because those calls can synchronise the whole device.  This entry
 * point takes the same arguments as qgmm_finalize minus the workspace, and
 * uses instead a file-scope device array of QGMM_STATIC_SCRATCH_BYTES (16 MiB)
 * inside the library.  Every GPU that loads the library holds that array until
 * the process exits.  The entry point allocates nothing (no cudaMalloc, no
 * cudaFree, no allocating library routine).
 *
 *  - Limit: the problem's workspace (qgmm_finalize_workspace) must fit in
 *    16 MiB.  Atomic mode needs 256 bytes, so it always fits; deterministic
 *    mode fits while its workspace (about m*n*4 bytes plus the bucket lists)
 *    stays within 16 MiB (for example m = 128, n = 7168).
 *    Larger problems return QGMM_ERR_SCRATCH_LIMIT before anything is launched.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - Every call shares the one array, which keeps the last call's contents.
 *    Each call clears what must start at zero (the status word and the
 *    deterministic mode's bucket counts) before using it.  Calls whose work
 *    overlaps on one GPU (for example on two streams, or from two host
 *    threads) race on the array and give wrong results: serialise them.
 *    Each device has its own copy of the array, so calls on different
 *    devices do not interfere.
 *  - Device-side input checks still run and bad rows are still skipped, but
 *    the status word lives in the library's array and is not reported.
 * Errors: as qgmm_finalize, and QGMM_ERR_SCRATCH_LIMIT.
 */
#define QGMM_STATIC_SCRATCH_BYTES ((size_t)16 << 20)
qgmm_status qgmm_finalize_static_scratch(const qgmm_problem *p, const int8_t *x1, const void *x2,
                                         const void *scale, const float *pertoken_scale,
                                         const int64_t *group_list, const float *logit,
                                         const void *row_index, const float *bias,
                                         const uint16_t *shared_input, float *out, void *cuda_stream);

/*
 * Per-token quantisation prologue (page 4, per_token_cast: the value times a
 * precomputed inverse scale; page 2, quant mode 7 "dynamic pertoken"):
 *   a = max_j |x[i][j]|;  scale_out[i] = a / 127;  inv = a > 0 ? 127 / a : 0
 *   x1_out[i][j] = clamp(round_half_even(x[i][j] * inv), -127, 127)
 * in f32 with IEEE division.  x_bf16: bf16 bits [rows, k]; x1_out int8
 * [rows, k]; scale_out f32 [rows].  1 <= rows <= 2^31-1, k % 8 == 0,
 * 8 <= k <= 65536; x_bf16 and x1_out 16-byte aligned.
 * Errors: NULL_PTR, SHAPE, ALIGNMENT, UNSUPPORTED, CUDA.
 */
qgmm_status qgmm_per_token_quant(const uint16_t *x_bf16, int64_t rows, int64_t k, int8_t *x1_out,
                                 float *scale_out, void *cuda_stream);

/*
 * Per-32-group FP8 cast (page 4, "PTOAS issue 1568", 背景: per_token_cast
 * multiplies the bf16 values of a 256-element tile by inverse scale factors
 * broadcast over groups of 32 and converts the products to FLOAT8 E4M3FN, with
 * packed scale factors).  How a scale factor is chosen is not on the page; the
 * library takes one E8M0 power of two per group of 32, which puts the group's
 * largest magnitude in E4M3's top binade (the per-32 scale format that page 1's
 * MxA8W4 mode reads):
 *   a        = max_j |x[i][32g + j]| over the group (NaN skipped)
 *   sf[i][g] = max(0, biased f32 exponent of a - 8)      (E8M0 code: 2^(sf - 127))
 *   q[i][c]  = E4M3(x[i][c] * 2^(127 - sf[i][c/32])), round to nearest even,
 *              magnitudes past 448 (infinities too) saturate to 448, NaN -> 0x7F
 * so x ~= q * 2^(sf - 127); the product is exact, the conversion the only
 * rounding.  x_bf16: bf16 bits [rows, k]; q_out: E4M3 bytes [rows, k]; sf_out:
 * E8M0 bytes [rows, k/32] (four per 32-bit word: the packed layout).
 * 1 <= rows <= 2^31-1, k % 32 == 0, 32 <= k <= 65536; x_bf16 16-byte and q_out
 * 8-byte aligned.  Errors: NULL_PTR, SHAPE, ALIGNMENT, UNSUPPORTED, CUDA.
 */
qgmm_status qgmm_per_token_quant_mxfp8(const uint16_t *x_bf16, int64_t rows, int64_t k, uint8_t *q_out,
                                       uint8_t *sf_out, void *cuda_stream);

/*
 * Parity hook (no counterpart on the pages): the op's exact integer stage, so a
 * test can compare it bit for bit with an independent computation.
 * The raw accumulators acc_out[i][j] = sum_kk x1[i][kk] * W(g, kk, j) -- int32, or
 * for QGMM_W_FP8_E4M3 the f32 accumulator's bits in the same 4-byte slots --
 * for every row i below the groups' total, written by the same grouped GEMM
 * that qgmm_finalize runs (no epilogue arithmetic, no combine).  Rows at or
 * past the total are not written.  acc_out: int32 [m, n], 16-byte aligned.
 * `p` supplies m, k, n, e, weight_type, group_list_type and the tiling hint;
 * the workspace is the atomic-mode one (>= 256 bytes).
 * Errors: as qgmm_finalize, and DTYPE for QGMM_W_MXFP4 (use qgmm_debug_accum_mx).
 */
qgmm_status qgmm_debug_accum(const qgmm_problem *p, const int8_t *x1, const void *x2,
                             const int64_t *group_list, int32_t *acc_out, void *workspace,
                             size_t ws_bytes, void *cuda_stream);

/*
 * The parity hook for QGMM_W_MXFP4 (qgmm_debug_accum has no scale arguments;
 * no counterpart on the pages): the block-scaled f32 accumulators acc_out[i][j]
 * (see QGMM_W_MXFP4 above) for every row i below the groups' total, written by the
 * same kernel qgmm_finalize runs for this type, with no epilogue arithmetic and no
 * combine.  x1 E4M3 [m, k], sfa E8M0 [m, k/32], x2 E2M1 pairs (e, n, k/2), sfb E8M0
 * [e, n, k/32], acc_out f32 [m, n]; all 16-byte aligned, x2 32-byte aligned;
 * workspace of qgmm_finalize_workspace(p) bytes (its scale atoms).
 * Errors: as qgmm_debug_accum, and DTYPE for any other weight type.
 */
qgmm_status qgmm_debug_accum_mx(const qgmm_problem *p, const uint8_t *x1, const uint8_t *sfa, const void *x2,
                                const uint8_t *sfb, const int64_t *group_list, float *acc_out, void *workspace,
                                size_t ws_bytes, void *cuda_stream);

/*
 * Page 1, return values of both stages: each call returns a status code (an
 * aclnnStatus there, qgmm_status here).  Input errors only the device can see
 * are reported through the workspace status word instead, read by this call.
 * Synchronise `cuda_stream`, then copy the workspace status word written by
 * the last qgmm_finalize / qgmm_debug_accum on that workspace to *flags (host).
 * Returns QGMM_ERR_DEVICE_INPUT when any QGMM_DEV_* bit is set, QGMM_OK when
 * none is, QGMM_ERR_CUDA when the copy fails.
 */
qgmm_status qgmm_device_status(const void *workspace, uint32_t *flags, void *cuda_stream);

/* A static English description of a status code (page 1, return values: the
 * status code of each stage; here the qgmm_status values above). */
const char *qgmm_status_string(qgmm_status s);

#ifdef __cplusplus
}
#endif

#endif /* QGMM_H */
