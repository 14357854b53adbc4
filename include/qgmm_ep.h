/*
 * qgmm_ep.h -- host-side plan of the expert-parallel dispatch that feeds the
 * grouped GEMM (libqgmm.so).
 *
 * Page "aclnnAlltoAllvQuantGroupedMatMul", function description and the list of
 * shape variables: the routed experts are spread over the epWorldSize cards of an
 * EP domain, e experts per card.  Each card first exchanges token rows with every
 * other card (AlltoAllv), then permutes what it received so that the rows of each
 * of its own experts are contiguous, then runs the quantised grouped matmul over
 * its own experts only; the shared expert's quantised matmul runs beside it.
 *
 * The layout this plan fixes (the readings where the page's formulas are not
 * legible):
 *   - A card's send buffer holds its rows grouped by destination card, then by
 *     that card's local expert: send_counts[d*e + j] rows for card d's expert j,
 *     chunk (d, j) before (d, j+1) before (d+1, 0).  BSK = sum of send_counts.
 *   - recv_counts[s*e + j] rows arrive from card s for this card's expert j.
 *     After the exchange the rows are in source-card order (chunk (s, j) before
 *     (s, j+1) before (s+1, 0)); the permute puts them in expert order, and inside
 *     one expert in source-card order: chunk (j=0, s=0), (0, 1), ..., (1, 0), ...
 *     The row order inside a chunk is kept.  A = sum of recv_counts.
 *   - The grouped matmul then sees group_counts[j] = sum_s recv_counts[s*e + j]
 *     rows for expert j (a type-1 group list).
 *
 * The library computes the offsets and moves the chunks a card keeps for itself
 * (qgmm_ep_permute_rows); the exchange with other cards runs over NCCL (each chunk
 * received straight into its permuted place, so the permute costs no pass of its
 * own), and the matmuls through qgmm_finalize.
 */
#ifndef QGMM_EP_H
#define QGMM_EP_H

#include <stdint.h>

#include "qgmm.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Plan one card's dispatch.  A host function: every pointer is a HOST pointer,
 * caller-owned; it touches no device and launches nothing.
 *   world         cards in the EP domain, 1 <= world
 *   e             experts per card, 1 <= e <= 32, e * world <= 256
 *                 (page 2: e in (0, 32], e * epWorldSize at most 256)
 *   send_counts   int64 [world * e], each >= 0; their sum BSK must satisfy
 *                 1 <= BSK < 52428800 (page 2: BSK in (0, 52428800))
 *   recv_counts   int64 [world * e], each >= 0; their sum A may be 0 (a card that
 *                 receives nothing runs no grouped matmul)
 *   send_offsets  out, int64 [world * e]: first send-buffer row of chunk (d, j)
 *   recv_offsets  out, int64 [world * e]: first row of chunk (s, j) in the
 *                 permuted receive buffer
 *   group_counts  out, int64 [e]: rows of expert j after the permute
 *   totals        out, int64 [2]: {BSK, A}
 * Errors: NULL_PTR (any pointer NULL), SHAPE (a limit above broken, or a count
 * below zero).  On error nothing is written.
 */
qgmm_status qgmm_ep_plan(int32_t world, int32_t e, const int64_t *send_counts, const int64_t *recv_counts,
                         int64_t *send_offsets, int64_t *recv_offsets, int64_t *group_counts, int64_t *totals);

#define QGMM_EP_MAX_CHUNKS 32   /* chunks per qgmm_ep_permute_rows call: one per local expert */

/*
 * The chunks a card addresses to itself, moved to their permuted places by one
 * kernel on `cuda_stream` (asynchronous).  For each chunk c with count[c] > 0, rows
 * [src_row[c], src_row[c] + count[c]) of src are copied to rows [dst_row[c], ...)
 * of dst.  src and dst are DEVICE pointers (4-byte aligned; 16-byte copies are used
 * when both and row_bytes allow), rows row_bytes apart (row_bytes >= 4,
 * row_bytes % 4 == 0); the chunk table (src_row, dst_row, count: int64 [nchunks],
 * 0 <= nchunks <= QGMM_EP_MAX_CHUNKS) is in HOST memory and is passed to the kernel
 * by value, so the caller may reuse it as soon as the call returns.  Source and
 * destination ranges must not overlap.  Nothing is launched when every count is 0.
 * Errors: NULL_PTR, SHAPE (a limit above broken, or a negative entry), ALIGNMENT,
 * CUDA.
 */
qgmm_status qgmm_ep_permute_rows(const void *src, void *dst, int64_t row_bytes, int32_t nchunks,
                                 const int64_t *src_row, const int64_t *dst_row, const int64_t *count,
                                 void *cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* QGMM_EP_H */
