/*
 * qgmm_probe.h -- C ABI of libqgmm_probe.so, the int8 tensor-core rate probe
 * that the grouped GEMM's roofline is read against.  (No counterpart on the
 * pages: it measures the device, not the op.)
 *
 * qgmm_probe_mma_i8 launches `clusters` CTA pairs (clusters of two CTAs, one
 * CTA per SM).  The leader of each pair issues `iters` back-to-back
 * tcgen05.mma.cta_group::2.kind::i8 instructions of shape M = 256, N = 256,
 * K = 32 on zeroed shared memory, accumulating into tensor memory, with no
 * memory traffic, then waits for them.  One launch performs
 *     clusters * iters * 256 * 256 * 32 multiply-accumulates (2 int ops each),
 * so timing it with CUDA events on `cuda_stream` gives the tensor pipe's int8
 * rate.  If `clock_out` (device, 2 x uint64) is not NULL, CTA 0 writes the SM
 * clock cycles and the %globaltimer nanoseconds of its issue-and-drain span.
 * `status` (device, uint32) gets bit 0 if the final bounded wait (one second)
 * ran out; the caller clears it.  Keep iters * 128 cycles well under a second.
 * Asynchronous on `cuda_stream`.  Returns 0, 2 (bad argument), 5 (device is
 * not compute capability 10.x) or 6 (a CUDA call failed).
 */
#ifndef QGMM_PROBE_H
#define QGMM_PROBE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

int qgmm_probe_mma_i8(int32_t clusters, int32_t iters, unsigned long long *clock_out, uint32_t *status,
                      void *cuda_stream);

/*
 * The same probe for other tile forms: N in [16, 256], a multiple of 16 (one
 * launch then performs clusters * iters * 256 * N * 32 MACs), and the operand
 * majors swapped when a_mn_major != 0 (A MN-major, B K-major; otherwise A
 * K-major, B MN-major).  qgmm_probe_mma_i8 is N = 256, a_mn_major = 0.
 */
int qgmm_probe_mma_i8_shape(int32_t clusters, int32_t iters, int32_t n, int32_t a_mn_major,
                            unsigned long long *clock_out, uint32_t *status, void *cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* QGMM_PROBE_H */
