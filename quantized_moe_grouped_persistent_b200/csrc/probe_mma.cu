// probe_mma.cu -- libqgmm_probe.so: a measurement of the int8 tensor-core rate on
// this device, the denominator the grouped GEMM's roofline is read against.
//
// Each CTA pair (a cluster of two) allocates TMEM and its leader issues a stream
// of tcgen05.mma.cta_group::2.kind::i8 (M = 256, N = 256, K = 32) reading zeroed
// shared memory, with no memory traffic and no per-MMA handshake, then waits for
// them with one commit.  CTA 0 of the grid records its SM clock cycles and
// %globaltimer nanoseconds around the issue loop, so the caller can also derive
// MACs per clock per SM.  The waits are bounded like every wait in the library.
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx_sm100.cuh"

#define QGMM_PROBE_API extern "C" __attribute__((visibility("default")))

namespace qgmm {
namespace probe {

constexpr int OPERAND_BYTES = 2 * 16384;   // one 128-row A half and one 128-column B half

__global__ void __launch_bounds__(64, 1) mma_i8_pair_probe(int32_t iters, int32_t n, int32_t a_mn_major,
                                                           unsigned long long *clock_out, uint32_t *status)
{
    __shared__ __align__(1024) uint8_t operands[OPERAND_BYTES];
    __shared__ uint64_t drain;
    __shared__ uint32_t holder;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool leader = ptx::cluster_ctarank() == 0;
    for (int i = threadIdx.x; i < OPERAND_BYTES / 16; i += blockDim.x)
        reinterpret_cast<uint4 *>(operands)[i] = make_uint4(0u, 0u, 0u, 0u);
    ptx::fence_async_shared();   // the zeros are read by the tensor core (async proxy)
    if (threadIdx.x == 0) {
        ptx::mbar_init(&drain, 1);
        abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc_pair(&holder, 256);
        ptx::tmem_relinquish_pair();
    }
    ptx::tc_fence_before();
    ptx::cluster_sync();
    ptx::tc_fence_after();
    const uint32_t tmem = holder;
    if (warp == 0 && lane == 0 && leader) {
        // A K-major and B MN-major (the grouped GEMM's int8 pair tile), or A MN-major
        // and B K-major (the same tile transposed)
        const uint32_t idesc = a_mn_major ? ptx::idesc_i8(256, n, false, true) : ptx::idesc_i8(256, n, true);
        const uint32_t a0 = ptx::smem_addr(operands), b0 = a0 + 16384;
        const unsigned long long c0 = clock64();
        const uint64_t g0 = ptx::globaltimer();
        for (int32_t it = 0; it < iters; ++it) {
            const uint32_t kk = static_cast<uint32_t>(it & 3);
            const uint64_t kmaj = ptx::smem_desc_sw128(a0 + kk * 32, 16, 1024);
            const uint64_t mnmaj = ptx::smem_desc_sw128(b0 + kk * 32 * 128, 16384, 1024);
            const uint64_t adesc = a_mn_major ? mnmaj : kmaj, bdesc = a_mn_major ? kmaj : mnmaj;
            ptx::mma_i8_pair(tmem, adesc, bdesc, idesc, it != 0 ? 1u : 0u);
        }
        ptx::mma_commit_pair(ptx::map_to_rank(&drain, 0));
        volatile int *ab = &abort_flag;
        if (!ptx::mbar_wait(&drain, 0, ab)) atomicOr(status, 1u);
        const unsigned long long c1 = clock64();
        const uint64_t g1 = ptx::globaltimer();
        if (blockIdx.x == 0 && clock_out) {
            clock_out[0] = c1 - c0;
            clock_out[1] = g1 - g0;
        }
    }
    ptx::tc_fence_before();
    ptx::cluster_sync();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(tmem, 256);
    }
}

}  // namespace probe
}  // namespace qgmm

QGMM_PROBE_API int qgmm_probe_mma_i8_shape(int32_t clusters, int32_t iters, int32_t n, int32_t a_mn_major,
                                           unsigned long long *clock_out, uint32_t *status, void *cuda_stream)
{
    if (clusters < 1 || iters < 1 || !status || n < 16 || n > 256 || n % 16) return 2;
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return 6;
    if (major != 10) return 5;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters), 1, 1);
    cfg.blockDim = dim3(64, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = static_cast<cudaStream_t>(cuda_stream);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, qgmm::probe::mma_i8_pair_probe, iters, n, a_mn_major ? 1 : 0, clock_out, status) !=
        cudaSuccess)
        return 6;
    return cudaGetLastError() == cudaSuccess ? 0 : 6;
}

QGMM_PROBE_API int qgmm_probe_mma_i8(int32_t clusters, int32_t iters, unsigned long long *clock_out,
                                     uint32_t *status, void *cuda_stream)
{
    return qgmm_probe_mma_i8_shape(clusters, iters, 256, 0, clock_out, status, cuda_stream);
}
