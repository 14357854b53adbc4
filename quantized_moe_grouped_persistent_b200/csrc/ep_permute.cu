// ep_permute.cu -- the expert-parallel dispatch's on-device row copies: the chunks a
// card addresses to itself (page "aclnnAlltoAllvQuantGroupedMatMul": AlltoAllv, then
// the permute to expert order), moved to their permuted places by one kernel.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/qgmm_ep.h"

#define QGMM_EP_API extern "C" __attribute__((visibility("default")))

namespace {

struct ChunkTable {
    int64_t src[QGMM_EP_MAX_CHUNKS];   // byte offsets
    int64_t dst[QGMM_EP_MAX_CHUNKS];
    int64_t end[QGMM_EP_MAX_CHUNKS];   // running sum of the chunks' sizes, in units
    int32_t n;
};

// Units of W bytes (16 or 4), grid-stride over the chunks laid end to end; a thread
// finds its chunk by walking the (short) running-sum table.
template <typename U>
__global__ void permute_chunks_kernel(const uint8_t *__restrict__ src, uint8_t *__restrict__ dst,
                                      const __grid_constant__ ChunkTable t)
{
    const int64_t total = t.end[t.n - 1];
    int c = 0;
    for (int64_t u = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; u < total;
         u += int64_t(gridDim.x) * blockDim.x) {
        while (u >= t.end[c]) ++c;           // u only grows, so c does too
        const int64_t k = u - (c ? t.end[c - 1] : 0);
        reinterpret_cast<U *>(dst + t.dst[c])[k] = reinterpret_cast<const U *>(src + t.src[c])[k];
    }
}

}  // namespace

QGMM_EP_API qgmm_status qgmm_ep_permute_rows(const void *src, void *dst, int64_t row_bytes, int32_t nchunks,
                                             const int64_t *src_row, const int64_t *dst_row, const int64_t *count,
                                             void *cuda_stream)
{
    if (!src_row || !dst_row || !count) return QGMM_ERR_NULL_PTR;
    if (nchunks < 0 || nchunks > QGMM_EP_MAX_CHUNKS || row_bytes < 4 || row_bytes % 4) return QGMM_ERR_SHAPE;
    int64_t units_total = 0;
    const bool wide = row_bytes % 16 == 0 && (reinterpret_cast<uintptr_t>(src) & 15u) == 0 &&
                      (reinterpret_cast<uintptr_t>(dst) & 15u) == 0;
    const int64_t w = wide ? 16 : 4;
    ChunkTable t = {};
    for (int32_t c = 0; c < nchunks; ++c) {
        if (src_row[c] < 0 || dst_row[c] < 0 || count[c] < 0) return QGMM_ERR_SHAPE;
        if (count[c] == 0) continue;
        t.src[t.n] = src_row[c] * row_bytes;
        t.dst[t.n] = dst_row[c] * row_bytes;
        units_total += count[c] * row_bytes / w;
        t.end[t.n] = units_total;
        ++t.n;
    }
    if (t.n == 0) return QGMM_OK;
    if (!src || !dst) return QGMM_ERR_NULL_PTR;
    if ((reinterpret_cast<uintptr_t>(src) & 3u) || (reinterpret_cast<uintptr_t>(dst) & 3u)) return QGMM_ERR_ALIGNMENT;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess)
        return QGMM_ERR_CUDA;
    const int64_t blocks_needed = (units_total + 255) / 256;
    const int grid = static_cast<int>(blocks_needed < 4 * int64_t(sms) ? blocks_needed : 4 * int64_t(sms));
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    if (wide)
        permute_chunks_kernel<uint4><<<grid, 256, 0, st>>>(static_cast<const uint8_t *>(src),
                                                           static_cast<uint8_t *>(dst), t);
    else
        permute_chunks_kernel<uint32_t><<<grid, 256, 0, st>>>(static_cast<const uint8_t *>(src),
                                                              static_cast<uint8_t *>(dst), t);
    return cudaGetLastError() == cudaSuccess ? QGMM_OK : QGMM_ERR_CUDA;
}
