// ep_plan.cu -- host-side offsets of the expert-parallel dispatch (page
// "aclnnAlltoAllvQuantGroupedMatMul", function description: AlltoAllv, then the
// permute to expert order, then each card's grouped matmul over its own experts).
// No device code: the exchange runs over NCCL and the matmuls through qgmm_finalize.
#include <cstdint>

#include "../../include/qgmm_ep.h"

#define QGMM_EP_API extern "C" __attribute__((visibility("default")))

namespace {
constexpr int64_t kMaxExpertsPerCard = 32;      // page 2: e in (0, 32]
constexpr int64_t kMaxExpertsInDomain = 256;    // page 2: e * epWorldSize at most 256
constexpr int64_t kBskLimit = 52428800;         // page 2: BSK in (0, 52428800)
}  // namespace

QGMM_EP_API qgmm_status qgmm_ep_plan(int32_t world, int32_t e, const int64_t *send_counts,
                                     const int64_t *recv_counts, int64_t *send_offsets, int64_t *recv_offsets,
                                     int64_t *group_counts, int64_t *totals)
{
    if (!send_counts || !recv_counts || !send_offsets || !recv_offsets || !group_counts || !totals)
        return QGMM_ERR_NULL_PTR;
    if (world < 1 || e < 1 || e > kMaxExpertsPerCard || int64_t(e) * world > kMaxExpertsInDomain)
        return QGMM_ERR_SHAPE;
    const int64_t chunks = int64_t(world) * e;
    int64_t bsk = 0, a = 0;
    for (int64_t c = 0; c < chunks; ++c) {
        if (send_counts[c] < 0 || recv_counts[c] < 0) return QGMM_ERR_SHAPE;
        bsk += send_counts[c];
        a += recv_counts[c];
        if (bsk >= kBskLimit || a >= (int64_t(1) << 40)) return QGMM_ERR_SHAPE;
    }
    if (bsk < 1) return QGMM_ERR_SHAPE;
    // send buffer: chunks in (destination card, expert) order
    int64_t row = 0;
    for (int64_t c = 0; c < chunks; ++c) {
        send_offsets[c] = row;
        row += send_counts[c];
    }
    // permuted receive buffer: expert-major, then source card
    row = 0;
    for (int32_t j = 0; j < e; ++j) {
        int64_t count = 0;
        for (int32_t s = 0; s < world; ++s) {
            const int64_t c = int64_t(s) * e + j;
            recv_offsets[c] = row;
            row += recv_counts[c];
            count += recv_counts[c];
        }
        group_counts[j] = count;
    }
    totals[0] = bsk;
    totals[1] = a;
    return QGMM_OK;
}
