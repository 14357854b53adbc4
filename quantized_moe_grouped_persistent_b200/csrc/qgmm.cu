// qgmm.cu -- host side of libqgmm.so: argument checks, workspace sizing, tile
// planning, TMA tensor maps and kernel launches for the C ABI in qgmm.h.
//
// Two-stage call as on the "aclnnGroupedMatmulFinalizeRoutingWeightNzV2" page
// (first call validates and sizes the workspace, second call runs on a
// stream).  The library allocates no memory and keeps no per-call state.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "kernels.cuh"

#define QGMM_API extern "C" __attribute__((visibility("default")))

namespace qgmm {
namespace {

constexpr size_t kAlign = 256;
constexpr int64_t kMaxM = int64_t(1) << 24;
constexpr int kMaxDevices = 64;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned32(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

struct DeviceInfo {
    int sms = 0;
    int major = 0;
    bool attr_set[3][3] = {};
    bool mx_attr_set[3] = {};
    bool pair_attr_set[3][3] = {};
    int pair_clusters[3][3] = {};   // co-resident CTA pairs of the pair kernel, per epilogue and weight kind
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

qgmm_status device_info(DeviceInfo **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QGMM_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceInfo &d = g_dev[dev];
    if (d.sms == 0) {
        int sms = 0, major = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return QGMM_ERR_CUDA;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
            return QGMM_ERR_CUDA;
        d.sms = sms;
        d.major = major;
    }
    if (d.major != 10) return QGMM_ERR_UNSUPPORTED;
    *out = &d;
    return QGMM_OK;
}

qgmm_status check_problem(const qgmm_problem *p)
{
    if (!p) return QGMM_ERR_NULL_PTR;
    if (p->weight_type != QGMM_W_INT8 && p->weight_type != QGMM_W_INT4_PACKED_INT32 &&
        p->weight_type != QGMM_W_FP8_E4M3 && p->weight_type != QGMM_W_MXFP4)
        return QGMM_ERR_DTYPE;
    if (p->group_list_type != QGMM_GROUP_CUMSUM && p->group_list_type != QGMM_GROUP_COUNTS) return QGMM_ERR_DTYPE;
    if (p->row_index_type != QGMM_IDX_INT64 && p->row_index_type != QGMM_IDX_INT32) return QGMM_ERR_DTYPE;
    if (p->scale_type != QGMM_SCALE_F32 && p->scale_type != QGMM_SCALE_BF16) return QGMM_ERR_DTYPE;
    if (p->m < 1 || p->m > kMaxM) return QGMM_ERR_SHAPE;
    if (p->k < BK || p->k > 65536 || p->k % BK) return QGMM_ERR_SHAPE;
    if (p->n < BN || p->n > 65536 || p->n % BN) return QGMM_ERR_SHAPE;
    if (p->e < 1 || p->e > MAX_E) return QGMM_ERR_SHAPE;
    if (p->output_bs < 1 || p->output_bs > (int64_t(1) << 31) - 2) return QGMM_ERR_SHAPE;
    if (p->shared_bs < 0 || p->shared_offset < 0 || p->shared_offset + p->shared_bs > p->output_bs)
        return QGMM_ERR_SHAPE;
    if (p->deterministic != 0 && p->deterministic != 1) return QGMM_ERR_SHAPE;
    if (p->expected_m_per_expert < 0) return QGMM_ERR_SHAPE;
    if (p->transpose_x2 != 0 && p->transpose_x2 != 1) return QGMM_ERR_SHAPE;
    if (p->transpose_x2 && p->weight_type == QGMM_W_INT4_PACKED_INT32) return QGMM_ERR_UNSUPPORTED;
    if (p->weight_type == QGMM_W_MXFP4 && !p->transpose_x2) return QGMM_ERR_UNSUPPORTED;   // (e, n, k) only
    if (p->ld_x2 < 0 || p->ld_sb < 0 || p->ld_out < 0 || p->ld_shared < 0) return QGMM_ERR_SHAPE;
    if (p->ld_x2 && (p->ld_x2 < p->n || p->ld_x2 % 32)) return QGMM_ERR_SHAPE;
    if (p->ld_sb && (p->ld_sb < p->n || p->ld_sb % 8)) return QGMM_ERR_SHAPE;
    if (p->ld_out && (p->ld_out < p->n || p->ld_out % 8)) return QGMM_ERR_SHAPE;
    if (p->ld_shared && (p->ld_shared < p->n || p->ld_shared % 8)) return QGMM_ERR_SHAPE;
    // x2's per-expert stride ld_x2 * k bytes stays below the tensor map's 2^40 limit
    if (p->ld_x2 > (int64_t(1) << 23) || p->ld_sb > (int64_t(1) << 32) || p->ld_out > (int64_t(1) << 32) ||
        p->ld_shared > (int64_t(1) << 32))
        return QGMM_ERR_SHAPE;
    return QGMM_OK;
}

// Column strides, 0 meaning n.
int64_t ld_x2(const qgmm_problem *p) { return p->ld_x2 ? p->ld_x2 : p->n; }
int64_t ld_sb(const qgmm_problem *p) { return p->ld_sb ? p->ld_sb : p->n; }
int64_t ld_out(const qgmm_problem *p) { return p->ld_out ? p->ld_out : p->n; }
int64_t ld_shared(const qgmm_problem *p) { return p->ld_shared ? p->ld_shared : p->n; }

// Segments of the deterministic mode's bucket fill (det_fill_kernel): about 1024
// source rows each, at most 1024 segments, and the per-segment histograms
// (segments x output_bs int32) held to max(2^24, m*n/16) entries -- a sixteenth of
// the f32 rows y the same workspace holds.
int64_t det_segments(const qgmm_problem *p)
{
    int64_t s = std::min<int64_t>(1024, std::max<int64_t>(1, (p->m + 1023) / 1024));
    const int64_t cap = std::max<int64_t>(int64_t(1) << 24, p->m * p->n / 16);
    return std::max<int64_t>(1, std::min<int64_t>(s, cap / p->output_bs));
}

struct DetLayout {
    size_t y, counts, starts, list, total;
};

DetLayout det_layout(const qgmm_problem *p)
{
    DetLayout L;
    L.y = kAlign;
    L.counts = L.y + align_up(size_t(p->m) * size_t(p->n) * 4);
    L.starts = L.counts + align_up(size_t(det_segments(p)) * size_t(p->output_bs) * 4);
    L.list = L.starts + align_up(size_t(p->output_bs + 1) * 4);
    L.total = L.list + align_up(size_t(p->m) * 4);
    return L;
}

// MxA8W4: the scale atoms the MX kernel's producer bulk-copies (mx_sf_atoms_*_kernel),
// after the mode's own workspace: x1's for every m-tile of the walk (at most
// ceil(m/128) + e) and k-block, the weights' for every expert, 128-column tile and
// k-block; 512 bytes each.
struct MxAtoms {
    size_t rows, cols, total;
};

MxAtoms mx_atoms(const qgmm_problem *p)
{
    MxAtoms A;
    const size_t kb = size_t(p->k / BK);
    A.rows = p->deterministic ? det_layout(p).total : kAlign;
    A.cols = A.rows + align_up((size_t((p->m + BM - 1) / BM) + size_t(p->e)) * kb * MX_SF_BYTES);
    A.total = A.cols + align_up(size_t(p->e) * size_t(p->n / MX_BN) * kb * MX_SF_BYTES);
    return A;
}

size_t workspace_bytes(const qgmm_problem *p)
{
    if (p->weight_type == QGMM_W_MXFP4) return mx_atoms(p).total;
    return p->deterministic ? det_layout(p).total : kAlign;
}

// Write the MX kernel's scale atoms into the workspace (two kernels on `st`).
qgmm_status mx_write_atoms(const qgmm_problem *p, const DeviceInfo *dev, const uint8_t *sfa, const uint8_t *sfb,
                           const int64_t *group_list, uint8_t *ws, cudaStream_t st)
{
    const MxAtoms A = mx_atoms(p);
    const int64_t mt_max = (p->m + BM - 1) / BM + p->e;
    const int grid_rows = static_cast<int>(mt_max < 4 * int64_t(dev->sms) ? mt_max : 4 * int64_t(dev->sms));
    mx_sf_atoms_rows_kernel<<<grid_rows, 128, 0, st>>>(sfa, p->m, static_cast<int32_t>(p->k), group_list,
                                                       static_cast<int>(p->e), p->group_list_type,
                                                       reinterpret_cast<uint32_t *>(ws + A.rows));
    const int64_t col_tiles = p->e * (p->n / MX_BN);
    const int grid_cols = static_cast<int>(col_tiles < 8 * int64_t(dev->sms) ? col_tiles : 8 * int64_t(dev->sms));
    mx_sf_atoms_cols_kernel<<<grid_cols, 128, 0, st>>>(sfb, static_cast<int>(p->e), static_cast<int32_t>(p->n),
                                                       ld_sb(p), static_cast<int32_t>(p->k),
                                                       reinterpret_cast<uint32_t *>(ws + A.cols));
    return cudaGetLastError() == cudaSuccess ? QGMM_OK : QGMM_ERR_CUDA;
}

int env_int(const char *name, int dflt)
{
    const char *v = std::getenv(name);
    if (!v || !*v) return dflt;
    return std::atoi(v);
}

struct Plan {
    int tile_rows;
    int slab_ntiles;
    int grid;
    bool pair;   // CTA-pair kernel (tcgen05 cta_group::2, 256-row tiles)
    int tail_mode;   // pair path: where a group's odd last <= 128 rows run (launch_gemm)
};

Plan make_plan(const qgmm_problem *p, int sms, int epi)
{
    Plan pl;
    const int64_t hint = p->expected_m_per_expert > 0 ? p->expected_m_per_expert : (p->m + p->e - 1) / p->e;
    pl.tile_rows = hint <= 16 ? 16 : hint <= 32 ? 32 : hint <= 64 ? 64 : 128;
    const int forced_rows = env_int("QGMM_TILE_ROWS", 0);
    if (forced_rows == 16 || forced_rows == 32 || forced_rows == 64 || forced_rows == 128) pl.tile_rows = forced_rows;

    const int NT = static_cast<int>(p->n / BN);
    int sw = NT;
    if (epi == EPI_ATOMIC) {
        // Output slab (output_bs x slab columns, f32): a wider slab lets the combine's
        // reductions miss L2, a narrower one re-reads x1 once per slab.  The budget
        // is half of x1's bytes, clamped to [32 MB, 128 MB (about L2)]: large prefill
        // (x1 268 MB) keeps ~117 MB slabs, W4A8 (x1 67 MB) ~29 MB slabs -- the best
        // widths measured for each (2.29 vs 2.32-2.56 ms; 0.733 vs 0.754 ms).
        const double per_ntile = double(p->output_bs) * BN * 4.0;
        const double x1_bytes = double(p->m) * double(p->k);
        const double budget = std::min(128.0 * 1024 * 1024, std::max(32.0 * 1024 * 1024, x1_bytes / 2));
        sw = 1;
        for (int d = 1; d <= NT; ++d)
            if (NT % d == 0 && d * per_ntile <= budget) sw = d;
    }
    const int forced_sw = env_int("QGMM_SLAB_NTILES", 0);
    if (forced_sw > 0 && forced_sw <= NT && NT % forced_sw == 0) sw = forced_sw;
    pl.slab_ntiles = sw;

    // Full-height tiles of int8 weights run on CTA pairs; decode-sized tiles run on
    // single CTAs.  int4 weights run on single CTAs unless QGMM_PAIR_W4=1: the pair
    // form (each CTA unpacks its own 128-column half) is exact but measured slower
    // (W4A8 at 256 and 512 rows per expert: 1.22 / 2.07 ms against 0.89 / 1.64 ms).
    if (p->weight_type == QGMM_W_MXFP4) pl.tile_rows = 128;   // the MX kernel's tile: 128 x 128
    pl.pair = pl.tile_rows == 128 && env_int("QGMM_PAIR", 1) != 0 && p->weight_type != QGMM_W_MXFP4 &&
              (p->weight_type != QGMM_W_INT4_PACKED_INT32 || env_int("QGMM_PAIR_W4", 0) != 0);
    const int rows_per_tile = pl.pair ? 256 : pl.tile_rows;
    const int64_t max_mt = (p->m + rows_per_tile - 1) / rows_per_tile + p->e;
    const int64_t max_tiles = max_mt * NT;
    pl.grid = static_cast<int>(max_tiles < sms ? max_tiles : sms);
    if (pl.grid < 1) pl.grid = 1;
    if (pl.pair) pl.grid = static_cast<int>(2 * (max_tiles < sms / 2 ? max_tiles : sms / 2));

    // Tail tiles (at most one per group and n-tile) cost a second launch's fill and
    // drain in mode 1, and a pair's full weight feed for <= 128 rows in mode 2.  Mode
    // 2 wins when the tail launch would be short (<= 8 waves of single CTAs) and so is
    // the pair launch (<= 32 waves of pairs): measured 5-10% faster at m = 4096-16384
    // over 32 experts, n = 7168; mode 1 is 2-5% faster at 256 experts (~30 tail waves)
    // and ties or wins once the pair launch is longer.
    pl.tail_mode = 1;
    if (pl.pair) {
        const double tail_waves = double(p->e) * NT / sms;
        const double pair_waves = double(p->m) / 256.0 * NT / (sms / 2);
        if (tail_waves <= 8.0 && pair_waves <= 32.0) pl.tail_mode = 2;
    }
    const int forced_tails = env_int("QGMM_PAIR_TAILS", -1);
    if (forced_tails >= 0 && forced_tails <= 2) pl.tail_mode = forced_tails;
    return pl;
}

// x1 map (box: 128 bytes x tile_rows) and weight map: int8 box 128 columns x BK
// rows (transposed int8: BK bytes x 128 n-rows); packed int4 box w4_box_words
// int32 words (8 columns each) x BK rows --
// 32 words (256 columns) for the single-CTA kernel, 16 (one CTA's 128 columns)
// for the CTA pair.
qgmm_status make_maps(const qgmm_problem *p, const int8_t *x1, const void *x2, int tile_rows, int w4_box_words,
                      CUtensorMap *ma, CUtensorMap *mb)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return QGMM_ERR_CUDA;
    {
        const cuuint64_t gdim[2] = {cuuint64_t(p->k), cuuint64_t(p->m)};
        const cuuint64_t gstride[1] = {cuuint64_t(p->k)};
        const cuuint32_t box[2] = {cuuint32_t(BK), cuuint32_t(tile_rows)};
        const cuuint32_t es[2] = {1, 1};
        if (enc(ma, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(x1), gdim, gstride, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return QGMM_ERR_CUDA;
    }
    const cuuint64_t ld = cuuint64_t(ld_x2(p));
    const bool bytes = p->weight_type != QGMM_W_INT4_PACKED_INT32;   // int8 or E4M3: one byte per element
    if (p->weight_type == QGMM_W_MXFP4) {
        // E2M1 pairs (e, n, k/2) through the padded 4-bit type: dimensions count 4-bit
        // values, strides bytes; a box of 128 k-values (64 bytes read, 128 bytes
        // written: each 16 values' 8 bytes, then 8 unused) x 128 n-rows, 128-byte
        // swizzle -- the layout of a K-major 8-bit tile.  The type needs a 32-byte
        // aligned base and strides that are multiples of 32 bytes (k % 128 == 0 gives them).
        const cuuint64_t kb = cuuint64_t(p->k / 2);
        const cuuint64_t gdim[3] = {cuuint64_t(p->k), cuuint64_t(p->n), cuuint64_t(p->e)};
        const cuuint64_t gstride[2] = {kb, kb * ld};
        const cuuint32_t box[3] = {cuuint32_t(BK), cuuint32_t(MX_BN), 1};
        const cuuint32_t es[3] = {1, 1, 1};
        if (enc(mb, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 3, const_cast<void *>(x2), gdim, gstride, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return QGMM_ERR_CUDA;
    } else if (bytes && p->transpose_x2) {
        // (e, n, k): K-major B, a box of 128 K bytes x 128 n-rows -- the x1 tile's layout
        const cuuint64_t gdim[3] = {cuuint64_t(p->k), cuuint64_t(p->n), cuuint64_t(p->e)};
        const cuuint64_t gstride[2] = {cuuint64_t(p->k), cuuint64_t(p->k) * ld};
        const cuuint32_t box[3] = {cuuint32_t(BK), 128, 1};
        const cuuint32_t es[3] = {1, 1, 1};
        if (enc(mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(x2), gdim, gstride, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return QGMM_ERR_CUDA;
    } else if (bytes) {
        const cuuint64_t gdim[3] = {cuuint64_t(p->n), cuuint64_t(p->k), cuuint64_t(p->e)};
        const cuuint64_t gstride[2] = {ld, ld * cuuint64_t(p->k)};
        const cuuint32_t box[3] = {128, cuuint32_t(BK), 1};
        const cuuint32_t es[3] = {1, 1, 1};
        if (enc(mb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(x2), gdim, gstride, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return QGMM_ERR_CUDA;
    } else {
        const cuuint64_t words = cuuint64_t(p->n / 8);
        const cuuint64_t gdim[3] = {words, cuuint64_t(p->k), cuuint64_t(p->e)};
        const cuuint64_t gstride[2] = {ld / 8 * 4, ld / 8 * 4 * cuuint64_t(p->k)};
        const cuuint32_t box[3] = {cuuint32_t(w4_box_words), cuuint32_t(BK), 1};
        const cuuint32_t es[3] = {1, 1, 1};
        if (enc(mb, CU_TENSOR_MAP_DATA_TYPE_INT32, 3, const_cast<void *>(x2), gdim, gstride, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return QGMM_ERR_CUDA;
    }
    return QGMM_OK;
}

template <int EPI>
qgmm_status launch_mx_t(DeviceInfo *dev, const Plan &pl, const CUtensorMap &ma, const CUtensorMap &mb,
                        const GemmArgs &a, cudaStream_t st)
{
    auto kern = grouped_gemm_mx_kernel<EPI>;
    const size_t smem = MxCfg::SMEM_BYTES;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!dev->mx_attr_set[EPI]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
                return QGMM_ERR_CUDA;
            dev->mx_attr_set[EPI] = true;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(pl.grid), 1, 1);
    cfg.blockDim = dim3(MxCfg::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    GemmArgs am = a;
    am.slab_ntiles = 2 * pl.slab_ntiles;   // the plan counts 256-column tiles, the MX kernel 128-column ones
    if (cudaLaunchKernelEx(&cfg, kern, ma, mb, am) != cudaSuccess) return QGMM_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? QGMM_OK : QGMM_ERR_CUDA;
}

// Weight kinds of the kernel instantiations: int8, packed int4, E4M3.
constexpr int WK_INT8 = 0, WK_INT4 = 1, WK_F8 = 2;

int weight_kind(const qgmm_problem *p)
{
    return p->weight_type == QGMM_W_INT4_PACKED_INT32 ? WK_INT4 : p->weight_type == QGMM_W_FP8_E4M3 ? WK_F8 : WK_INT8;
}

template <int EPI, bool W4, bool F8 = false>
qgmm_status launch_gemm_t(DeviceInfo *dev, const Plan &pl, const CUtensorMap &ma, const CUtensorMap &mb,
                          const GemmArgs &a, cudaStream_t st)
{
    auto kern = grouped_gemm_kernel<EPI, W4, F8>;
    const size_t smem = GemmCfg<W4>::SMEM_BYTES;
    const int wk = W4 ? WK_INT4 : F8 ? WK_F8 : WK_INT8;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!dev->attr_set[EPI][wk]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
                return QGMM_ERR_CUDA;
            dev->attr_set[EPI][wk] = true;
        }
    }
    // Programmatic dependent launch: the GEMM's prologue and mainloop may
    // overlap the preceding output-init kernel; its epilogue waits for it.
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(pl.grid), 1, 1);
    cfg.blockDim = dim3(GemmCfg<W4>::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, ma, mb, a) != cudaSuccess) return QGMM_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? QGMM_OK : QGMM_ERR_CUDA;
}

template <int EPI, bool W4, bool F8 = false>
qgmm_status launch_pair_t(DeviceInfo *dev, const Plan &pl, const CUtensorMap &ma, const CUtensorMap &mb,
                          const GemmArgs &a, cudaStream_t st)
{
    auto kern = grouped_gemm_pair_kernel<EPI, W4, F8>;
    const int wk = W4 ? WK_INT4 : F8 ? WK_F8 : WK_INT8;
    const size_t smem = PairCfg<W4>::SMEM_BYTES;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(PairCfg<W4>::THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;   // the occupancy query below uses the cluster shape only
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!dev->pair_attr_set[EPI][wk]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
                return QGMM_ERR_CUDA;
            cfg.gridDim = dim3(static_cast<unsigned>(dev->sms & ~1), 1, 1);
            int clusters = 0;
            if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess || clusters < 1)
                return QGMM_ERR_CUDA;
            dev->pair_clusters[EPI][wk] = clusters;
            dev->pair_attr_set[EPI][wk] = true;
        }
    }
    int grid = pl.grid;
    if (grid > 2 * dev->pair_clusters[EPI][wk]) grid = 2 * dev->pair_clusters[EPI][wk];
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, kern, ma, mb, a) != cudaSuccess) return QGMM_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? QGMM_OK : QGMM_ERR_CUDA;
}

// Kernel launches of one grouped GEMM under plan `pl` (launch_gemm below).
int gemm_launches(const Plan &pl) { return pl.pair && pl.tail_mode == 1 ? 2 : 1; }

// mb: weight map of the main launch; mb_tail: weight map of the single-CTA
// tail launch (they differ only for int4 weights on CTA pairs).
// One launch of the pair kernel / the single-CTA kernel for a runtime epilogue and weight kind.
template <int EPI>
qgmm_status launch_pair_wk(int wk, DeviceInfo *dev, const Plan &pl, const CUtensorMap &ma, const CUtensorMap &mb,
                           const GemmArgs &a, cudaStream_t st)
{
    switch (wk) {
    case WK_INT4: return launch_pair_t<EPI, true>(dev, pl, ma, mb, a, st);
    case WK_F8: return launch_pair_t<EPI, false, true>(dev, pl, ma, mb, a, st);
    default: return launch_pair_t<EPI, false>(dev, pl, ma, mb, a, st);
    }
}

template <int EPI>
qgmm_status launch_single_wk(int wk, DeviceInfo *dev, const Plan &pl, const CUtensorMap &ma, const CUtensorMap &mb,
                             const GemmArgs &a, cudaStream_t st)
{
    switch (wk) {
    case WK_INT4: return launch_gemm_t<EPI, true>(dev, pl, ma, mb, a, st);
    case WK_F8: return launch_gemm_t<EPI, false, true>(dev, pl, ma, mb, a, st);
    default: return launch_gemm_t<EPI, false>(dev, pl, ma, mb, a, st);
    }
}

qgmm_status launch_pair_any(int epi, int wk, DeviceInfo *dev, const Plan &pl, const CUtensorMap &ma,
                            const CUtensorMap &mb, const GemmArgs &a, cudaStream_t st)
{
    switch (epi) {
    case EPI_ATOMIC: return launch_pair_wk<EPI_ATOMIC>(wk, dev, pl, ma, mb, a, st);
    case EPI_STORE_Y: return launch_pair_wk<EPI_STORE_Y>(wk, dev, pl, ma, mb, a, st);
    default: return launch_pair_wk<EPI_RAW_ACC>(wk, dev, pl, ma, mb, a, st);
    }
}

qgmm_status launch_single_any(int epi, int wk, DeviceInfo *dev, const Plan &pl, const CUtensorMap &ma,
                              const CUtensorMap &mb, const GemmArgs &a, cudaStream_t st)
{
    switch (epi) {
    case EPI_ATOMIC: return launch_single_wk<EPI_ATOMIC>(wk, dev, pl, ma, mb, a, st);
    case EPI_STORE_Y: return launch_single_wk<EPI_STORE_Y>(wk, dev, pl, ma, mb, a, st);
    default: return launch_single_wk<EPI_RAW_ACC>(wk, dev, pl, ma, mb, a, st);
    }
}

qgmm_status launch_gemm(int epi, DeviceInfo *dev, const qgmm_problem *p, const Plan &pl, const CUtensorMap &ma,
                        const CUtensorMap &mb, const CUtensorMap &mb_tail, const GemmArgs &a, cudaStream_t st)
{
    const int wk = weight_kind(p);
    if (std::getenv("QGMM_LOG"))
        std::fprintf(stderr,
                     "qgmm: gemm epi=%d weights=%d pair=%d m=%lld k=%lld n=%lld e=%lld tile_rows=%d slab=%d grid=%d\n",
                     epi, wk, int(pl.pair), (long long)p->m, (long long)p->k, (long long)p->n, (long long)p->e,
                     pl.tile_rows, pl.slab_ntiles, pl.grid);
    if (p->weight_type == QGMM_W_MXFP4) {
        Plan pm = pl;
        const int64_t tiles = ((p->m + BM - 1) / BM + p->e) * (p->n / MX_BN);
        pm.grid = static_cast<int>(tiles < dev->sms ? tiles : dev->sms);
        switch (epi) {
        case EPI_ATOMIC: return launch_mx_t<EPI_ATOMIC>(dev, pm, ma, mb, a, st);
        case EPI_STORE_Y: return launch_mx_t<EPI_STORE_Y>(dev, pm, ma, mb, a, st);
        default: return launch_mx_t<EPI_RAW_ACC>(dev, pm, ma, mb, a, st);
        }
    }
    if (pl.pair) {
        // Pairs of 128-row half tiles on CTA pairs.  A group's odd last half tile
        // (its final <= 128 rows) goes, by pl.tail_mode (make_plan's choice, or
        // QGMM_PAIR_TAILS):
        //   1 to a single-CTA launch right after the pair launch;
        //   2 to an M = 128 pair tile (64 rows per CTA) after the group's other tiles;
        //   0 to a full 256-row pair tile padded with rows it ignores.
        // All three give identical results.
        const int tail_mode = pl.tail_mode;
        const bool tails = tail_mode == 1;
        GemmArgs ap = a;
        ap.sched = tail_mode == 2 ? SCHED_PAIRS_TAIL128 : tails ? SCHED_PAIRS : SCHED_PAIRS_ALL;
        const qgmm_status s = launch_pair_any(epi, wk, dev, pl, ma, mb, ap, st);
        if (s != QGMM_OK || !tails) return s;
        GemmArgs at = a;
        at.sched = SCHED_TAILS;
        Plan pt = pl;
        const int64_t tail_tiles = p->e * (p->n / BN);
        pt.grid = static_cast<int>(tail_tiles < dev->sms ? tail_tiles : dev->sms);
        return launch_single_any(epi, wk, dev, pt, ma, mb_tail, at, st);
    }
    return launch_single_any(epi, wk, dev, pl, ma, mb, a, st);
}

GemmArgs base_args(const qgmm_problem *p, const int64_t *group_list, const Plan &pl, uint32_t *status)
{
    GemmArgs a;
    std::memset(&a, 0, sizeof a);
    a.group_list = group_list;
    a.m = p->m;
    a.e = static_cast<int32_t>(p->e);
    a.group_list_type = p->group_list_type;
    a.k = static_cast<int32_t>(p->k);
    a.n = static_cast<int32_t>(p->n);
    a.tile_rows = pl.tile_rows;
    a.sched = SCHED_TILES;
    // Test hook for the failure path: with QGMM_TEST_STALL_PRODUCER=1 the GEMM's
    // producer issues no copy, every consumer wait runs out after its one-second
    // bound, the kernel sets QGMM_DEV_TIMEOUT, frees its TMEM and returns.
    a.stall_producer = env_int("QGMM_TEST_STALL_PRODUCER", 0) != 0 ? 1 : 0;
    a.slab_ntiles = pl.slab_ntiles;
    a.b_kmajor = p->transpose_x2;
    a.row_index_type = p->row_index_type;
    a.output_bs = p->output_bs;
    a.store_rows = p->m;
    a.status = status;
    a.ld_sb = ld_sb(p);
    a.ldd = p->n;   // y and acc_out rows; the atomic combine's launch sets ld_out
    return a;
}

int grid_for(int64_t work, int per_block, int sms, int blocks_per_sm)
{
    int64_t g = (work + per_block - 1) / per_block;
    const int64_t cap = int64_t(sms) * blocks_per_sm;
    if (g > cap) g = cap;
    if (g < 1) g = 1;
    return static_cast<int>(g);
}

}  // namespace
}  // namespace qgmm

using namespace qgmm;

QGMM_API qgmm_status qgmm_finalize_workspace(const qgmm_problem *p, size_t *ws_bytes)
{
    if (!ws_bytes) return QGMM_ERR_NULL_PTR;
    const qgmm_status s = check_problem(p);
    if (s != QGMM_OK) return s;
    *ws_bytes = workspace_bytes(p);
    return QGMM_OK;
}

namespace {
qgmm_status finalize_impl(const qgmm_problem *p, const int8_t *x1, const void *x2, const void *scale,
                          const float *pertoken_scale, const int64_t *group_list, const float *logit,
                          const void *row_index, const float *bias, const uint16_t *shared_input, float *out,
                          void *workspace, size_t ws_bytes, void *cuda_stream, cudaEvent_t ev_begin,
                          cudaEvent_t ev_end)
{
    qgmm_status s = check_problem(p);
    if (s != QGMM_OK) return s;
    if (!x1 || !x2 || !group_list || !out || !workspace) return QGMM_ERR_NULL_PTR;
    if (p->shared_bs > 0 && !shared_input) return QGMM_ERR_NULL_PTR;
    const bool mx = p->weight_type == QGMM_W_MXFP4;
    if (mx && (!scale || !pertoken_scale)) return QGMM_ERR_NULL_PTR;   // the block scales are required
    if (!aligned16(x1) || !aligned16(x2) || !aligned16(out) || (p->shared_bs > 0 && !aligned16(shared_input)) ||
        (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 || !aligned16(scale) || !aligned16(bias) ||
        (mx && (!aligned16(pertoken_scale) || !aligned32(x2))))   // the padded 4-bit copy's base: 32 bytes
        return QGMM_ERR_ALIGNMENT;
    if (ws_bytes < workspace_bytes(p)) return QGMM_ERR_WORKSPACE_TOO_SMALL;
    DeviceInfo *dev = nullptr;
    if ((s = device_info(&dev)) != QGMM_OK) return s;

    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    uint32_t *status = static_cast<uint32_t *>(workspace);
    const int epi = p->deterministic ? EPI_STORE_Y : EPI_ATOMIC;
    const Plan pl = make_plan(p, dev->sms, epi);
    CUtensorMap ma, mb, mb_tail;
    if ((s = make_maps(p, x1, x2, pl.tile_rows, pl.pair ? 16 : 32, &ma, &mb)) != QGMM_OK) return s;
    mb_tail = mb;
    if (pl.pair && p->weight_type == QGMM_W_INT4_PACKED_INT32 &&
        (s = make_maps(p, x1, x2, pl.tile_rows, 32, &ma, &mb_tail)) != QGMM_OK)
        return s;

    GemmArgs a = base_args(p, group_list, pl, status);
    if (mx) {
        // MxA8W4: scale and pertoken_scale hold the E8M0 block scales of the weights
        // and of x1; the epilogue's own scale and pertokenScale are then 1.  The MX
        // kernel reads them as per-stage atoms written into the workspace first.
        if ((s = mx_write_atoms(p, dev, reinterpret_cast<const uint8_t *>(pertoken_scale),
                                static_cast<const uint8_t *>(scale), group_list, static_cast<uint8_t *>(workspace),
                                st)) != QGMM_OK)
            return s;
        const MxAtoms A = mx_atoms(p);
        a.sfa = static_cast<const uint8_t *>(workspace) + A.rows;
        a.sfb = static_cast<const uint8_t *>(workspace) + A.cols;
    } else {
        a.scale = scale;
        a.scale_bf16 = p->scale_type == QGMM_SCALE_BF16;
        a.pts = pertoken_scale;
    }
    a.logit = logit;
    a.bias = bias;
    a.row_index = row_index;
    const uint16_t *shared = p->shared_bs > 0 ? shared_input : nullptr;

    if (!p->deterministic && !row_index && !shared) {
        // Identity routing without sharedInput: an output row receives at most one
        // source row, so the GEMM stores it (as 0 + y, the combine's value) instead of
        // reducing into a zeroed output; only the rows past the groups' total are zeroed.
        output_tail_zero_kernel<<<grid_for(p->output_bs, 1, dev->sms, 2), 256, 0, st>>>(
            out, p->output_bs, static_cast<int32_t>(p->n), ld_out(p), group_list, static_cast<int>(p->e),
            p->group_list_type, p->m, status);
        if (cudaGetLastError() != cudaSuccess) return QGMM_ERR_CUDA;
        a.out = out;
        a.ldd = ld_out(p);
        a.store_rows = p->output_bs;
        if (ev_begin && cudaEventRecord(ev_begin, st) != cudaSuccess) return QGMM_ERR_CUDA;
        if ((s = launch_gemm(EPI_STORE_Y, dev, p, pl, ma, mb, mb_tail, a, st)) != QGMM_OK) return s;
        if (ev_end && cudaEventRecord(ev_end, st) != cudaSuccess) return QGMM_ERR_CUDA;
        return QGMM_OK;
    }
    if (!p->deterministic) {
        output_init_kernel<<<grid_for(p->output_bs, 1, dev->sms, 2), 256, 0, st>>>(
            out, p->output_bs, static_cast<int32_t>(p->n), ld_out(p), shared, ld_shared(p), p->shared_bs,
            p->shared_offset, status);
        if (cudaGetLastError() != cudaSuccess) return QGMM_ERR_CUDA;
        a.out = out;
        a.ldd = ld_out(p);
        if (ev_begin && cudaEventRecord(ev_begin, st) != cudaSuccess) return QGMM_ERR_CUDA;
        if ((s = launch_gemm(EPI_ATOMIC, dev, p, pl, ma, mb, mb_tail, a, st)) != QGMM_OK) return s;
        if (ev_end && cudaEventRecord(ev_end, st) != cudaSuccess) return QGMM_ERR_CUDA;
        return QGMM_OK;
    }

    const DetLayout L = det_layout(p);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    float *y = reinterpret_cast<float *>(ws + L.y);
    int32_t *counts = reinterpret_cast<int32_t *>(ws + L.counts);
    int32_t *starts = reinterpret_cast<int32_t *>(ws + L.starts);
    int32_t *list = reinterpret_cast<int32_t *>(ws + L.list);
    const int e = static_cast<int>(p->e);
    const int64_t nseg = det_segments(p);
    // destination buckets of source rows, filled in ascending source-row order
    det_clear_kernel<<<grid_for(nseg * p->output_bs, 256, dev->sms, 4), 256, 0, st>>>(counts, nseg * p->output_bs,
                                                                                      status);
    det_hist_kernel<<<grid_for(p->m, 256, dev->sms, 4), 256, 0, st>>>(
        group_list, e, p->group_list_type, p->m, row_index, p->row_index_type, p->output_bs,
        static_cast<int32_t>(nseg), counts, status);
    det_colscan_kernel<<<grid_for(p->output_bs, 256, dev->sms, 4), 256, 0, st>>>(counts, static_cast<int32_t>(nseg),
                                                                                 p->output_bs, starts);
    det_scan_kernel<<<1, 1024, 0, st>>>(starts, p->output_bs);
    det_fill_kernel<<<grid_for(nseg, 8, dev->sms, 8), 256, 0, st>>>(
        group_list, e, p->group_list_type, p->m, row_index, p->row_index_type, p->output_bs,
        static_cast<int32_t>(nseg), counts, starts, list);
    if (cudaGetLastError() != cudaSuccess) return QGMM_ERR_CUDA;
    a.out = y;
    if (ev_begin && cudaEventRecord(ev_begin, st) != cudaSuccess) return QGMM_ERR_CUDA;
    if ((s = launch_gemm(EPI_STORE_Y, dev, p, pl, ma, mb, mb_tail, a, st)) != QGMM_OK) return s;
    if (ev_end && cudaEventRecord(ev_end, st) != cudaSuccess) return QGMM_ERR_CUDA;
    det_reduce_kernel<<<grid_for(p->output_bs, 1, dev->sms, 8), 256, 0, st>>>(
        out, y, static_cast<int32_t>(p->n), ld_out(p), starts, list, p->output_bs, shared, ld_shared(p),
        p->shared_bs, p->shared_offset);
    return cudaGetLastError() == cudaSuccess ? QGMM_OK : QGMM_ERR_CUDA;
}
}  // namespace

QGMM_API qgmm_status qgmm_finalize(const qgmm_problem *p, const int8_t *x1, const void *x2, const void *scale,
                                   const float *pertoken_scale, const int64_t *group_list, const float *logit,
                                   const void *row_index, const float *bias, const uint16_t *shared_input,
                                   float *out, void *workspace, size_t ws_bytes, void *cuda_stream)
{
    return finalize_impl(p, x1, x2, scale, pertoken_scale, group_list, logit, row_index, bias, shared_input, out,
                         workspace, ws_bytes, cuda_stream, nullptr, nullptr);
}

QGMM_API qgmm_status qgmm_finalize_profiled(const qgmm_problem *p, const int8_t *x1, const void *x2,
                                            const void *scale, const float *pertoken_scale,
                                            const int64_t *group_list, const float *logit, const void *row_index,
                                            const float *bias, const uint16_t *shared_input, float *out,
                                            void *workspace, size_t ws_bytes, void *cuda_stream,
                                            void *gemm_begin_event, void *gemm_end_event)
{
    if (!gemm_begin_event || !gemm_end_event) return QGMM_ERR_NULL_PTR;
    return finalize_impl(p, x1, x2, scale, pertoken_scale, group_list, logit, row_index, bias, shared_input, out,
                         workspace, ws_bytes, cuda_stream, static_cast<cudaEvent_t>(gemm_begin_event),
                         static_cast<cudaEvent_t>(gemm_end_event));
}

QGMM_API qgmm_status qgmm_finalize_launches(const qgmm_problem *p, int32_t *launches)
{
    qgmm_status s = check_problem(p);
    if (s != QGMM_OK) return s;
    if (!launches) return QGMM_ERR_NULL_PTR;
    DeviceInfo *dev = nullptr;
    if ((s = device_info(&dev)) != QGMM_OK) return s;
    const Plan pl = make_plan(p, dev->sms, p->deterministic ? EPI_STORE_Y : EPI_ATOMIC);
    // atomic: output init; deterministic: clear, histogram, column scan, scan, fill, then the reduce;
    // MxA8W4 also writes its two kinds of scale atoms first
    *launches = (p->deterministic ? 6 : 1) + gemm_launches(pl) + (p->weight_type == QGMM_W_MXFP4 ? 2 : 0);
    return QGMM_OK;
}

QGMM_API qgmm_status qgmm_plan(const qgmm_problem *p, int32_t sms, qgmm_plan_info *info)
{
    qgmm_status s = check_problem(p);
    if (s != QGMM_OK) return s;
    if (!info) return QGMM_ERR_NULL_PTR;
    if (sms < 2) return QGMM_ERR_SHAPE;
    const Plan pl = make_plan(p, sms, p->deterministic ? EPI_STORE_Y : EPI_ATOMIC);
    info->tile_rows = pl.tile_rows;
    info->pair = pl.pair ? 1 : 0;
    info->tail_mode = pl.tail_mode;
    info->slab_ntiles = pl.slab_ntiles;
    info->grid = pl.grid;
    info->gemm_launches = gemm_launches(pl);
    return QGMM_OK;
}

QGMM_API qgmm_status qgmm_debug_accum(const qgmm_problem *p, const int8_t *x1, const void *x2,
                                      const int64_t *group_list, int32_t *acc_out, void *workspace,
                                      size_t ws_bytes, void *cuda_stream)
{
    qgmm_status s = check_problem(p);
    if (s != QGMM_OK) return s;
    if (p->weight_type == QGMM_W_MXFP4) return QGMM_ERR_DTYPE;   // needs the block scales: qgmm_debug_accum_mx
    if (!x1 || !x2 || !group_list || !acc_out || !workspace) return QGMM_ERR_NULL_PTR;
    if (!aligned16(x1) || !aligned16(x2) || !aligned16(acc_out) ||
        (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
        return QGMM_ERR_ALIGNMENT;
    if (ws_bytes < kAlign) return QGMM_ERR_WORKSPACE_TOO_SMALL;
    DeviceInfo *dev = nullptr;
    if ((s = device_info(&dev)) != QGMM_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    uint32_t *status = static_cast<uint32_t *>(workspace);
    const Plan pl = make_plan(p, dev->sms, EPI_RAW_ACC);
    CUtensorMap ma, mb, mb_tail;
    if ((s = make_maps(p, x1, x2, pl.tile_rows, pl.pair ? 16 : 32, &ma, &mb)) != QGMM_OK) return s;
    mb_tail = mb;
    if (pl.pair && p->weight_type == QGMM_W_INT4_PACKED_INT32 &&
        (s = make_maps(p, x1, x2, pl.tile_rows, 32, &ma, &mb_tail)) != QGMM_OK)
        return s;
    clear_status_kernel<<<1, 1, 0, st>>>(status);
    if (cudaGetLastError() != cudaSuccess) return QGMM_ERR_CUDA;
    GemmArgs a = base_args(p, group_list, pl, status);
    a.acc_out = acc_out;
    return launch_gemm(EPI_RAW_ACC, dev, p, pl, ma, mb, mb_tail, a, st);
}

QGMM_API qgmm_status qgmm_debug_accum_mx(const qgmm_problem *p, const uint8_t *x1, const uint8_t *sfa,
                                         const void *x2, const uint8_t *sfb, const int64_t *group_list,
                                         float *acc_out, void *workspace, size_t ws_bytes, void *cuda_stream)
{
    qgmm_status s = check_problem(p);
    if (s != QGMM_OK) return s;
    if (p->weight_type != QGMM_W_MXFP4) return QGMM_ERR_DTYPE;
    if (!x1 || !sfa || !x2 || !sfb || !group_list || !acc_out || !workspace) return QGMM_ERR_NULL_PTR;
    if (!aligned16(x1) || !aligned32(x2) || !aligned16(acc_out) || !aligned16(sfa) || !aligned16(sfb) ||
        (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0)
        return QGMM_ERR_ALIGNMENT;
    if (ws_bytes < workspace_bytes(p)) return QGMM_ERR_WORKSPACE_TOO_SMALL;
    DeviceInfo *dev = nullptr;
    if ((s = device_info(&dev)) != QGMM_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    uint32_t *status = static_cast<uint32_t *>(workspace);
    const Plan pl = make_plan(p, dev->sms, EPI_RAW_ACC);
    CUtensorMap ma, mb;
    if ((s = make_maps(p, reinterpret_cast<const int8_t *>(x1), x2, pl.tile_rows, 32, &ma, &mb)) != QGMM_OK)
        return s;
    if ((s = mx_write_atoms(p, dev, sfa, sfb, group_list, static_cast<uint8_t *>(workspace), st)) != QGMM_OK) return s;
    clear_status_kernel<<<1, 1, 0, st>>>(status);
    if (cudaGetLastError() != cudaSuccess) return QGMM_ERR_CUDA;
    GemmArgs a = base_args(p, group_list, pl, status);
    a.acc_out = reinterpret_cast<int32_t *>(acc_out);
    const MxAtoms A = mx_atoms(p);
    a.sfa = static_cast<const uint8_t *>(workspace) + A.rows;
    a.sfb = static_cast<const uint8_t *>(workspace) + A.cols;
    return launch_gemm(EPI_RAW_ACC, dev, p, pl, ma, mb, mb, a, st);
}

QGMM_API qgmm_status qgmm_per_token_quant(const uint16_t *x_bf16, int64_t rows, int64_t k, int8_t *x1_out,
                                          float *scale_out, void *cuda_stream)
{
    if (!x_bf16 || !x1_out || !scale_out) return QGMM_ERR_NULL_PTR;
    if (rows < 1 || rows > (int64_t(1) << 31) - 1 || k < 8 || k > 65536 || k % 8) return QGMM_ERR_SHAPE;
    if (!aligned16(x_bf16) || !aligned16(x1_out)) return QGMM_ERR_ALIGNMENT;
    DeviceInfo *dev = nullptr;
    qgmm_status s = device_info(&dev);
    if (s != QGMM_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    per_token_quant_kernel<<<grid_for(rows, 8, dev->sms, 8), 256, 0, st>>>(x_bf16, rows, static_cast<int32_t>(k),
                                                                           x1_out, scale_out);
    return cudaGetLastError() == cudaSuccess ? QGMM_OK : QGMM_ERR_CUDA;
}

QGMM_API qgmm_status qgmm_per_token_quant_mxfp8(const uint16_t *x_bf16, int64_t rows, int64_t k, uint8_t *q_out,
                                                uint8_t *sf_out, void *cuda_stream)
{
    if (!x_bf16 || !q_out || !sf_out) return QGMM_ERR_NULL_PTR;
    if (rows < 1 || rows > (int64_t(1) << 31) - 1 || k < 32 || k > 65536 || k % 32) return QGMM_ERR_SHAPE;
    if (!aligned16(x_bf16) || (reinterpret_cast<uintptr_t>(q_out) & 7u)) return QGMM_ERR_ALIGNMENT;
    DeviceInfo *dev = nullptr;
    qgmm_status s = device_info(&dev);
    if (s != QGMM_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    const int64_t chunks = rows * ((k + 255) / 256);
    per_token_quant_mxfp8_kernel<<<grid_for(chunks, 8, dev->sms, 8), 256, 0, st>>>(
        x_bf16, rows, static_cast<int32_t>(k), q_out, sf_out);
    return cudaGetLastError() == cudaSuccess ? QGMM_OK : QGMM_ERR_CUDA;
}

QGMM_API qgmm_status qgmm_device_status(const void *workspace, uint32_t *flags, void *cuda_stream)
{
    if (!workspace || !flags) return QGMM_ERR_NULL_PTR;
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return QGMM_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpy(&v, workspace, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return QGMM_ERR_CUDA;
    *flags = v;
    return v ? QGMM_ERR_DEVICE_INPUT : QGMM_OK;
}

QGMM_API const char *qgmm_status_string(qgmm_status s)
{
    switch (s) {
    case QGMM_OK: return "ok";
    case QGMM_ERR_NULL_PTR: return "a required pointer is NULL";
    case QGMM_ERR_SHAPE: return "a size is out of range";
    case QGMM_ERR_DTYPE: return "unknown weight, row-index or group-list type";
    case QGMM_ERR_WORKSPACE_TOO_SMALL: return "workspace smaller than qgmm_finalize_workspace reports";
    case QGMM_ERR_UNSUPPORTED: return "device is not sm_100 (B200)";
    case QGMM_ERR_CUDA: return "a CUDA call failed";
    case QGMM_ERR_DEVICE_INPUT: return "the device found invalid group_list or row_index values";
    case QGMM_ERR_ALIGNMENT: return "a pointer is not suitably aligned";
    case QGMM_ERR_SCRATCH_LIMIT: return "the problem needs more scratch than the library's static array holds";
    }
    return "unknown status";
}

// ---------------------------------------------------------------------------
// qgmm_finalize for callers that cannot allocate device memory.  The
// workspace is this file-scope array instead of caller memory; every GPU that
// loads the library holds it until the process exits.
static __device__ __align__(256) unsigned char qgmm_static_scratch[QGMM_STATIC_SCRATCH_BYTES];

namespace qgmm {
namespace {
void *g_static_scratch_addr[kMaxDevices] = {};

// Device address of qgmm_static_scratch on the current device, looked up once
// per device.  In host code the array's name is only a host-side stand-in, so
// it is never handed to a kernel directly.
qgmm_status static_scratch_address(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QGMM_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_static_scratch_addr[dev]) {
        void *p = nullptr;
        const cudaError_t rc = cudaGetSymbolAddress(&p, qgmm_static_scratch);
        if (rc != cudaSuccess || !p) return QGMM_ERR_CUDA;
        g_static_scratch_addr[dev] = p;
    }
    *out = g_static_scratch_addr[dev];
    return QGMM_OK;
}
}  // namespace
}  // namespace qgmm

QGMM_API qgmm_status qgmm_finalize_static_scratch(const qgmm_problem *p, const int8_t *x1, const void *x2,
                                                  const void *scale, const float *pertoken_scale,
                                                  const int64_t *group_list, const float *logit,
                                                  const void *row_index, const float *bias,
                                                  const uint16_t *shared_input, float *out, void *cuda_stream)
{
    qgmm_status s = check_problem(p);
    if (s != QGMM_OK) return s;
    if (workspace_bytes(p) > QGMM_STATIC_SCRATCH_BYTES) return QGMM_ERR_SCRATCH_LIMIT;
    DeviceInfo *dev = nullptr;
    if ((s = device_info(&dev)) != QGMM_OK) return s;
    void *scratch = nullptr;
    if ((s = static_scratch_address(&scratch)) != QGMM_OK) return s;
    return finalize_impl(p, x1, x2, scale, pertoken_scale, group_list, logit, row_index, bias, shared_input, out,
                         scratch, QGMM_STATIC_SCRATCH_BYTES, cuda_stream, nullptr, nullptr);
}
