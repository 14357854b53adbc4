// kernels.cuh -- sm_100a kernels of the fused int8 GroupedMatmul +
// MoeFinalizeRouting op ("aclnnGroupedMatmulFinalizeRoutingWeightNzV2":
// grouped matmul whose output rows are combined into the output by index;
// dequant rule of "matmul支持pertoken量化模式", 计算示例).
//
//   K1 output_init_kernel       out = sharedInput rows at the offset, else 0
//   K2 grouped_gemm_kernel      persistent grouped GEMM, tcgen05 kind::i8 into
//                               TMEM, TMA-fed smem ring, epilogue fused in
//                               registers (atomic combine | f32 rows | raw int32)
//   K3 det_* kernels            destination-sorted segmented reduce (fixed order)
//   K0 per_token_quant_kernel   bf16 -> int8 + absmax/127 per row
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "ptx_sm100.cuh"
#include "../../include/qgmm.h"

namespace qgmm {

// ---------------------------------------------------------------- tiling
constexpr int BM = 128;          // MMA M: TMEM lanes per accumulator
constexpr int BN = 256;          // MMA N: TMEM columns per accumulator
constexpr int BK = 128;          // K bytes per pipeline stage (one 128-byte swizzle row)
constexpr int UMMA_K = 32;       // K of one tcgen05.mma kind::i8
constexpr int A_STAGE_BYTES = BM * BK;       // 16 KB (box height may be smaller)
constexpr int B_STAGE_BYTES = BK * BN;       // 32 KB: two 128-column MN-major atoms
constexpr int P_STAGE_BYTES = BK * BN / 2;   // 16 KB: packed int4 staging
constexpr int B_ATOM_BYTES = BK * 128;       // one 128-column atom (LBO)
constexpr int TMEM_COLS = 2 * BN;            // double-buffered accumulator
constexpr int MAX_E = 1024;
constexpr int EPI_LD = 36;                   // staging row stride in floats (conflict-free float4 access)

enum Epilogue : int { EPI_ATOMIC = 0, EPI_STORE_Y = 1, EPI_RAW_ACC = 2 };

// Row tiling of each expert's rows.  A group of r rows has h = ceil(r / 128)
// half tiles of 128 rows.
//   SCHED_TILES      ceil(r / tile_rows) tiles of tile_rows rows (single CTA)
//   SCHED_PAIRS      floor(h / 2) pair tiles of 256 rows (CTA pair); an odd
//                    last half tile is left to a SCHED_TAILS launch
//   SCHED_PAIRS_ALL  ceil(h / 2) pair tiles of 256 rows, tails included
//   SCHED_TAILS      h % 2 tiles: the group's last 128 rows when h is odd
//   SCHED_PAIRS_TAIL128  ceil(h / 2) pair tiles; when h is odd the last one is an
//                    M = 128 pair tile (64 rows per CTA) over the final <= 128 rows
enum Schedule : int { SCHED_TILES = 0, SCHED_PAIRS = 1, SCHED_PAIRS_ALL = 2, SCHED_TAILS = 3, SCHED_PAIRS_TAIL128 = 4 };

__device__ __forceinline__ int32_t tiles_of_group(int64_t rows, int sched, int tile_rows)
{
    const int64_t h = (rows + 127) / 128;
    switch (sched) {
    case SCHED_PAIRS: return static_cast<int32_t>(h / 2);
    case SCHED_PAIRS_ALL:
    case SCHED_PAIRS_TAIL128: return static_cast<int32_t>((h + 1) / 2);
    case SCHED_TAILS: return static_cast<int32_t>(h & 1);
    default: return static_cast<int32_t>((rows + tile_rows - 1) / tile_rows);
    }
}

template <bool W4>
struct GemmCfg {
    static constexpr int STAGES = W4 ? 3 : 4;
    // producer, MMA, then 8 epilogue warps (int8) or 4 epilogue + 8 unpack warps (int4:
    // two unpack warps per SM sub-partition, measured 12% faster than one)
    static constexpr int NUM_WARPS = W4 ? 14 : 10;
    static constexpr int EPI_WARPS = W4 ? 4 : 8;
    static constexpr int THREADS = NUM_WARPS * 32;
    static constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES + (W4 ? P_STAGE_BYTES : 0);
    static constexpr int NUM_BARS = 3 * STAGES + 2 + 2 + 1;
    static constexpr int CTRL_BYTES = (NUM_BARS * 8 + 16 + 15) / 16 * 16;
    static constexpr int TABLE_BYTES = (2 * (MAX_E + 1) * 4 + 15) / 16 * 16;
    static constexpr int EPI_STAGE_BYTES = 4 * 32 * EPI_LD * 4;   // per epilogue warp: 32 rows x 32 cols (+pad)
    static constexpr int ROWINFO_BYTES = 4 * 32 * 16;              // per row: pts, logit, destination
    static constexpr size_t OFF_CTRL = size_t(STAGES) * STAGE_BYTES;
    static constexpr size_t OFF_TABLE = OFF_CTRL + CTRL_BYTES;
    static constexpr size_t OFF_EPI = OFF_TABLE + TABLE_BYTES;
    static constexpr size_t OFF_ROWS = OFF_EPI + EPI_STAGE_BYTES;
    static constexpr size_t SMEM_BYTES = 1024 + OFF_ROWS + ROWINFO_BYTES;
    static_assert(SMEM_BYTES <= 232448, "shared memory above the sm_100 per-block limit");
};

struct GemmArgs {
    const int64_t *group_list;
    int64_t m;
    int32_t e, group_list_type;
    int32_t k, n;
    int32_t tile_rows;     // rows per m-tile = TMA box height of x1 (16, 32, 64 or 128)
    int32_t sched;         // which m-tiles this launch covers (SCHED_*)
    int32_t stall_producer;  // test hook: the producer issues no copy, so the MMA wait must run out
    int32_t slab_ntiles;   // n-tiles per slab; divides n / BN
    int32_t b_kmajor;      // int8 x2 stored (e, n, k): K-major B tiles, the x1 tile's layout
    const void *scale;     // f32 [e, ld_sb], or bf16 bits when scale_bf16
    int32_t scale_bf16;
    int64_t ld_sb;         // row stride of scale and bias (elements)
    const float *pts, *logit, *bias;
    const void *row_index;
    int32_t row_index_type;
    int64_t output_bs;
    float *out;            // EPI_ATOMIC: out [output_bs, ldd]; EPI_STORE_Y: y [store_rows, ldd]
    int64_t store_rows;    // EPI_STORE_Y: rows of its destination (m for y; output_bs when it is out)
    int32_t *acc_out;      // EPI_RAW_ACC: [m, ldd]
    int64_t ldd;           // row stride of the destination (out, y or acc_out)
    const uint8_t *sfa;    // MX kernel: E8M0 scales of x1 [m, k/32]
    const uint8_t *sfb;    // MX kernel: E8M0 scales of the weights [e, ld_sb, k/32]
    uint32_t *status;
};

// ---------------------------------------------------------------- groups
// Warp-cooperative decode of groupList (page 1, parameter constraints):
// off[g+1] = end row of group g, cum[g+1] = m-tiles of groups 0..g.
// Invalid lists are sanitised so every offset stays in [0, m] and monotone
// (type 0: running max of clamp(end, 0, m); type 1: clamp of the running sum
// of max(count, 0)); the returned QGMM_DEV_* bits say what was wrong.
__device__ __forceinline__ uint32_t decode_groups_warp(const int64_t *gl, int e, int type, int64_t m,
                                                       int tile_rows, int sched, int32_t *off, int32_t *cum)
{
    const int lane = threadIdx.x & 31;
    uint32_t flags = 0;
    int64_t carry_end = 0;     // end of the previous chunk's last group
    int64_t carry_sum = 0;     // type 1: unclamped running sum
    int32_t carry_cum = 0;
    if (lane == 0) {
        off[0] = 0;
        cum[0] = 0;
    }
    for (int base = 0; base < e; base += 32) {
        const int g = base + lane;
        const bool in = g < e;
        const int64_t v = in ? gl[g] : 0;
        if (in && v < 0) flags |= QGMM_DEV_GROUP_NEGATIVE;
        int64_t end;
        if (type == 0) {
            if (in && g > 0 && v < gl[g - 1]) flags |= QGMM_DEV_GROUP_NOT_MONOTONE;
            if (in && v > m) flags |= QGMM_DEV_GROUP_TOTAL_GT_M;
            int64_t s = v < 0 ? 0 : (v > m ? m : v);
            if (!in) s = 0;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int64_t o = __shfl_up_sync(0xffffffffu, s, d);
                if (lane >= d && o > s) s = o;
            }
            end = s > carry_end ? s : carry_end;
        } else {
            int64_t s = (in && v > 0) ? v : 0;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int64_t o = __shfl_up_sync(0xffffffffu, s, d);
                if (lane >= d) s += o;
            }
            s += carry_sum;
            carry_sum = __shfl_sync(0xffffffffu, s, 31);
            if (in && s > m) flags |= QGMM_DEV_GROUP_TOTAL_GT_M;
            end = s > m ? m : s;
        }
        int64_t start = __shfl_up_sync(0xffffffffu, end, 1);
        if (lane == 0) start = carry_end;
        const int64_t rows = end - start;
        int32_t mt = in ? tiles_of_group(rows, sched, tile_rows) : 0;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int32_t o = __shfl_up_sync(0xffffffffu, mt, d);
            if (lane >= d) mt += o;
        }
        mt += carry_cum;
        if (in) {
            off[g + 1] = static_cast<int32_t>(end);
            cum[g + 1] = mt;
        }
        carry_end = __shfl_sync(0xffffffffu, end, 31);
        carry_cum = __shfl_sync(0xffffffffu, mt, 31);
    }
    // OR-reduce the flags across the warp
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) flags |= __shfl_xor_sync(0xffffffffu, flags, d);
    __syncwarp();
    return flags;
}

struct TileCoord {
    int g, row0, row_end, nt;
    int mt;      // m-tile index in the walk (the expert-major order of the groups' tiles)
    bool tail;   // SCHED_PAIRS_TAIL128: an M = 128 pair tile
};

// Tile t of the persistent walk.  Order: slab of slab_ntiles n-tiles, then
// expert, then m-tile, then the n-tiles of the slab -- so consecutive tiles
// (taken by neighbouring CTAs at the same time) share one x1 row tile and one
// expert's weight columns, and one slab of the output stays hot in L2.
__device__ __forceinline__ TileCoord tile_coord(int t, int MT, int SW, const int32_t *off, const int32_t *cum,
                                                int e, int tile_rows, int sched)
{
    const int per_slab = MT * SW;
    const int s = t / per_slab;
    const int r = t - s * per_slab;
    const int mt = r / SW;
    TileCoord c;
    c.mt = mt;
    c.nt = s * SW + (r - mt * SW);
    int lo = 0, hi = e;  // cum[lo] <= mt < cum[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (cum[mid] <= mt) lo = mid;
        else hi = mid;
    }
    c.g = lo;
    c.row_end = off[lo + 1];
    c.tail = false;
    if (sched == SCHED_PAIRS_TAIL128) {
        const int h = (off[lo + 1] - off[lo] + 127) / 128;
        const int j = mt - cum[lo];
        c.row0 = off[lo] + j * 256;
        c.tail = (h & 1) && j == h / 2;
    } else if (sched == SCHED_TAILS)
        c.row0 = off[lo] + 128 * ((off[lo + 1] - off[lo] + 127) / 128 - 1);
    else if (sched == SCHED_PAIRS || sched == SCHED_PAIRS_ALL)
        c.row0 = off[lo] + (mt - cum[lo]) * 256;
    else
        c.row0 = off[lo] + (mt - cum[lo]) * tile_rows;
    return c;
}

__device__ __forceinline__ int64_t load_row_index(const void *ri, int type, int64_t i)
{
    if (ri == nullptr) return i;
    if (type == QGMM_IDX_INT64) return __ldg(static_cast<const long long *>(ri) + i);
    return static_cast<int64_t>(__ldg(static_cast<const int *>(ri) + i));
}

// int4 (two's complement, lowest nibble = lowest column) -> int8 holding 16 times
// the value, 8 values per word.  Each nibble moves to the high half of its byte,
// and that byte read as int8 is the nibble's two's-complement value times 16, with
// no sign fill.  The MMA then accumulates 16 * acc; the epilogue shifts it back
// (W4_ACC_SHIFT), exactly, since |16 * acc| <= 16 * 65536 * 128 * 8 = 2^30 for k <= 65536.
constexpr int W4_ACC_SHIFT = 4;
__device__ __forceinline__ void unpack_int4x8(uint32_t w, uint32_t &lo_out, uint32_t &hi_out)
{
    const uint32_t ev = (w << 4) & 0xF0F0F0F0u;   // nibbles 0, 2, 4, 6
    const uint32_t od = w & 0xF0F0F0F0u;          // nibbles 1, 3, 5, 7
    lo_out = __byte_perm(ev, od, 0x5140);         // columns 0..3
    hi_out = __byte_perm(ev, od, 0x7362);         // columns 4..7
}

// ---------------------------------------------------------------- K2 epilogue helpers
// scale[idx .. idx+3] (idx % 4 == 0) or [idx, idx+1] (idx even) as f32.  A bf16
// scale is widened exactly: its 16 bits are the upper half of the f32.
__device__ __forceinline__ float4 load_scale4(const GemmArgs &a, int64_t idx)
{
    if (a.scale_bf16) {
        const uint2 v = __ldg(reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(a.scale) + idx));
        return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u), __uint_as_float(v.y << 16),
                           __uint_as_float(v.y & 0xFFFF0000u));
    }
    return __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(a.scale) + idx));
}

__device__ __forceinline__ float2 load_scale2(const GemmArgs &a, int64_t idx)
{
    if (a.scale_bf16) {
        const uint32_t v = __ldg(reinterpret_cast<const unsigned int *>(static_cast<const uint16_t *>(a.scale) + idx));
        return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
    }
    return __ldg(reinterpret_cast<const float2 *>(static_cast<const float *>(a.scale) + idx));
}

constexpr int NCHUNK = BN / 32;   // 32-column chunks per accumulator

// Thread = accumulator row: write its 32 values of one chunk into the warp's
// staging rows (f32 of the int32 value, or its raw bits for the debug output).
// SHIFT undoes the int4 path's x16 operand scale (arithmetic shift, exact).
// FACC: the accumulator already is f32 (E4M3 operands); its bits pass through.
template <int EPI, int SHIFT, bool FACC = false>
__device__ __forceinline__ void epi_stage_chunk(float *stage, int lane, const uint32_t (&r)[32])
{
    float *srow = stage + lane * EPI_LD;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
        int a[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) a[u] = static_cast<int>(r[4 * v + u]) >> SHIFT;
        float4 f;
        if constexpr (EPI == EPI_RAW_ACC || FACC) {
            f = make_float4(__int_as_float(a[0]), __int_as_float(a[1]), __int_as_float(a[2]), __int_as_float(a[3]));
        } else {
            f = make_float4(__int2float_rn(a[0]), __int2float_rn(a[1]), __int2float_rn(a[2]), __int2float_rn(a[3]));
        }
        *reinterpret_cast<float4 *>(srow + 4 * v) = f;
    }
}

// Transposed read of a staged chunk: lane (sub, col4) takes 4 columns of rows
// sub, sub+4, ..., so each warp instruction covers 4 rows x 128 contiguous bytes.
// The dequant runs here in the op's order: ((f32(acc) * scale) * pts + bias) * logit.
template <int EPI>
__device__ __forceinline__ void epi_write_chunk(const GemmArgs &args, const float *stage, const float *rp,
                                                const float *rl, const long long *rd, int sub, int col4, int64_t ldd,
                                                int64_t chunk_col0, float4 s4, float4 b4)
{
    const int64_t col = chunk_col0 + col4;
#pragma unroll
    for (int it = 0; it < 8; ++it) {
        const int row = sub + 4 * it;
        const long long d = rd[row];
        const float4 v = *reinterpret_cast<const float4 *>(stage + row * EPI_LD + col4);
        if (d >= 0) {
            if constexpr (EPI == EPI_RAW_ACC) {
                *reinterpret_cast<int4 *>(args.acc_out + d * ldd + col) =
                    make_int4(__float_as_int(v.x), __float_as_int(v.y), __float_as_int(v.z), __float_as_int(v.w));
            } else {
                const float p = rp[row], l = rl[row];
                const float y0 = __fmul_rn(__fadd_rn(__fmul_rn(__fmul_rn(v.x, s4.x), p), b4.x), l);
                const float y1 = __fmul_rn(__fadd_rn(__fmul_rn(__fmul_rn(v.y, s4.y), p), b4.y), l);
                const float y2 = __fmul_rn(__fadd_rn(__fmul_rn(__fmul_rn(v.z, s4.z), p), b4.z), l);
                const float y3 = __fmul_rn(__fadd_rn(__fmul_rn(__fmul_rn(v.w, s4.w), p), b4.w), l);
                if constexpr (EPI == EPI_ATOMIC) {
                    ptx::red_add_v4(args.out + d * ldd + col, y0, y1, y2, y3);
                } else {   // stored as 0 + y, the value a sum starting from zero gives (-0 becomes +0)
                    *reinterpret_cast<float4 *>(args.out + d * ldd + col) = make_float4(
                        __fadd_rn(y0, 0.f), __fadd_rn(y1, 0.f), __fadd_rn(y2, 0.f), __fadd_rn(y3, 0.f));
                }
            }
        }
    }
}

// Shared-memory scratch of one epilogue warp.
struct EpiSmem {
    float *stage;      // 32 rows x EPI_LD floats
    float *rp, *rl;    // per-row pertoken scale and logit
    long long *rd;     // per-row output row (-1: skip)
};

__device__ __forceinline__ EpiSmem epi_smem(float *epi_stage, float *row_pts, float *row_lg, long long *row_dst, int slot)
{
    EpiSmem sm;
    sm.stage = epi_stage + slot * (32 * EPI_LD);
    sm.rp = row_pts + slot * 32;
    sm.rl = row_lg + slot * 32;
    sm.rd = row_dst + slot * 32;
    return sm;
}

// Epilogue of one accumulator tile for one warp, which owns TMEM lane quarter
// q (accumulator rows 32q .. 32q+31 of this CTA).  Accumulator row r is source
// row row_base + r; it is valid when r < rows_here and the source row lies
// below the group's end.  A 32x32 chunk is read with tcgen05.ld (thread = row),
// converted to f32 and staged in shared memory, then read back transposed so
// that 8 lanes cover one row's 32 columns (128 contiguous bytes) and one warp
// instruction writes 4 row segments.  The dequant runs in the transposed phase,
// in the op's order ((f32(acc) * scale) * pts + bias) * logit.  Per-row data
// and this lane's scale/bias columns are fetched before waiting for the
// accumulator, and TMEM chunk k+1 is loaded while chunk k is written out.
// SHIFT: W4_ACC_SHIFT for int4 weights, else 0.  Returns false if the wait for
// the accumulator ran out.
template <int EPI, int NCH, int SHIFT, bool FACC = false>
__device__ __forceinline__ bool epilogue_tile(const GemmArgs &args, const TileCoord &c, int64_t row_base,
                                              int rows_here, int row_off, uint32_t tmem_acc, int q, int tmem_col,
                                              int glob_col, int lane, uint64_t *tfull_bar, uint32_t use,
                                              volatile int *abort_flag, const EpiSmem &sm, int tile_n = BN)
{
    const int64_t ldd = args.ldd;
    const int col_begin = glob_col;       // tile column of this warp's first TMEM column
    const int sub = lane >> 3;            // row (mod 4) handled in the transposed phase
    const int col4 = (lane & 7) * 4;      // first of the 4 columns handled in the transposed phase
    const int r_in = row_off + lane;
    const int64_t i = row_base + r_in;
    float pts = 1.0f, lg = 1.0f;
    long long dst = -1;
    if (r_in < rows_here && i < c.row_end) {
        if (args.pts) pts = __ldg(args.pts + i);
        if (args.logit) lg = __ldg(args.logit + i);
        if (EPI == EPI_ATOMIC) {
            const int64_t d = load_row_index(args.row_index, args.row_index_type, i);
            if (d < 0 || d >= args.output_bs) atomicOr(args.status, QGMM_DEV_ROW_INDEX_RANGE);
            else dst = d;
        } else if (EPI == EPI_STORE_Y && i >= args.store_rows) {
            atomicOr(args.status, QGMM_DEV_ROW_INDEX_RANGE);   // identity routing past output_bs
        } else {
            dst = i;
        }
    }
    sm.rp[lane] = pts;
    sm.rl[lane] = lg;
    sm.rd[lane] = dst;
    const bool any = __any_sync(0xffffffffu, dst >= 0);
    float4 sc[NCH], bs[NCH];
#pragma unroll
    for (int k = 0; k < NCH; ++k) {
        sc[k] = make_float4(1.f, 1.f, 1.f, 1.f);
        bs[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (EPI != EPI_RAW_ACC && any) {
        const int64_t base = static_cast<int64_t>(c.g) * args.ld_sb + static_cast<int64_t>(c.nt) * tile_n + col_begin + col4;
        if (args.scale) {
#pragma unroll
            for (int k = 0; k < NCH; ++k) sc[k] = load_scale4(args, base + k * 32);
        }
        if (args.bias) {
#pragma unroll
            for (int k = 0; k < NCH; ++k) bs[k] = __ldg(reinterpret_cast<const float4 *>(args.bias + base + k * 32));
        }
    }
    __syncwarp();
    if (!ptx::mbar_wait(tfull_bar, use, abort_flag)) return false;
    ptx::tc_fence_after();
    if (any) {
        const int64_t n0 = static_cast<int64_t>(c.nt) * tile_n + col_begin;
        const uint32_t tbase = tmem_acc + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(tmem_col);
        uint32_t ra[32], rb[32];
        ptx::tmem_ld_32x32b_x32(tbase, ra);
#pragma unroll
        for (int pc = 0; pc < NCH; pc += 2) {
            ptx::tmem_ld_wait(ra);
            epi_stage_chunk<EPI, SHIFT, FACC>(sm.stage, lane, ra);
            ptx::tmem_ld_32x32b_x32(tbase + static_cast<uint32_t>((pc + 1) * 32), rb);
            __syncwarp();
            epi_write_chunk<EPI>(args, sm.stage, sm.rp, sm.rl, sm.rd, sub, col4, ldd, n0 + pc * 32, sc[pc], bs[pc]);
            __syncwarp();
            ptx::tmem_ld_wait(rb);
            epi_stage_chunk<EPI, SHIFT, FACC>(sm.stage, lane, rb);
            if (pc + 2 < NCH) ptx::tmem_ld_32x32b_x32(tbase + static_cast<uint32_t>((pc + 2) * 32), ra);
            __syncwarp();
            epi_write_chunk<EPI>(args, sm.stage, sm.rp, sm.rl, sm.rd, sub, col4, ldd, n0 + (pc + 1) * 32, sc[pc + 1],
                                 bs[pc + 1]);
            __syncwarp();
        }
    }
    ptx::tc_fence_before();
    __syncwarp();
    return true;
}

// Direct epilogue (int8 kernels): one warp owns TMEM lane quarter q and the
// EPI_COLS columns [col_begin, col_begin + EPI_COLS) of the tile.  tcgen05.ld
// .16x256b gives thread t the rows t/4 and t/4 + 8 of a 16-lane half and two
// adjacent columns of every 8-column block, so 4 threads cover 32 contiguous
// bytes of a row and each warp instruction reduces 8 rows x 32 bytes (whole
// sectors) straight from registers; no shared-memory round trip.  Per-row
// data of the thread's 4 rows and its scale/bias columns are loaded before the
// wait for the accumulator.  The dequant runs in the op's order
// ((f32(acc) * scale) * pts + bias) * logit.  Returns false if the wait ran out.
constexpr int EPI_COLS = 128;
constexpr int EPI_CHUNKS = EPI_COLS / 64;

template <int EPI, bool FACC>
__device__ __forceinline__ void epi_direct_rows(const GemmArgs &args, const uint32_t (&v)[32], long long dA,
                                                long long dB, float pA, float pB, float lA, float lB,
                                                const float2 (&sc)[8], const float2 (&bs)[8], int64_t ldd, int64_t col0)
{
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int64_t col = col0 + 8 * j;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const long long d = h ? dB : dA;
            if (d < 0) continue;
            const uint32_t u0 = v[4 * j + 2 * h], u1 = v[4 * j + 2 * h + 1];
            if constexpr (EPI == EPI_RAW_ACC) {
                *reinterpret_cast<int2 *>(args.acc_out + d * ldd + col) =
                    make_int2(static_cast<int>(u0), static_cast<int>(u1));
            } else {
                const float p = h ? pB : pA, l = h ? lB : lA;
                const float a0 = FACC ? __uint_as_float(u0) : __int2float_rn(static_cast<int>(u0));
                const float a1 = FACC ? __uint_as_float(u1) : __int2float_rn(static_cast<int>(u1));
                const float y0 = __fmul_rn(__fadd_rn(__fmul_rn(__fmul_rn(a0, sc[j].x), p), bs[j].x), l);
                const float y1 = __fmul_rn(__fadd_rn(__fmul_rn(__fmul_rn(a1, sc[j].y), p), bs[j].y), l);
                if constexpr (EPI == EPI_ATOMIC) {
                    ptx::red_add_v2(args.out + d * ldd + col, y0, y1);
                } else {   // stored as 0 + y, as in the staged epilogue
                    *reinterpret_cast<float2 *>(args.out + d * ldd + col) =
                        make_float2(__fadd_rn(y0, 0.f), __fadd_rn(y1, 0.f));
                }
            }
        }
    }
}

template <int EPI, bool FACC>
__device__ __forceinline__ bool epilogue_tile_direct(const GemmArgs &args, const TileCoord &c, int64_t row_base,
                                                     int rows_here, uint32_t tmem_acc, int q, int col_begin, int lane,
                                                     uint64_t *tfull_bar, uint32_t use, volatile int *abort_flag)
{
    const int64_t ldd = args.ldd;
    const int t0 = lane & 3, t1 = lane >> 2;
    float pts[4], lg[4];
    long long dst[4];
    bool mine = false;
#pragma unroll
    for (int k = 0; k < 4; ++k) {   // k: (16-lane half) * 2 + (upper 8 rows of the half)
        const int r_in = q * 32 + (k >> 1) * 16 + (k & 1) * 8 + t1;
        const int64_t i = row_base + r_in;
        pts[k] = 1.0f;
        lg[k] = 1.0f;
        dst[k] = -1;
        if (r_in < rows_here && i < c.row_end) {
            if (args.pts) pts[k] = __ldg(args.pts + i);
            if (args.logit) lg[k] = __ldg(args.logit + i);
            if (EPI == EPI_ATOMIC) {
                const int64_t d = load_row_index(args.row_index, args.row_index_type, i);
                if (d < 0 || d >= args.output_bs) atomicOr(args.status, QGMM_DEV_ROW_INDEX_RANGE);
                else dst[k] = d;
            } else if (EPI == EPI_STORE_Y && i >= args.store_rows) {
                atomicOr(args.status, QGMM_DEV_ROW_INDEX_RANGE);   // identity routing past output_bs
            } else {
                dst[k] = i;
            }
        }
        mine |= dst[k] >= 0;
    }
    const bool any = __any_sync(0xffffffffu, mine);
    const int64_t n0 = static_cast<int64_t>(c.nt) * BN + col_begin + 2 * t0;
    float2 sc[EPI_CHUNKS][8], bs[EPI_CHUNKS][8];
#pragma unroll
    for (int ch = 0; ch < EPI_CHUNKS; ++ch)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            sc[ch][j] = make_float2(1.f, 1.f);
            bs[ch][j] = make_float2(0.f, 0.f);
        }
    if (EPI != EPI_RAW_ACC && any) {
        const int64_t base = static_cast<int64_t>(c.g) * args.ld_sb + n0;
        if (args.scale) {
#pragma unroll
            for (int ch = 0; ch < EPI_CHUNKS; ++ch)
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    sc[ch][j] = load_scale2(args, base + 64 * ch + 8 * j);
        }
        if (args.bias) {
#pragma unroll
            for (int ch = 0; ch < EPI_CHUNKS; ++ch)
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    bs[ch][j] = __ldg(reinterpret_cast<const float2 *>(args.bias + base + 64 * ch + 8 * j));
        }
    }
    __syncwarp();
    if (!ptx::mbar_wait(tfull_bar, use, abort_flag)) return false;
    ptx::tc_fence_after();
    if (any) {
#pragma unroll
        for (int ch = 0; ch < EPI_CHUNKS; ++ch) {
            uint32_t va[32], vb[32];
            const uint32_t col = tmem_acc + static_cast<uint32_t>(col_begin + 64 * ch);
            ptx::tmem_ld_16x256b_x8(col + (static_cast<uint32_t>(q * 32) << 16), va);
            ptx::tmem_ld_16x256b_x8(col + (static_cast<uint32_t>(q * 32 + 16) << 16), vb);
            ptx::tmem_ld_wait2(va, vb);
            epi_direct_rows<EPI, FACC>(args, va, dst[0], dst[1], pts[0], pts[1], lg[0], lg[1], sc[ch], bs[ch], ldd,
                                 n0 + 64 * ch);
            epi_direct_rows<EPI, FACC>(args, vb, dst[2], dst[3], pts[2], pts[3], lg[2], lg[3], sc[ch], bs[ch], ldd,
                                 n0 + 64 * ch);
        }
    }
    ptx::tc_fence_before();
    __syncwarp();
    return true;
}

// ---------------------------------------------------------------- K2
// F8: E4M3 operands (tcgen05.mma kind::f8f6f4, f32 accumulators); same tiles and
// shared-memory layout as int8, one byte per element and K = 32 per instruction.
template <int EPI, bool W4, bool F8 = false>
__global__ void __launch_bounds__(GemmCfg<W4>::THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                        const GemmArgs args)
{
    using Cfg = GemmCfg<W4>;
    constexpr int S = Cfg::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *smem_a = smem;
    uint8_t *smem_b = smem_a + S * A_STAGE_BYTES;
    uint8_t *smem_p = smem_b + S * B_STAGE_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_CTRL);
    uint64_t *full = bars;            // operands ready for the MMA
    uint64_t *empty = bars + S;       // MMA finished reading the stage
    uint64_t *pfull = bars + 2 * S;   // W4: packed tile + x1 tile landed
    uint64_t *tfull = bars + 3 * S;   // accumulator buffer ready for the epilogue
    uint64_t *tempty = tfull + 2;     // epilogue drained the accumulator buffer
    uint64_t *drain = tempty + 2;     // all issued MMAs completed
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + Cfg::NUM_BARS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    int32_t *off = reinterpret_cast<int32_t *>(smem + Cfg::OFF_TABLE);
    int32_t *cum = off + (MAX_E + 1);
    float *epi_stage = reinterpret_cast<float *>(smem + Cfg::OFF_EPI);
    float *row_pts = reinterpret_cast<float *>(smem + Cfg::OFF_ROWS);
    float *row_lg = row_pts + 4 * 32;
    long long *row_dst = reinterpret_cast<long long *>(row_lg + 4 * 32);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(&full[s], W4 ? 8 : 1);   // W4: the 8 unpack warps
            ptx::mbar_init(&empty[s], 1);
            ptx::mbar_init(&pfull[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&tfull[b], 1);
            ptx::mbar_init(&tempty[b], Cfg::EPI_WARPS);
        }
        ptx::mbar_init(drain, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    volatile uint32_t *group_flags = reinterpret_cast<volatile uint32_t *>(tmem_holder + 2);
    if (warp == 0) {
        const uint32_t flags = decode_groups_warp(args.group_list, args.e, args.group_list_type, args.m,
                                                  args.tile_rows, args.sched, off, cum);
        if (lane == 0) {
            *group_flags = flags;
            ptx::prefetch_tmap(&map_a);
            ptx::prefetch_tmap(&map_b);
        }
    } else if (warp == 1) {
        ptx::tmem_alloc(tmem_holder, TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    const int e = args.e;
    const int MT = cum[e];
    const int NT = args.n / BN;
    const int SW = args.slab_ntiles;
    const int T = MT * NT;
    const int KB = args.k / BK;
    const int tile_rows = args.tile_rows;

    // The status word is cleared by the kernel this one may overlap under programmatic
    // dependent launch: wait for that kernel before setting a bit in it.
    auto fail = [&]() {
        ptx::pdl_wait_primary();
        atomicOr(args.status, QGMM_DEV_TIMEOUT);
        *abort_flag = 1;
    };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint32_t a_bytes = static_cast<uint32_t>(tile_rows) * BK;
            uint32_t issued[S];
#pragma unroll
            for (int s = 0; s < S; ++s) issued[s] = 0;
            int stage = 0;
            uint32_t phase = 0;
            bool ok = args.stall_producer == 0;
            for (int t = blockIdx.x; t < T && ok; t += gridDim.x) {
                const TileCoord c = tile_coord(t, MT, SW, off, cum, e, tile_rows, args.sched);
                const int n0 = c.nt * BN;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!ptx::mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
                        fail();
                        ok = false;
                        break;
                    }
                    if constexpr (W4) {
                        ptx::mbar_arrive_expect_tx(&pfull[stage], a_bytes + P_STAGE_BYTES);
                        ptx::tma_load_2d(smem_a + stage * A_STAGE_BYTES, &map_a, &pfull[stage], kb * BK, c.row0);
                        ptx::tma_load_3d(smem_p + stage * P_STAGE_BYTES, &map_b, &pfull[stage], n0 / 8, kb * BK,
                                         c.g);
                    } else {
                        ptx::mbar_arrive_expect_tx(&full[stage], a_bytes + B_STAGE_BYTES);
                        ptx::tma_load_2d(smem_a + stage * A_STAGE_BYTES, &map_a, &full[stage], kb * BK, c.row0);
                        uint8_t *b = smem_b + stage * B_STAGE_BYTES;
                        if (args.b_kmajor) {   // 128 n-rows of 128 K bytes per box
                            ptx::tma_load_3d(b, &map_b, &full[stage], kb * BK, n0, c.g);
                            ptx::tma_load_3d(b + B_ATOM_BYTES, &map_b, &full[stage], kb * BK, n0 + 128, c.g);
                        } else {               // 128 n-columns of BK k-rows per box
                            ptx::tma_load_3d(b, &map_b, &full[stage], n0, kb * BK, c.g);
                            ptx::tma_load_3d(b + B_ATOM_BYTES, &map_b, &full[stage], n0 + 128, kb * BK, c.g);
                        }
                    }
                    ++issued[stage];
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // let the copies already in flight land before the CTA leaves
                for (int s = 0; s < S; ++s) {
                    if (issued[s] == 0) continue;
                    uint64_t *bar = W4 ? &pfull[s] : &full[s];
                    const uint32_t par = (issued[s] - 1u) & 1u;
                    volatile int never = 0;
                    ptx::mbar_wait(bar, par, &never);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            // int4 tiles are always unpacked MN-major; int8 (e, n, k) weights land K-major
            const bool bk = !W4 && args.b_kmajor != 0;
            const uint32_t idesc = F8 ? ptx::idesc_e4m3(BM, BN, !bk) : ptx::idesc_i8(BM, BN, !bk);
            const uint32_t b_kstep = bk ? UMMA_K : UMMA_K * 128, b_lbo = bk ? 16 : B_ATOM_BYTES;
            int stage = 0;
            uint32_t phase = 0;
            int lt = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < T && ok; t += gridDim.x, ++lt) {
                const int buf = lt & 1;
                const uint32_t use = static_cast<uint32_t>(lt >> 1) & 1u;
                if (!ptx::mbar_wait(&tempty[buf], use ^ 1u, abort_flag)) {
                    fail();
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!ptx::mbar_wait(&full[stage], phase, abort_flag)) {
                        fail();
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t a0 = ptx::smem_addr(smem_a + stage * A_STAGE_BYTES);
                    const uint32_t b0 = ptx::smem_addr(smem_b + stage * B_STAGE_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / UMMA_K; ++kk) {
                        // A: K-major, 128-byte rows, 8-row groups 1024 B apart; step K by 32 bytes
                        const uint64_t adesc = ptx::smem_desc_sw128(a0 + kk * UMMA_K, 16, 1024);
                        // B: MN-major, 128-column atoms B_ATOM_BYTES apart, 8-row K groups 1024 B
                        // apart; or K-major like A, 8-row n groups 1024 B apart
                        const uint64_t bdesc = ptx::smem_desc_sw128(b0 + kk * b_kstep, b_lbo, 1024);
                        if constexpr (F8)
                            ptx::mma_e4m3(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                        else
                            ptx::mma_i8(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    ptx::mma_commit(&empty[stage]);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) ptx::mma_commit(&tfull[buf]);
            }
            ptx::mma_commit(drain);
            volatile int never = 0;
            ptx::mbar_wait(drain, 0, &never);
        }
        __syncwarp();
    } else if (!W4) {
        // ------------------------------------------------ epilogue, int8: 8 warps, direct from TMEM
        ptx::pdl_wait_primary();   // the output (and status word) are initialised by the previous kernel
        if (warp == 2 && lane == 0 && blockIdx.x == 0 && *group_flags) atomicOr(args.status, *group_flags);
        const int q = warp & 3;
        const int col_begin = ((warp - 2) >> 2) * EPI_COLS;
        int lt = 0;
        for (int t = blockIdx.x; t < T; t += gridDim.x, ++lt) {
            const TileCoord c = tile_coord(t, MT, SW, off, cum, e, tile_rows, args.sched);
            const int buf = lt & 1;
            const uint32_t use = static_cast<uint32_t>(lt >> 1) & 1u;
            if (!epilogue_tile_direct<EPI, F8>(args, c, c.row0, tile_rows, tmem_base + static_cast<uint32_t>(buf * BN), q,
                                           col_begin, lane, &tfull[buf], use, abort_flag)) {
                fail();
                break;
            }
            if (lane == 0) ptx::mbar_arrive(&tempty[buf]);
        }
    } else if (warp < 6) {
        // ------------------------------------------------ epilogue, W4: 4 warps, staged through smem
        ptx::pdl_wait_primary();
        if (warp == 2 && lane == 0 && blockIdx.x == 0 && *group_flags) atomicOr(args.status, *group_flags);
        const int q = warp & 3;
        const EpiSmem sm = epi_smem(epi_stage, row_pts, row_lg, row_dst, q);
        int lt = 0;
        for (int t = blockIdx.x; t < T; t += gridDim.x, ++lt) {
            const TileCoord c = tile_coord(t, MT, SW, off, cum, e, tile_rows, args.sched);
            const int buf = lt & 1;
            const uint32_t use = static_cast<uint32_t>(lt >> 1) & 1u;
            if (!epilogue_tile<EPI, NCHUNK, W4 ? W4_ACC_SHIFT : 0>(args, c, c.row0, tile_rows, q * 32,
                                            tmem_base + static_cast<uint32_t>(buf * BN), q, 0, 0, lane, &tfull[buf],
                                            use, abort_flag, sm)) {
                fail();
                break;
            }
            if (lane == 0) ptx::mbar_arrive(&tempty[buf]);
        }
    } else if constexpr (W4) {
        // ------------------------------------------------ int4 -> int8 unpack into the MN-major B tile
        // Each warp covers 4 k rows x 8 packed 16-byte chunks (qc: columns 32qc ..
        // 32qc+31).  In every group of 8 lanes, lanes 0-3 take chunks 0-3 (atom 0) of
        // one row and lanes 4-7 chunks 4-7 (atom 1) of the neighbouring row, so the 8
        // swizzled int8 stores hit 8 different 16-byte bank groups (the two rows'
        // chunk parities differ) and the 8 packed loads do too.
        const int ut = threadIdx.x - 6 * 32;    // 0..255
        const int l = ut & 31;
        const int qc = l & 7;
        const int r0 = 4 * (ut >> 5) + ((((l >> 2) ^ (l >> 3)) & 1) | ((l >> 3) & 2));   // row offset 0..3 in the warp
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < T && ok; t += gridDim.x) {
            for (int kb = 0; kb < KB; ++kb) {
                if (!ptx::mbar_wait(&pfull[stage], phase, abort_flag)) {
                    fail();
                    ok = false;
                    break;
                }
                const uint8_t *p = smem_p + stage * P_STAGE_BYTES;
                uint8_t *b = smem_b + stage * B_STAGE_BYTES;
#pragma unroll
                for (int it = 0; it < 4; ++it) {
                    const int kr = r0 + 32 * it;          // k row within the stage
                    const uint4 w = *reinterpret_cast<const uint4 *>(p + kr * 128 + qc * 16);
                    uint4 o0, o1;
                    unpack_int4x8(w.x, o0.x, o0.y);
                    unpack_int4x8(w.y, o0.z, o0.w);
                    unpack_int4x8(w.z, o1.x, o1.y);
                    unpack_int4x8(w.w, o1.z, o1.w);
                    const int atom = qc >> 2;                 // 128-column atom
                    const int c0 = (2 * qc) & 7;              // 16-column chunk inside the atom
                    uint8_t *rowp = b + atom * B_ATOM_BYTES + kr * 128;
                    *reinterpret_cast<uint4 *>(rowp + ((c0 ^ (kr & 7)) << 4)) = o0;
                    *reinterpret_cast<uint4 *>(rowp + (((c0 + 1) ^ (kr & 7)) << 4)) = o1;
                }
                ptx::fence_async_shared();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&full[stage]);
                if (++stage == S) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ---------------------------------------------------------------- K2, CTA-pair form
// Two CTAs of a cluster share one 256 x 256 tile: each loads 128 rows of x1
// and 128 columns of the expert's weights, the leader issues
// tcgen05.mma.cta_group::2 (M = 256, N = 256) that reads both CTAs' halves, and
// each CTA's TMEM receives its own 128 accumulator rows.  Per SM this moves a
// third fewer operand bytes per MAC than the single-CTA 128 x 256 tile, and a
// 32 KB stage instead of 48 KB lets the same shared memory hold five stages.
constexpr int PAIR_ROWS = 256;                 // rows per pair tile
constexpr int PAIR_A_BYTES = 128 * BK;         // this CTA's rows
constexpr int PAIR_B_BYTES = BK * 128;         // this CTA's columns (one MN-major atom)

template <bool W4>
struct PairCfg {
    // int8: 5 stages of (x1 half 16 KB + weight half 16 KB).
    // int4: 4 stages of (x1 half 16 KB + unpacked weight half 16 KB + packed half
    //       8 KB), plus 4 unpack warps.
    // Both: 4 staged epilogue warps, one per TMEM lane quarter, over all 256
    // columns (measured ~2% faster at large prefill than 8 warps of 128 columns).
    static constexpr int STAGES = W4 ? 4 : 5;
    static constexpr int EPI_WARPS = 4;
    static constexpr int THREADS = (2 + EPI_WARPS + (W4 ? 4 : 0)) * 32;
    static constexpr int P_BYTES = W4 ? PAIR_B_BYTES / 2 : 0;
    static constexpr int STAGE_BYTES = PAIR_A_BYTES + PAIR_B_BYTES + P_BYTES;
    static constexpr int NUM_BARS = 3 * STAGES + 2 + 2 + 1;
    static constexpr int CTRL_BYTES = (NUM_BARS * 8 + 16 + 15) / 16 * 16;
    static constexpr int TABLE_BYTES = (2 * (MAX_E + 1) * 4 + 15) / 16 * 16;
    static constexpr int EPI_STAGE_BYTES = EPI_WARPS * 32 * EPI_LD * 4;   // per warp 32 rows x 32 cols (+pad)
    static constexpr int ROWINFO_BYTES = EPI_WARPS * 32 * 16;
    static constexpr size_t OFF_CTRL = size_t(STAGES) * STAGE_BYTES;
    static constexpr size_t OFF_TABLE = OFF_CTRL + CTRL_BYTES;
    static constexpr size_t OFF_EPI = OFF_TABLE + TABLE_BYTES;
    static constexpr size_t OFF_ROWS = OFF_EPI + EPI_STAGE_BYTES;
    static constexpr size_t SMEM_BYTES = 1024 + OFF_ROWS + ROWINFO_BYTES;
    static_assert(SMEM_BYTES <= 232448, "shared memory above the sm_100 per-block limit");
};

template <int EPI, bool W4, bool F8 = false>
__global__ void __launch_bounds__(PairCfg<W4>::THREADS, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                             const GemmArgs args)
{
    using Cfg = PairCfg<W4>;
    constexpr int S = Cfg::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *smem_a = smem;
    uint8_t *smem_b = smem_a + S * PAIR_A_BYTES;
    uint8_t *smem_p = smem_b + S * PAIR_B_BYTES;       // W4: packed int4 weight half
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_CTRL);
    uint64_t *full = bars;            // leader: both CTAs' operands landed
    uint64_t *empty = bars + S;       // both: pair MMAs finished reading the stage
    uint64_t *tfull = bars + 2 * S;   // both: accumulator buffer ready
    uint64_t *tempty = tfull + 2;     // leader: both CTAs' epilogues drained the buffer
    uint64_t *drain = tempty + 2;     // leader: all issued MMAs completed
    uint64_t *pfull = drain + 1;      // W4, both: this CTA's x1 half and packed weight half landed
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + Cfg::NUM_BARS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    int32_t *off = reinterpret_cast<int32_t *>(smem + Cfg::OFF_TABLE);
    int32_t *cum = off + (MAX_E + 1);
    float *epi_stage = reinterpret_cast<float *>(smem + Cfg::OFF_EPI);
    float *row_pts = reinterpret_cast<float *>(smem + Cfg::OFF_ROWS);
    float *row_lg = row_pts + Cfg::EPI_WARPS * 32;
    long long *row_dst = reinterpret_cast<long long *>(row_lg + Cfg::EPI_WARPS * 32);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();
    const bool leader = rank == 0;
    const int cluster = blockIdx.x >> 1;
    const int nclusters = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(&full[s], W4 ? 8 : 1);   // W4: the 4 unpack warps of each CTA
            ptx::mbar_init(&empty[s], 1);
            ptx::mbar_init(&pfull[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&tfull[b], 1);
            ptx::mbar_init(&tempty[b], 2 * Cfg::EPI_WARPS);   // the epilogue warps of both CTAs
        }
        ptx::mbar_init(drain, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    volatile uint32_t *group_flags = reinterpret_cast<volatile uint32_t *>(tmem_holder + 2);
    if (warp == 0) {
        const uint32_t flags =
            decode_groups_warp(args.group_list, args.e, args.group_list_type, args.m, PAIR_ROWS, args.sched, off, cum);
        if (lane == 0) {
            *group_flags = flags;
            ptx::prefetch_tmap(&map_a);
            ptx::prefetch_tmap(&map_b);
        }
    } else if (warp == 1) {
        ptx::tmem_alloc_pair(tmem_holder, TMEM_COLS);
        ptx::tmem_relinquish_pair();
    }
    ptx::tc_fence_before();
    ptx::cluster_sync();   // barriers of both CTAs initialised before any TMA or remote arrive
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    const int e = args.e;
    const int MT = cum[e];
    const int NT = args.n / BN;
    const int SW = args.slab_ntiles;
    const int T = MT * NT;
    const int KB = args.k / BK;

    // The status word is cleared by the kernel this one may overlap under programmatic
    // dependent launch: wait for that kernel before setting a bit in it.
    auto fail = [&]() {
        ptx::pdl_wait_primary();
        atomicOr(args.status, QGMM_DEV_TIMEOUT);
        *abort_flag = 1;
    };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both CTAs)
        if (lane == 0) {
            constexpr uint32_t TX = 2u * (PAIR_A_BYTES + PAIR_B_BYTES);   // both halves count on the leader
            uint32_t issued[S];
#pragma unroll
            for (int s = 0; s < S; ++s) issued[s] = 0;
            int stage = 0;
            uint32_t phase = 0;
            bool ok = args.stall_producer == 0;
            for (int t = cluster; t < T && ok; t += nclusters) {
                const TileCoord c = tile_coord(t, MT, SW, off, cum, e, PAIR_ROWS, args.sched);
                const int my_row = c.row0 + (c.tail ? 64 : 128) * static_cast<int>(rank);
                const int my_col = c.nt * BN + 128 * static_cast<int>(rank);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!ptx::mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) {
                        fail();
                        ok = false;
                        break;
                    }
                    if constexpr (W4) {
                        // this CTA's x1 half and packed weight half, counted on its own barrier;
                        // the unpack warps report to the leader once the int8 half is written
                        ptx::mbar_arrive_expect_tx(&pfull[stage], PAIR_A_BYTES + Cfg::P_BYTES);
                        ptx::tma_load_2d(smem_a + stage * PAIR_A_BYTES, &map_a, &pfull[stage], kb * BK, my_row);
                        ptx::tma_load_3d(smem_p + stage * Cfg::P_BYTES, &map_b, &pfull[stage], my_col / 8, kb * BK,
                                         c.g);
                    } else {
                        if (leader) ptx::mbar_arrive_expect_tx(&full[stage], TX);
                        const uint32_t fb = ptx::map_to_rank(&full[stage], 0);
                        ptx::tma_load_2d_pair(smem_a + stage * PAIR_A_BYTES, &map_a, fb, kb * BK, my_row);
                        if (args.b_kmajor)
                            ptx::tma_load_3d_pair(smem_b + stage * PAIR_B_BYTES, &map_b, fb, kb * BK, my_col, c.g);
                        else
                            ptx::tma_load_3d_pair(smem_b + stage * PAIR_B_BYTES, &map_b, fb, my_col, kb * BK, c.g);
                    }
                    ++issued[stage];
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok && (W4 || leader)) {
                // let the copies already in flight land before the CTA leaves
                for (int s = 0; s < S; ++s) {
                    if (issued[s] == 0) continue;
                    volatile int never = 0;
                    ptx::mbar_wait(W4 ? &pfull[s] : &full[s], (issued[s] - 1u) & 1u, &never);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader CTA only)
        if (lane == 0 && leader) {
            const bool bk = args.b_kmajor != 0;
            const uint32_t IDESC_FULL = F8 ? ptx::idesc_e4m3(2 * BM, BN, !bk)   // 256 rows: 128 per CTA
                                           : ptx::idesc_i8(2 * BM, BN, !bk);
            const uint32_t IDESC_TAIL = F8 ? ptx::idesc_e4m3(BM, BN, !bk)       // 128 rows: 64 per CTA
                                           : ptx::idesc_i8(BM, BN, !bk);
            const uint32_t b_kstep = bk ? UMMA_K : UMMA_K * 128, b_lbo = bk ? 16 : B_ATOM_BYTES;
            int stage = 0;
            uint32_t phase = 0;
            int lt = 0;
            bool ok = true;
            for (int t = cluster; t < T && ok; t += nclusters, ++lt) {
                const bool tail = args.sched == SCHED_PAIRS_TAIL128 &&
                                  tile_coord(t, MT, SW, off, cum, e, PAIR_ROWS, args.sched).tail;
                const uint32_t IDESC = tail ? IDESC_TAIL : IDESC_FULL;
                const int buf = lt & 1;
                const uint32_t use = static_cast<uint32_t>(lt >> 1) & 1u;
                if (!ptx::mbar_wait(&tempty[buf], use ^ 1u, abort_flag)) {
                    fail();
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!ptx::mbar_wait<W4>(&full[stage], phase, abort_flag)) {
                        fail();
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t a0 = ptx::smem_addr(smem_a + stage * PAIR_A_BYTES);
                    const uint32_t b0 = ptx::smem_addr(smem_b + stage * PAIR_B_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / UMMA_K; ++kk) {
                        const uint64_t adesc = ptx::smem_desc_sw128(a0 + kk * UMMA_K, 16, 1024);
                        const uint64_t bdesc = ptx::smem_desc_sw128(b0 + kk * b_kstep, b_lbo, 1024);
                        if constexpr (F8)
                            ptx::mma_e4m3_pair(d_tmem, adesc, bdesc, IDESC, (kb | kk) != 0 ? 1u : 0u);
                        else
                            ptx::mma_i8_pair(d_tmem, adesc, bdesc, IDESC, (kb | kk) != 0 ? 1u : 0u);
                    }
                    ptx::mma_commit_pair(ptx::map_to_rank(&empty[stage], 0));
                    ptx::mma_commit_pair(ptx::map_to_rank(&empty[stage], 1));
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) {
                    ptx::mma_commit_pair(ptx::map_to_rank(&tfull[buf], 0));
                    ptx::mma_commit_pair(ptx::map_to_rank(&tfull[buf], 1));
                }
            }
            ptx::mma_commit_pair(ptx::map_to_rank(drain, 0));
            volatile int never = 0;
            ptx::mbar_wait(drain, 0, &never);
        }
        __syncwarp();
    } else if (warp < 2 + Cfg::EPI_WARPS) {
        // ------------------------------------------------ epilogue (both CTAs, own rows)
        ptx::pdl_wait_primary();   // the output (and status word) are initialised by the previous kernel
        if (warp == 2 && lane == 0 && blockIdx.x == 0 && *group_flags) atomicOr(args.status, *group_flags);
        const int q = warp & 3;   // TMEM lane quarter of this warp; it covers all 256 columns
        constexpr int SHIFT = W4 ? W4_ACC_SHIFT : 0;
        const EpiSmem sm = epi_smem(epi_stage, row_pts, row_lg, row_dst, warp - 2);
        uint32_t tempty_leader[2];
        tempty_leader[0] = ptx::map_to_rank(&tempty[0], 0);
        tempty_leader[1] = ptx::map_to_rank(&tempty[1], 0);
        int lt = 0;
        for (int t = cluster; t < T; t += nclusters, ++lt) {
            const TileCoord c = tile_coord(t, MT, SW, off, cum, e, PAIR_ROWS, args.sched);
            const int buf = lt & 1;
            const uint32_t use = static_cast<uint32_t>(lt >> 1) & 1u;
            const uint32_t acc = tmem_base + static_cast<uint32_t>(buf * BN);
            const int64_t base_tail = static_cast<int64_t>(c.row0) + 64 * static_cast<int>(rank);
            const int64_t base_full = static_cast<int64_t>(c.row0) + 128 * static_cast<int>(rank);
            bool ok;
            if (c.tail) {
                // M=128 pair tile: this CTA's 64 rows; TMEM lanes 0-63 hold columns 0-127,
                // lanes 64-127 hold columns 128-255, in the buffer's first 128 columns.
                ok = epilogue_tile<EPI, 4, SHIFT, F8>(args, c, base_tail, 64, 32 * (q & 1), acc, q, 0, (q >> 1) * 128,
                                                      lane, &tfull[buf], use, abort_flag, sm);
            } else {
                ok = epilogue_tile<EPI, NCHUNK, SHIFT, F8>(args, c, base_full, 128, q * 32, acc, q, 0, 0, lane,
                                                           &tfull[buf], use, abort_flag, sm);
            }
            if (!ok) {
                fail();
                break;
            }
            if (lane == 0) ptx::mbar_arrive_cluster(tempty_leader[buf]);
        }
    } else if constexpr (W4) {
        // ------------------------------------------------ int4 -> int8 unpack of this CTA's weight half
        // Packed stage: BK rows x 64 bytes (128 columns, 8 per int32 word).  Unpacked:
        // one 128-column MN-major atom, BK rows x 128 bytes, 128-byte swizzle.
        const int ut = threadIdx.x - (2 + Cfg::EPI_WARPS) * 32;   // 0..127
        const uint32_t full_leader0 = ptx::map_to_rank(&full[0], 0);
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int t = cluster; t < T && ok; t += nclusters) {
            for (int kb = 0; kb < KB; ++kb) {
                if (!ptx::mbar_wait(&pfull[stage], phase, abort_flag)) {
                    fail();
                    ok = false;
                    break;
                }
                const uint8_t *pk = smem_p + stage * Cfg::P_BYTES;
                uint8_t *bb = smem_b + stage * PAIR_B_BYTES;
                const int qc = ut & 3;                   // 16-byte packed chunk: columns 32*qc .. 32*qc+31
#pragma unroll
                for (int it = 0; it < 4; ++it) {
                    const int kr = (ut >> 2) + 32 * it;  // k row within the stage
                    const uint4 w = *reinterpret_cast<const uint4 *>(pk + kr * 64 + qc * 16);
                    uint4 o0, o1;
                    unpack_int4x8(w.x, o0.x, o0.y);
                    unpack_int4x8(w.y, o0.z, o0.w);
                    unpack_int4x8(w.z, o1.x, o1.y);
                    unpack_int4x8(w.w, o1.z, o1.w);
                    const int c0 = 2 * qc;               // 16-column chunk inside the atom
                    uint8_t *rowp = bb + kr * 128;
                    *reinterpret_cast<uint4 *>(rowp + ((c0 ^ (kr & 7)) << 4)) = o0;
                    *reinterpret_cast<uint4 *>(rowp + (((c0 + 1) ^ (kr & 7)) << 4)) = o1;
                }
                ptx::fence_async_shared();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive_cluster_release(full_leader0 + stage * 8u);
                if (++stage == S) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    }

    ptx::tc_fence_before();
    ptx::cluster_sync();   // no remote arrive or pair MMA still targets either CTA
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

// ---------------------------------------------------------------- K2, MxA8W4 form
// Page 1's Atlas 350 MxA8W4 mode: x1 FLOAT8 E4M3 [m, k] with an E8M0 scale per 32
// k-elements (sfa [m, k/32]); weights FP4 E2M1, transposed (e, n, k) and packed two
// per byte (lower k in the low nibble), with an E8M0 scale per 32 k-elements (sfb
// [e, n, k/32]).  Single CTA, M = 128 rows x N = 128 columns per tile, K = 128 per
// stage.  The producer TMA-loads the x1 tile (128-byte swizzle) and the packed
// weight tile through the padded 4-bit tensor-map type: every 16 E2M1 values (8
// bytes in global memory) land in a 16-byte shared-memory chunk, data first, then 8
// unused bytes, so the tile has the K-major 128-byte-swizzled layout of an 8-bit
// operand, which is what tcgen05.mma reads for an E2M1 operand of kind::mxf8f6f4
// (measured: the tensor core takes a group's 16 values from the chunk's first 8
// bytes, lower nibble first, and ignores the rest).  The copy's transaction count
// is the packed bytes (8 KB per stage), not the 16 KB it writes.  The stage's scale
// words (4 blocks of each of the tile's rows and columns) arrive as two 512-byte
// atoms, bulk-copied on the same barrier, already in the 32 x 16-byte layout that
// tcgen05.cp .32x128b.warpx4 takes: byte (r % 32) * 16 + (r / 32) * 4 + b.  A pre-pass
// (mx_sf_atoms_rows_kernel, mx_sf_atoms_cols_kernel) writes the atoms; loading the
// words row by row in the producer cost a third of the kernel's time.  The MMA
// thread copies the scale words
// into tensor memory and issues tcgen05.mma.kind::mxf8f6f4.block_scale (E4M3 x
// E2M1, one scale byte per 32 K per row of A and column of B, selected per
// instruction), accumulating f32 in TMEM.
// The epilogue is the staged one with unit scale and pertokenScale: the block
// scales already sit inside the accumulator, so y = (acc + bias) * logit.
constexpr int MX_BN = 128;                     // output columns per MX tile
constexpr int MX_SF_BYTES = 512;               // one stage's scale words of 128 rows (or columns)
constexpr uint32_t MX_TMEM_SF = 2 * MX_BN;     // TMEM column of the scale-factor buffers

struct MxCfg {
    static constexpr int STAGES = 5;
    static constexpr int EPI_WARPS = 4;
    static constexpr int THREADS = (2 + EPI_WARPS) * 32;
    static constexpr int A_BYTES = BM * BK;            // x1 tile
    static constexpr int B_BYTES = MX_BN * BK;         // padded E2M1 weight tile (16 values per 16 bytes)
    static constexpr int B_TX_BYTES = MX_BN * BK / 2;  // the bytes its copy reads, which the barrier counts
    static constexpr int NUM_BARS = 2 * STAGES + 2 + 2 + 1;
    static constexpr int CTRL_BYTES = (NUM_BARS * 8 + 16 + 15) / 16 * 16;
    static constexpr int TABLE_BYTES = (2 * (MAX_E + 1) * 4 + 15) / 16 * 16;
    static constexpr int EPI_STAGE_BYTES = EPI_WARPS * 32 * EPI_LD * 4;
    static constexpr int ROWINFO_BYTES = EPI_WARPS * 32 * 16;
    static constexpr size_t OFF_B = size_t(STAGES) * A_BYTES;
    static constexpr size_t OFF_SFA = OFF_B + size_t(STAGES) * B_BYTES;
    static constexpr size_t OFF_SFB = OFF_SFA + size_t(STAGES) * MX_SF_BYTES;
    static constexpr size_t OFF_CTRL = OFF_SFB + size_t(STAGES) * MX_SF_BYTES;
    static constexpr size_t OFF_TABLE = OFF_CTRL + CTRL_BYTES;
    static constexpr size_t OFF_EPI = OFF_TABLE + TABLE_BYTES;
    static constexpr size_t OFF_ROWS = OFF_EPI + EPI_STAGE_BYTES;
    static constexpr size_t SMEM_BYTES = 1024 + OFF_ROWS + ROWINFO_BYTES;
    static_assert(SMEM_BYTES <= 232448, "shared memory above the sm_100 per-block limit");
};

template <int EPI>
__global__ void __launch_bounds__(MxCfg::THREADS, 1)
    grouped_gemm_mx_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                           const GemmArgs args)
{
    using Cfg = MxCfg;
    constexpr int S = Cfg::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *smem_a = smem;
    uint8_t *smem_b = smem + Cfg::OFF_B;
    uint8_t *smem_sfa = smem + Cfg::OFF_SFA;
    uint8_t *smem_sfb = smem + Cfg::OFF_SFB;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_CTRL);
    uint64_t *full = bars;            // x1 and weight tiles landed, scale words written
    uint64_t *empty = bars + S;       // MMAs finished reading the stage
    uint64_t *tfull = bars + 2 * S;   // accumulator buffer ready for the epilogue
    uint64_t *tempty = tfull + 2;     // epilogue drained the accumulator buffer
    uint64_t *drain = tempty + 2;     // all issued MMAs completed
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(bars + Cfg::NUM_BARS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_holder + 1);
    int32_t *off = reinterpret_cast<int32_t *>(smem + Cfg::OFF_TABLE);
    int32_t *cum = off + (MAX_E + 1);
    float *epi_stage = reinterpret_cast<float *>(smem + Cfg::OFF_EPI);
    float *row_pts = reinterpret_cast<float *>(smem + Cfg::OFF_ROWS);
    float *row_lg = row_pts + Cfg::EPI_WARPS * 32;
    long long *row_dst = reinterpret_cast<long long *>(row_lg + Cfg::EPI_WARPS * 32);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(&full[s], 1);   // the producer's expect_tx arrival; the copies complete the bytes
            ptx::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(&tfull[b], 1);
            ptx::mbar_init(&tempty[b], Cfg::EPI_WARPS);
        }
        ptx::mbar_init(drain, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    volatile uint32_t *group_flags = reinterpret_cast<volatile uint32_t *>(tmem_holder + 2);
    if (warp == 0) {
        const uint32_t flags = decode_groups_warp(args.group_list, args.e, args.group_list_type, args.m, BM,
                                                  SCHED_TILES, off, cum);
        if (lane == 0) {
            *group_flags = flags;
            ptx::prefetch_tmap(&map_a);
            ptx::prefetch_tmap(&map_b);
        }
    } else if (warp == 1) {
        ptx::tmem_alloc(tmem_holder, 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    const int e = args.e;
    const int MT = cum[e];
    const int NT = args.n / MX_BN;
    const int SW = args.slab_ntiles;
    const int T = MT * NT;
    const int KB = args.k / BK;

    // The status word is cleared by the kernel this one may overlap under programmatic
    // dependent launch: wait for that kernel before setting a bit in it.
    auto fail = [&]() {
        ptx::pdl_wait_primary();
        atomicOr(args.status, QGMM_DEV_TIMEOUT);
        *abort_flag = 1;
    };

    if (warp == 0) {
        // ------------------------------------------------ producer: TMA (lane 0) and scale words (all lanes)
        uint32_t issued[S];
#pragma unroll
        for (int s = 0; s < S; ++s) issued[s] = 0;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = args.stall_producer == 0;
        for (int t = blockIdx.x; t < T && ok; t += gridDim.x) {
            const TileCoord c = tile_coord(t, MT, SW, off, cum, e, BM, SCHED_TILES);
            const int n0 = c.nt * MX_BN;
            for (int kb = 0; kb < KB; ++kb) {
                bool got = true;
                if (lane == 0) got = ptx::mbar_wait(&empty[stage], phase ^ 1u, abort_flag);
                got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
                if (!got) {
                    if (lane == 0) fail();
                    ok = false;
                    break;
                }
                if (lane == 0) {
                    // the x1 tile, the padded weight tile, and the stage's two 512-byte scale
                    // atoms (arranged by mx_sf_atoms_*_kernel in the layout tcgen05.cp takes)
                    ptx::mbar_arrive_expect_tx(&full[stage], Cfg::A_BYTES + Cfg::B_TX_BYTES + 2 * MX_SF_BYTES);
                    ptx::tma_load_2d(smem_a + stage * Cfg::A_BYTES, &map_a, &full[stage], kb * BK, c.row0);
                    ptx::tma_load_3d(smem_b + stage * Cfg::B_BYTES, &map_b, &full[stage], kb * BK, n0, c.g);
                    ptx::bulk_load(smem_sfa + stage * MX_SF_BYTES,
                                   args.sfa + (static_cast<int64_t>(c.mt) * KB + kb) * MX_SF_BYTES, MX_SF_BYTES,
                                   &full[stage]);
                    ptx::bulk_load(smem_sfb + stage * MX_SF_BYTES,
                                   args.sfb + ((static_cast<int64_t>(c.g) * NT + c.nt) * KB + kb) * MX_SF_BYTES,
                                   MX_SF_BYTES, &full[stage]);
                }
                ++issued[stage];
                if (++stage == S) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok && lane == 0) {
            // let the copies already in flight land before the CTA leaves
            for (int s = 0; s < S; ++s) {
                if (issued[s] == 0) continue;
                volatile int never = 0;
                ptx::mbar_wait(&full[s], (issued[s] - 1u) & 1u, &never);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t sf_buf = 0;
            int lt = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < T && ok; t += gridDim.x, ++lt) {
                const int buf = lt & 1;
                const uint32_t use = static_cast<uint32_t>(lt >> 1) & 1u;
                if (!ptx::mbar_wait(&tempty[buf], use ^ 1u, abort_flag)) {
                    fail();
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * MX_BN);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!ptx::mbar_wait(&full[stage], phase, abort_flag)) {
                        fail();
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    // this stage's scale words into TMEM (two buffers, alternating per k-block)
                    const uint32_t sfa_t = tmem_base + MX_TMEM_SF + 8u * sf_buf;
                    sf_buf ^= 1u;
                    const uint32_t sfb_t = sfa_t + 4u;
                    ptx::tmem_cp_32x128b_warpx4(sfa_t, ptx::smem_desc_noswizzle(
                                                           ptx::smem_addr(smem_sfa + stage * MX_SF_BYTES), 16, 128));
                    ptx::tmem_cp_32x128b_warpx4(sfb_t, ptx::smem_desc_noswizzle(
                                                           ptx::smem_addr(smem_sfb + stage * MX_SF_BYTES), 16, 128));
                    const uint32_t a0 = ptx::smem_addr(smem_a + stage * Cfg::A_BYTES);
                    const uint32_t b0 = ptx::smem_addr(smem_b + stage * Cfg::B_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / UMMA_K; ++kk) {
                        const uint64_t adesc = ptx::smem_desc_sw128(a0 + kk * UMMA_K, 16, 1024);
                        const uint64_t bdesc = ptx::smem_desc_sw128(b0 + kk * UMMA_K, 16, 1024);
                        ptx::mma_mx_e4m3(d_tmem, adesc, bdesc, ptx::idesc_mx_e4m3(BM, MX_BN, kk, kk, true), sfa_t,
                                         sfb_t, (kb | kk) != 0 ? 1u : 0u);
                    }
                    ptx::mma_commit(&empty[stage]);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) ptx::mma_commit(&tfull[buf]);
            }
            ptx::mma_commit(drain);
            volatile int never = 0;
            ptx::mbar_wait(drain, 0, &never);
        }
        __syncwarp();
    } else if (warp < 2 + Cfg::EPI_WARPS) {
        // ------------------------------------------------ epilogue: 4 warps, staged through smem
        ptx::pdl_wait_primary();
        if (warp == 2 && lane == 0 && blockIdx.x == 0 && *group_flags) atomicOr(args.status, *group_flags);
        const int q = warp & 3;
        const EpiSmem sm = epi_smem(epi_stage, row_pts, row_lg, row_dst, q);
        int lt = 0;
        for (int t = blockIdx.x; t < T; t += gridDim.x, ++lt) {
            const TileCoord c = tile_coord(t, MT, SW, off, cum, e, BM, SCHED_TILES);
            const int buf = lt & 1;
            const uint32_t use = static_cast<uint32_t>(lt >> 1) & 1u;
            if (!epilogue_tile<EPI, MX_BN / 32, 0, true>(args, c, c.row0, BM, q * 32,
                                                         tmem_base + static_cast<uint32_t>(buf * MX_BN), q, 0, 0,
                                                         lane, &tfull[buf], use, abort_flag, sm, MX_BN)) {
                fail();
                break;
            }
            if (lane == 0) ptx::mbar_arrive(&tempty[buf]);
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, 512);
    }
}

// ---------------------------------------------------------------- MxA8W4 scale atoms
// Atom layout (512 bytes, the 32 x 16-byte source of tcgen05.cp .32x128b.warpx4):
// word i * 4 + j holds the scale bytes of k-blocks 4 kb .. 4 kb + 3 of the tile's
// row (or column) i + 32 j.  x1's atoms are indexed (m-tile of the MX kernel's walk,
// kb), the weights' (expert * n/128 + 128-column tile, kb).  One block of 128
// threads per tile; thread i * 4 + j walks its row's words over k.
__global__ void mx_sf_atoms_rows_kernel(const uint8_t *__restrict__ sfa, int64_t m, int32_t k, const int64_t *gl,
                                        int e, int type, uint32_t *__restrict__ atoms)
{
    __shared__ int32_t off[MAX_E + 1], cum[MAX_E + 1];
    if (threadIdx.x < 32) decode_groups_warp(gl, e, type, m, BM, SCHED_TILES, off, cum);   // the MX kernel's tiles
    __syncthreads();
    const int MT = cum[e];
    const int KB = k / BK;
    const int i = threadIdx.x >> 2, j = threadIdx.x & 3;
    for (int mt = blockIdx.x; mt < MT; mt += gridDim.x) {
        int lo = 0, hi = e;   // cum[lo] <= mt < cum[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (cum[mid] <= mt) lo = mid;
            else hi = mid;
        }
        const int64_t r = int64_t(off[lo]) + int64_t(mt - cum[lo]) * BM + i + 32 * j;
        const uint32_t *src = reinterpret_cast<const uint32_t *>(sfa + (r < m ? r : 0) * (k / 32));
        uint32_t *dst = atoms + int64_t(mt) * KB * 128 + threadIdx.x;
        for (int kb = 0; kb < KB; ++kb) dst[int64_t(kb) * 128] = r < m ? __ldg(src + kb) : 0u;   // rows past m: 0
    }
}

__global__ void mx_sf_atoms_cols_kernel(const uint8_t *__restrict__ sfb, int e, int32_t n, int64_t ld_sb, int32_t k,
                                        uint32_t *__restrict__ atoms)
{
    const int NT = n / MX_BN, KB = k / BK;
    const int i = threadIdx.x >> 2, j = threadIdx.x & 3;
    for (int64_t a = blockIdx.x; a < int64_t(e) * NT; a += gridDim.x) {
        const int64_t g = a / NT, nt = a - g * NT;
        const uint32_t *src = reinterpret_cast<const uint32_t *>(sfb + (g * ld_sb + nt * MX_BN + i + 32 * j) * (k / 32));
        uint32_t *dst = atoms + a * KB * 128 + threadIdx.x;
        for (int kb = 0; kb < KB; ++kb) dst[int64_t(kb) * 128] = __ldg(src + kb);
    }
}

// ---------------------------------------------------------------- K1
// out[r][:] = f32(shared[r - off][:]) for r in [off, off + bs), else 0, over n
// columns; out rows are ld apart, shared rows ld_sh apart.  Also clears the
// call's status word.  A block walks whole rows; a thread step reads
// 8 bf16 (16 bytes) and writes two float4.  The host launches 2 blocks of 256
// threads per SM, which leaves room on every SM for a grouped-GEMM CTA that
// programmatic dependent launch lets start while this kernel still runs.
__global__ void output_init_kernel(float *__restrict__ out, int64_t output_bs, int32_t n, int64_t ld,
                                   const uint16_t *__restrict__ shared, int64_t ld_sh, int64_t shared_bs,
                                   int64_t shared_off, uint32_t *status)
{
    ptx::pdl_launch_dependents();   // the grouped GEMM may start its prologue and mainloop now
    if (blockIdx.x == 0 && threadIdx.x == 0) *status = 0u;
    const int n8 = n / 8;           // n % 256 == 0
    for (int64_t r = blockIdx.x; r < output_bs; r += gridDim.x) {
        float4 *dst = reinterpret_cast<float4 *>(out + r * ld);
        const bool sh = shared != nullptr && r >= shared_off && r < shared_off + shared_bs;
        const uint4 *src = reinterpret_cast<const uint4 *>(shared + (sh ? (r - shared_off) * ld_sh : 0));
        for (int c = threadIdx.x; c < n8; c += blockDim.x) {
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
            if (sh) {
                const uint4 h = __ldg(src + c);   // bf16 -> f32 is exact: the bits move up 16 places
                a = make_float4(__uint_as_float(h.x << 16), __uint_as_float(h.x & 0xFFFF0000u),
                                __uint_as_float(h.y << 16), __uint_as_float(h.y & 0xFFFF0000u));
                b = make_float4(__uint_as_float(h.z << 16), __uint_as_float(h.z & 0xFFFF0000u),
                                __uint_as_float(h.w << 16), __uint_as_float(h.w & 0xFFFF0000u));
            }
            dst[2 * c] = a;
            dst[2 * c + 1] = b;
        }
    }
}

__global__ void clear_status_kernel(uint32_t *status)
{
    ptx::pdl_launch_dependents();
    *status = 0u;
}

// ---------------------------------------------------------------- K3 (deterministic combine)
// The destination-sorted list of source rows is built in source-row order, so no
// bucket is ever sorted.  The rows below the total are cut into nseg segments of
// L = ceil(total / nseg) consecutive rows.  Workspace:
//   counts[nseg][output_bs]  per-segment histogram of destinations, then (after
//                            det_colscan) the segment's first slot inside each bucket
//   starts[output_bs + 1]    bucket boundaries (exclusive scan of the bucket sizes)
//   list[m]                  source rows grouped by destination, ascending in each
// det_fill gives each segment to one warp, which walks its rows in ascending order,
// so every bucket receives segment 0's rows first, each segment's rows in order.
__global__ void det_clear_kernel(int32_t *counts, int64_t entries, uint32_t *status)
{
    if (blockIdx.x == 0 && threadIdx.x == 0) *status = 0u;
    for (int64_t r = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; r < entries;
         r += int64_t(gridDim.x) * blockDim.x)
        counts[r] = 0;
}

// Shared by the histogram and fill kernels: rows below the total (from groupList).
__device__ __forceinline__ int64_t groups_total_block(const int64_t *gl, int e, int type, int64_t m, int32_t *off,
                                                      int32_t *cum, uint32_t *status, bool report)
{
    if (threadIdx.x < 32) {
        const uint32_t f = decode_groups_warp(gl, e, type, m, BM, SCHED_TILES, off, cum);
        if (threadIdx.x == 0 && report && f) atomicOr(status, f);
    }
    __syncthreads();
    return off[e];
}

// K1 for identity routing without sharedInput: every output row then receives at
// most one source row, which the grouped GEMM stores directly (EPI_STORE_Y into out);
// this kernel zeroes the rows at or past the groups' total, which receive none, and
// clears the call's status word.
__global__ void output_tail_zero_kernel(float *__restrict__ out, int64_t output_bs, int32_t n, int64_t ld,
                                        const int64_t *gl, int e, int type, int64_t m, uint32_t *status)
{
    ptx::pdl_launch_dependents();   // the grouped GEMM may start its prologue and mainloop now
    if (blockIdx.x == 0 && threadIdx.x == 0) *status = 0u;
    __shared__ int32_t off[MAX_E + 1], cum[MAX_E + 1];
    const int64_t total = groups_total_block(gl, e, type, m, off, cum, status, false);   // the GEMM reports
    const int n4 = n / 4;
    for (int64_t r = total + blockIdx.x; r < output_bs; r += gridDim.x) {
        float4 *dst = reinterpret_cast<float4 *>(out + r * ld);
        for (int c = threadIdx.x; c < n4; c += blockDim.x) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

__global__ void det_hist_kernel(const int64_t *gl, int e, int type, int64_t m, const void *row_index, int ri_type,
                                int64_t output_bs, int32_t nseg, int32_t *counts, uint32_t *status)
{
    __shared__ int32_t off[MAX_E + 1], cum[MAX_E + 1];
    const int64_t total = groups_total_block(gl, e, type, m, off, cum, status, blockIdx.x == 0);
    const int64_t seg_len = (total + nseg - 1) / nseg;
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t d = load_row_index(row_index, ri_type, i);
        if (d < 0 || d >= output_bs) {
            atomicOr(status, QGMM_DEV_ROW_INDEX_RANGE);
            continue;
        }
        atomicAdd(counts + (i / seg_len) * output_bs + d, 1);
    }
}

// Per destination d: counts[s][d] <- rows of d in segments before s; sizes[d] <- all rows of d.
__global__ void det_colscan_kernel(int32_t *counts, int32_t nseg, int64_t output_bs, int32_t *sizes)
{
    for (int64_t d = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; d < output_bs;
         d += int64_t(gridDim.x) * blockDim.x) {
        int32_t run = 0;
        for (int32_t s = 0; s < nseg; ++s) {
            int32_t *c = counts + s * output_bs + d;
            const int32_t v = *c;
            *c = run;
            run += v;
        }
        sizes[d] = run;
    }
}

// Single block, in place: starts[0..output_bs) holds the bucket sizes on entry and
// their exclusive scan on exit; starts[output_bs] = the sum.
__global__ void det_scan_kernel(int32_t *starts, int64_t output_bs)
{
    __shared__ int32_t warp_sums[32];
    __shared__ int32_t carry;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int64_t base = 0; base < output_bs; base += blockDim.x) {
        const int64_t r = base + threadIdx.x;
        const int32_t v = r < output_bs ? starts[r] : 0;
        int32_t s = v;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int32_t o = __shfl_up_sync(0xffffffffu, s, d);
            if (lane >= d) s += o;
        }
        if (lane == 31) warp_sums[w] = s;
        __syncthreads();
        if (w == 0) {
            int32_t ws = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int32_t o = __shfl_up_sync(0xffffffffu, ws, d);
                if (lane >= d) ws += o;
            }
            if (lane < nw) warp_sums[lane] = ws;
        }
        __syncthreads();
        const int32_t excl = carry + (w ? warp_sums[w - 1] : 0) + s - v;
        if (r < output_bs) starts[r] = excl;
        __syncthreads();
        if (threadIdx.x == blockDim.x - 1) carry = excl + v;
        __syncthreads();
    }
    if (threadIdx.x == 0) starts[output_bs] = carry;
}

// One warp per segment, 32 source rows at a time in ascending order.  Lanes with the
// same destination find each other with __match_any_sync and take consecutive slots
// in lane order after the segment's cursor for that destination; the group's lowest
// lane then advances the cursor.
__global__ void det_fill_kernel(const int64_t *gl, int e, int type, int64_t m, const void *row_index, int ri_type,
                                int64_t output_bs, int32_t nseg, int32_t *cursor, const int32_t *starts,
                                int32_t *list)
{
    __shared__ int32_t off[MAX_E + 1], cum[MAX_E + 1];
    const int64_t total = groups_total_block(gl, e, type, m, off, cum, nullptr, false);
    const int64_t seg_len = (total + nseg - 1) / nseg;
    const int lane = threadIdx.x & 31;
    const int wpb = blockDim.x >> 5;
    for (int64_t s = int64_t(blockIdx.x) * wpb + (threadIdx.x >> 5); s < nseg; s += int64_t(gridDim.x) * wpb) {
        const int64_t r0 = s * seg_len;
        const int64_t r1 = r0 + seg_len < total ? r0 + seg_len : total;
        for (int64_t base = r0; base < r1; base += 32) {
            const int64_t i = base + lane;
            long long d = -1;
            if (i < r1) {
                d = load_row_index(row_index, ri_type, i);
                if (d < 0 || d >= output_bs) d = -1;
            }
            const uint32_t grp = __match_any_sync(0xffffffffu, d);
            int32_t *cur = cursor + s * output_bs + (d < 0 ? 0 : d);
            int32_t slot = 0;
            if (d >= 0) {
                slot = *cur;
                list[starts[d] + slot + __popc(grp & ((1u << lane) - 1u))] = static_cast<int32_t>(i);
            }
            __syncwarp();
            if (d >= 0 && lane == __ffs(grp) - 1) *cur = slot + __popc(grp);
            __syncwarp();
        }
    }
}

// out[r][:] = shared-or-0, then += y[j][:] for the bucket's rows j in ascending order.
// y rows are n apart, out rows ld apart, shared rows ld_sh apart.
__global__ void det_reduce_kernel(float *__restrict__ out, const float *__restrict__ y, int32_t n, int64_t ld,
                                  const int32_t *__restrict__ starts, const int32_t *__restrict__ list,
                                  int64_t output_bs, const uint16_t *__restrict__ shared, int64_t ld_sh,
                                  int64_t shared_bs, int64_t shared_off)
{
    const int32_t q_per_row = n / 4;
    for (int64_t r = blockIdx.x; r < output_bs; r += gridDim.x) {
        const int32_t a = starts[r], b = starts[r + 1];
        const bool sh = shared && r >= shared_off && r < shared_off + shared_bs;
        for (int32_t c4 = threadIdx.x; c4 < q_per_row; c4 += blockDim.x) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            if (sh) {
                const uint2 h = __ldg(reinterpret_cast<const uint2 *>(shared + (r - shared_off) * ld_sh) + c4);
                acc.x = __uint_as_float(h.x << 16);
                acc.y = __uint_as_float(h.x & 0xFFFF0000u);
                acc.z = __uint_as_float(h.y << 16);
                acc.w = __uint_as_float(h.y & 0xFFFF0000u);
            }
            // a bucket holds about topK rows: issue its loads together, then add in order
            for (int32_t x0 = a; x0 < b; x0 += 8) {
                float4 v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (x0 + u < b) v[u] = __ldg(reinterpret_cast<const float4 *>(y + int64_t(list[x0 + u]) * n) + c4);
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (x0 + u < b) {
                        acc.x = __fadd_rn(acc.x, v[u].x);
                        acc.y = __fadd_rn(acc.y, v[u].y);
                        acc.z = __fadd_rn(acc.z, v[u].z);
                        acc.w = __fadd_rn(acc.w, v[u].w);
                    }
            }
            reinterpret_cast<float4 *>(out + r * ld)[c4] = acc;
        }
    }
}

// ---------------------------------------------------------------- K0
// One warp per row: absmax over the row, then q = clamp(rn(x * (127/a)), +-127)
// and scale = a / 127, all in IEEE f32 (page 4, per_token_cast: value times a
// precomputed inverse).  k % 8 == 0; 16-byte vector loads, 8-byte stores.
// Non-finite inputs follow IEEE f32: fmaxf skips NaN elements in the absmax, an
// infinite element makes a = inf, scale = inf and inv = 0; a product x * inv that
// is NaN (a NaN input, or an infinite one times a zero inverse) gives code 0.
__global__ void per_token_quant_kernel(const uint16_t *__restrict__ x, int64_t rows, int32_t k, int8_t *__restrict__ q,
                                       float *__restrict__ scale_out)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps_total = int64_t(gridDim.x) * (blockDim.x >> 5);
    const int32_t v_per_row = k / 8;
    for (int64_t row = blockIdx.x * int64_t(blockDim.x >> 5) + (threadIdx.x >> 5); row < rows; row += warps_total) {
        const uint4 *src = reinterpret_cast<const uint4 *>(x + row * k);
        float a = 0.f;
        for (int32_t v = lane; v < v_per_row; v += 32) {
            const uint4 h = __ldg(src + v);
            const uint32_t w[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                a = fmaxf(a, fabsf(__uint_as_float(w[u] << 16)));
                a = fmaxf(a, fabsf(__uint_as_float(w[u] & 0xFFFF0000u)));
            }
        }
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, d));
        const float inv = a > 0.f ? __fdiv_rn(127.0f, a) : 0.0f;
        if (lane == 0) scale_out[row] = __fdiv_rn(a, 127.0f);
        uint2 *dst = reinterpret_cast<uint2 *>(q + row * k);
        for (int32_t v = lane; v < v_per_row; v += 32) {
            const uint4 h = __ldg(src + v);
            const uint32_t w[4] = {h.x, h.y, h.z, h.w};
            uint32_t packed[2] = {0u, 0u};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float t0 = __fmul_rn(__uint_as_float(w[u] << 16), inv);
                const float t1 = __fmul_rn(__uint_as_float(w[u] & 0xFFFF0000u), inv);
                // a NaN product has no integer code and becomes 0; infinities saturate
                const float r0 = t0 != t0 ? 0.0f : fminf(fmaxf(rintf(t0), -127.0f), 127.0f);
                const float r1 = t1 != t1 ? 0.0f : fminf(fmaxf(rintf(t1), -127.0f), 127.0f);
                const uint32_t b0 = static_cast<uint32_t>(static_cast<int32_t>(r0)) & 0xFFu;
                const uint32_t b1 = static_cast<uint32_t>(static_cast<int32_t>(r1)) & 0xFFu;
                packed[u >> 1] |= (b0 | (b1 << 8)) << (16 * (u & 1));
            }
            dst[v] = make_uint2(packed[0], packed[1]);
        }
    }
}

// ---------------------------------------------------------------- K0, FP8 form
// Per-32-group FP8 E4M3 cast (page 4, per_token_cast: the bf16 values times the
// group's broadcast inverse scale, converted to FLOAT8 E4M3FN).  Scale factors are
// E8M0 codes, one per 32 elements:
//   sf = max(0, biased f32 exponent of max|x| - 8),  inv = 2^(127 - sf)  (exact)
//   q  = E4M3(x * inv), round to nearest even, saturating at 448; NaN -> 0x7F
// x * inv is exact (a power of two), so the conversion is the only rounding.  One
// thread takes 8 bf16 (16 bytes), four neighbouring lanes a group, a warp 256
// elements of one row; k % 32 == 0.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    uint32_t v = r;
    if (lo != lo) v = (v & 0xFF00u) | 0x7Fu;          // a NaN element codes as 0x7F
    if (hi != hi) v = (v & 0x00FFu) | 0x7F00u;
    return v;
}

__global__ void per_token_quant_mxfp8_kernel(const uint16_t *__restrict__ x, int64_t rows, int32_t k,
                                             uint8_t *__restrict__ q, uint8_t *__restrict__ sf)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps_total = int64_t(gridDim.x) * (blockDim.x >> 5);
    const int32_t chunks_per_row = (k + 255) / 256;
    const int64_t chunks = rows * chunks_per_row;
    for (int64_t c = blockIdx.x * int64_t(blockDim.x >> 5) + (threadIdx.x >> 5); c < chunks; c += warps_total) {
        const int64_t row = c / chunks_per_row;
        const int32_t col = static_cast<int32_t>(c - row * chunks_per_row) * 256 + lane * 8;
        const bool valid = col < k;                    // k % 32 == 0: a group is all valid or all not
        uint4 h = make_uint4(0u, 0u, 0u, 0u);
        if (valid) h = __ldg(reinterpret_cast<const uint4 *>(x + row * k + col));
        const uint32_t w[4] = {h.x, h.y, h.z, h.w};
        float v[8];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            v[2 * u] = __uint_as_float(w[u] << 16);
            v[2 * u + 1] = __uint_as_float(w[u] & 0xFFFF0000u);
        }
        float a = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) a = fmaxf(a, fabsf(v[u]));   // fmaxf skips NaN
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
        const int biased = static_cast<int>((__float_as_uint(a) >> 23) & 0xFFu);
        const int code = biased > 8 ? biased - 8 : 0;
        const float inv = __uint_as_float(static_cast<uint32_t>(254 - code) << 23);
        if (!valid) continue;
        uint32_t lo = 0u, hi = 0u;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            lo |= e4m3x2(__fmul_rn(v[2 * u], inv), __fmul_rn(v[2 * u + 1], inv)) << (16 * u);
            hi |= e4m3x2(__fmul_rn(v[4 + 2 * u], inv), __fmul_rn(v[5 + 2 * u], inv)) << (16 * u);
        }
        *reinterpret_cast<uint2 *>(q + row * k + col) = make_uint2(lo, hi);
        if ((lane & 3) == 0) sf[row * (k / 32) + col / 32] = static_cast<uint8_t>(code);
    }
}

}  // namespace qgmm
