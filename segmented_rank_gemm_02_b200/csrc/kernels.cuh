// kernels.cuh -- interface between the host library and the sm_100a kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace mlora {

enum TileMode : int { MODE_APPLY = 0, MODE_SHRINK = 1, MODE_EXPAND = 2 };

// Grouped positions in one work tile of the segmented (decode-family) kernel: the
// top half of one m16 MMA tile (batches of long decode segments at rank <= 16 use
// 16-row tiles, the whole m16 tile; see lora_decode.cu).
constexpr int kTileRows = 8;

// Device status bits (same values as the MLORA_FLAG_* macros of the public header).
constexpr unsigned kFlagBadOffsets = 1u;
constexpr unsigned kFlagBadSlot = 2u;
constexpr unsigned kFlagBadRank = 4u;
constexpr unsigned kFlagBadRow = 8u;
constexpr unsigned kFlagSlotEmpty = 16u;
constexpr unsigned kFlagTimeout = 32u;
constexpr unsigned kFlagStaleSlot = 64u;

// Smallest rank bucket (8, 16, 32, 64) holding rank r; 0 if r is out of range.
__host__ __device__ constexpr int rank_bucket(int r)
{
    return r <= 0 ? 0 : r <= 8 ? 8 : r <= 16 ? 16 : r <= 32 ? 32 : r <= 64 ? 64 : 0;
}

// Projections one fused launch of the decode-shaped kernel may cover.
constexpr int kMaxFused = 4;

// What differs between the projections of a fused launch: each has its own pool
// (same d_in and slot numbering, its own d_out) and its own output.  Entry 0 repeats
// the single-projection fields of TileParams.
struct ProjView {
    const __nv_bfloat16 *pool;
    int64_t slot_stride;
    int64_t b_offset;
    const int32_t *slot_rank;
    const float *slot_scale;
    const uint32_t *slot_gen;
    unsigned int *status;       // this projection's status word (its slot problems)
    int32_t d_out, n_slice;
    __nv_bfloat16 *Y;
    int64_t ldy;
    float *ws;                  // fused long-segment shrink: this projection's H workspace
    int64_t ws_ld;
};

// Everything one launch of the segmented tile kernel needs.  Passed by value.
struct TileParams {
    // adapter pool: slot a's A block starts at pool + a * slot_stride and holds
    // [d_in/8][R][8] bf16 (R = bucket of the slot's rank); its B block starts
    // b_offset elements later and holds [R/8][d_out][8] bf16.
    const __nv_bfloat16 *pool;
    int64_t slot_stride;
    int64_t b_offset;
    const int32_t *slot_rank;   // [n_slots], 0 = empty
    const float *slot_scale;    // [n_slots], alpha / rank
    const uint32_t *slot_gen;   // [n_slots], generation of what the slot holds
    int32_t n_slots;
    unsigned int *status;       // device status word (MLORA_FLAG_* bits)
    int32_t d_in, d_out;
    // segment metadata (device)
    int32_t n_segments, n_rows, n_tokens;
    const int32_t *offsets;
    const int32_t *slots;
    const int32_t *ranks;       // may be null
    const float *scales;        // may be null
    const int32_t *token_indices;  // may be null (identity)
    const uint32_t *generations;   // may be null: slot generation each segment expects
    // tensors
    const __nv_bfloat16 *X;
    int64_t ldx;
    __nv_bfloat16 *Y;
    int64_t ldy;
    float *H;
    int64_t ldh;
    // decomposition: CTA c of a cluster owns d_in columns [c*k_slice, (c+1)*k_slice)
    // for the shrink and d_out columns [c*n_slice, (c+1)*n_slice) for the expand.
    int32_t k_slice, n_slice;
    // segments with at least this many grouped positions go to the long-segment
    // (tensor-memory) kernels; the others to the decode-shaped kernel
    int32_t long_rows;
    // decode-shaped kernel launched with programmatic dependent launch: its CTAs may
    // start while the previous kernel finishes, prefetch their first tile's adapter
    // slices into L2 and wait for that kernel before reading anything else.  Used
    // only for batches without long segments (the long-segment kernels want the
    // opposite shared-memory / L1 split and stream enough to evict the prefetch).
    int32_t early;
    // long-segment kernels: H of the long tiles, [n_tokens][ws_ld] fp32 (the pool's
    // workspace in the fused apply, the caller's H in standalone shrink / expand)
    float *ws;
    int64_t ws_ld;
    int32_t ksplit;            // CTAs per shrink cluster, each one part of d_in
    int32_t k_part;            // d_in columns per part (multiple of 64)
    // TMA views (bf16, 128-byte swizzle) of X [n_rows, d_in] and Y [n_rows, d_out]:
    // 64 x 128 tiles for runs of consecutive rows, 64 x 1 rows for gathers
    CUtensorMap x_tile, x_rows, y_tile, y_rows;
    // TMA views of the pool's B blocks, one per rank bucket 8, 16, 32, 64: a box is
    // one 128-column chunk of one slot's B (all its rank groups), [R/8][128][8] in
    // shared memory; its second coordinate is (first column) / b_col_div
    CUtensorMap b_map[4];
    int32_t b_col_div;
    // decode-shaped kernel: the projections it applies (1 unless fused; all share X,
    // d_in, the segment metadata and the slot numbering)
    int32_t n_proj;
    ProjView proj[kMaxFused];
    // per-tensor scale of FP8 activation codes (dtype boundary variants only)
    float x_scale;
};

// A segment [p0, p1) goes to the long-segment kernels when it holds at least
// long_rows grouped positions whose rows are consecutive in X and Y -- a prefill
// request -- judged from its first and last row; scattered rows of a much-used
// adapter (decode rows of many requests) stay with the decode-shaped kernel.  Every
// kernel applies the same test to the same metadata, so each segment is taken by
// exactly one of them.  (A segment whose rows are a permuted run still passes; the
// long kernels then gather its rows, which is correct, only slower.)
__device__ __forceinline__ bool long_segment(const TileParams &p, int p0, int p1)
{
    if (p1 - p0 < p.long_rows) return false;
    if (p.token_indices == nullptr) return true;
    return p.token_indices[p1 - 1] - p.token_indices[p0] == p1 - p0 - 1;
}

// Rows per tile of the long-segment kernels (one M=128 tensor-memory tile).
constexpr int kLongTileRows = 128;
// d_out columns per chunk of the long-segment expand.
constexpr int kExpandChunk = 128;

// Long-segment shrink (H of the long tiles into p.ws) and expand (reads p.ws; in
// MODE_EXPAND it also reports the tiles' metadata problems); persistent grids.
// np >= 2: one launch for projections 0 .. np-1 of a fused call (projection 0 from
// p's own fields, the others from p.proj[j], each H into its own workspace).
cudaError_t launch_long_shrink(int rmax_bucket, const TileParams &p, int64_t max_tiles,
                               cudaStream_t stream, int np = 1);
cudaError_t launch_long_expand(int rmax_bucket, int mode, const TileParams &p, int64_t max_tiles,
                               cudaStream_t stream);
cudaError_t prepare_long_kernels();

// CTAs per shrink cluster (1..8) for about `tiles` long tiles: the split of d_in
// that minimises waves of resident clusters times 64-column blocks per CTA.
int long_shrink_split(int rmax_bucket, int d_in, int64_t tiles);

// Launch the tile kernel for the pool's largest rank bucket `rmax_bucket`
// (8/16/32/64) in mode `mode`, with clusters of `cluster` CTAs: as many clusters as
// can be resident at once, but no more than `max_tiles` (each loops over tiles).
cudaError_t launch_tile_kernel(int mode, int rmax_bucket, const TileParams &p, int cluster,
                               int64_t max_tiles, cudaStream_t stream);

// The fused apply (MODE_APPLY, one projection) at another dtype boundary of a quantized
// base model: dt = 3 * xt + yt, xt 0 = bf16 X, 1 = FP8 e4m3 codes (times p.x_scale);
// yt 0 = bf16 Y, 1 = fp16, 2 = fp32 (1 <= dt <= 5; 0 is launch_tile_kernel's path).
cudaError_t launch_tile_kernel_dt(int dt, int rmax_bucket, const TileParams &p, int cluster, int64_t max_tiles,
                                  cudaStream_t stream);

// Fused launch over p.n_proj projections (MODE_APPLY): a work item is one tile of one
// projection, and the items of a tile are adjacent so its X rows come from HBM once.
cudaError_t launch_tile_kernel_fused(int rmax_bucket, const TileParams &p, int cluster,
                                     int64_t max_items, cudaStream_t stream);

// Set per-kernel attributes (dynamic shared memory) on the current device.
cudaError_t prepare_tile_kernels();

// Repack one adapter from the PEFT layout into a pool slot and publish its rank, scale
// and generation.
cudaError_t launch_repack_slot(__nv_bfloat16 *slot_base, int64_t b_offset, int R, int rank,
                               int d_in, int d_out, const __nv_bfloat16 *A_src,
                               const __nv_bfloat16 *B_src, int32_t *slot_rank_entry,
                               float *slot_scale_entry, float scale, uint32_t *slot_gen_entry,
                               uint32_t generation, cudaStream_t stream);

// Publish a slot's rank, scale and generation without touching its weights (clear).
cudaError_t launch_publish_slot(int32_t *slot_rank_entry, float *slot_scale_entry,
                                uint32_t *slot_gen_entry, int rank, float scale,
                                uint32_t generation, cudaStream_t stream);

// ---- fused base GEMM + LoRA (base_gemm.cu)

constexpr int kGemmRows = 256;   // rows of Y per GEMM tile (a pair of CTAs, 128 each)
// Per 256-row block: the number of distinct slots, then (slot, rank bucket) pairs.
constexpr int kBlockSlotsPitch = 1 + 2 * kGemmRows;

// Everything one launch of the fused base GEMM needs.  Passed by value.
struct GemmParams {
    CUtensorMap x_map;          // X [n_rows][d_in] bf16, box 64 x 128, 128-byte swizzle
    CUtensorMap w_map;          // W [d_out][d_in] bf16, box 64 x 128, 128-byte swizzle
    CUtensorMap b_map[4];       // the pool's B blocks per rank bucket 8..64: one box is one slot's
                                // 128-column chunk, [R/8][128][8] in shared memory
    int32_t b_col_div;          // the box's second coordinate is (first column) / b_col_div
    const int4 *row_info;       // [n_rows] {grouped position or -1, slot, scale bits, rank}
    const int32_t *block_slots; // [n_mblk][kBlockSlotsPitch]
    const float *H;             // [n_tokens][ldh] fp32, grouped order (the shrink's output)
    int64_t ldh;
    __nv_bfloat16 *Y;           // [n_rows][ldy] bf16, written for every row
    int64_t ldy;
    unsigned int *status;
    int32_t n_rows, d_in, d_out, n_mblk, n_nblk;
};

// row_info for every row (memset to -1, then the valid segments' rows); reports the
// segments' problems in p.status.
cudaError_t launch_row_map(const TileParams &p, int4 *row_info, cudaStream_t stream);
// The distinct slots of each 256-row block of rows.
cudaError_t launch_block_slots(const int4 *row_info, int n_rows, int32_t *block_slots, cudaStream_t stream);
// Tile width (256 or 512 columns of Y) for n_mblk 256-row blocks and d_out columns.
int choose_gemm_cols(int n_mblk, int d_out);
// Persistent GEMM over all (256-row, gn-column) tiles, one pair of CTAs per two SMs;
// p.n_nblk = ceil(d_out / gn).  With `pdl` it is launched with programmatic dependent
// launch after the kernel before it, whose results (H) it reads only after waiting.
cudaError_t launch_base_gemm(int gn, const GemmParams &p, cudaStream_t stream, bool pdl);
cudaError_t prepare_base_gemm();

}  // namespace mlora
