// lora_decode.cu -- segmented LoRA shrink / expand / fused apply for sm_100a,
// the decode-shaped family: many short segments, a few rows per adapter.
//
// The computation (page "Multi-LoRA Serving: adapter batching", section "What
// metadata a segmented kernel needs"): for each adapter segment g with slot a
// and each grouped position p of it, with t = token_indices[p],
//     H[p, :] = X[t, :] A_a^T                       (shrink, rank r)
//     Y[t, :] = bf16(Y[t, :] + s_g H[p, :] B_a^T)   (expand + scatter)
//
// Work decomposition.  A work tile is (segment, up to 16 consecutive grouped
// positions: the rows of one m16 MMA tile, so an adapter's slices are read once per 16
// rows of its segment).  A thread-block cluster of C CTAs owns a tile: CTA c covers its
// slice of d_in in the shrink (split-K) and its slice of d_out in the expand.
// Each CTA pushes its partial H tile (16 x R fp32) into every CTA of the cluster
// with st.async (distributed shared memory, completion counted on the receiver's
// mbarrier), and each sums the C partials in CTA order, so in the fused mode H
// never leaves the chip.  The grid holds as many
// clusters as can be resident at once; each loops over tiles.
//
// Split-K GEMV with register operands.  Decode tiles are too small for staged
// copies to pay off, so every thread loads its mma.sync operands straight from
// global memory with 128-bit loads:
//   * shrink: per 32-column block of d_in, thread (g, t) of a warp loads 8
//     consecutive bf16 of X rows g and g + 8 and of adapter row n at columns
//     8t..8t+7; the two k16 mma steps of the block consume them in that order.  The sum over k
//     does not care which columns share a step, as long as X and A agree.
//   * expand: four n8 mma tiles cover 32 output columns; the B row a lane feeds
//     is chosen so that thread (g, t) ends up owning columns 8t..8t+7 of row g,
//     (and row g + 8), so Y0 is read and Y written as one 16-byte vector per thread
//     and row.  The rank index inside each k16 step is permuted the same way for H
//     and B.
//
// Rank buckets.  A kernel is compiled for the pool's largest bucket RMAX and runs
// every tile with code specialised for its own slot's bucket R <= RMAX, so a
// rank-8 adapter moves and multiplies rank-8 data even in a rank-64 pool.
//
// Precision.  fp32 accumulation throughout.  For the expand, H is split into bf16
// hi + lo parts and both are multiplied on the tensor cores, so H enters the
// product with about 2^-17 relative error instead of bf16's 2^-9.
//
// Back-to-back launches.  For batches without long segments and about one wave of
// tiles, the kernel is launched with programmatic dependent launch: its CTAs may
// start while the previous kernel in the stream finishes, bring their first tile's
// adapter slices into L2 from a speculative read of the metadata (adapter weights
// only change through load_slot) and their rows' X and Y0 slices, and wait
// (griddepcontrol.wait) before reading the metadata, X or Y for real.  A stale
// guess costs bandwidth, never correctness.  In such launches a cluster with a
// second tile also prefetches that tile's adapter slices while it runs the first.
//
// Fused projections.  With FUSED, one launch applies several projections that share
// X and the metadata (q/k/v, gate/up), each with its own pool and output; a work
// item is (tile, projection), projection fastest, so a tile's X rows are read from
// HBM once.
//
// Invalid metadata never traps: bad segments and rows are skipped and flagged in
// the status word; every CTA of a cluster reaches the same decisions, so cluster
// barriers always match.  Its one wait on other CTAs (the partial-H exchange) is
// bounded: on expiry it flags a timeout and leaves the tile's rows alone.
#include <climits>
#include <mutex>
#include <type_traits>

#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace mlora {

namespace {

constexpr int kMaxWarps = 8;     // CTAs of 256 threads, or 128 (see launch_rmax)
// Grouped positions per work tile: 8 (rows g of the m16 MMA tile; rows 8..15 zero) or
// 16 (rows g and g + 8).  16-row tiles read each adapter slice once per 16 rows of a
// segment instead of 8 but need more registers and shared memory per CTA, so they are
// used only where segments are long and the rank small (block70b, 2048 rows over 128
// rank-16 adapters: 391.7 -> 361.9 us per step; with 8 or fewer rows per segment, or
// rank 64, they measured much slower).
constexpr int kMaxTM = 16;
constexpr int kMaxCluster = 8;

template <int RMAX, int NT, int TM = kTileRows>
struct DecodeCfg {
    static constexpr int kWarps = NT / 32;
    static constexpr int WPART_FLOATS = kWarps * TM * RMAX;   // per-warp partial H
    // partial H tiles pushed by the cluster's CTAs, [tile parity][source CTA][TM * R]
    static constexpr int RECV_FLOATS = 2 * kMaxCluster * TM * RMAX;
    static constexpr int HPITCH = RMAX + 4;
    static constexpr int HFULL_FLOATS = TM * HPITCH;          // full H (after the cluster sum)
    static constexpr int SMEM = 4 * (WPART_FLOATS + RECV_FLOATS + HFULL_FLOATS);
    static constexpr int MIN_BLOCKS = (RMAX <= 16 ? (TM == 16 ? 3 : 4) : 2) * (256 / NT);
};

// Per-R register operands: one k32 block of the shrink, one 32-column group of the
// expand.  Every warp keeps two of each in flight.
template <int R>
struct RankCfg {
    static constexpr int NT = R / 8;                  // n8 tiles of the shrink
    static constexpr int KS = R <= 8 ? 1 : R / 16;    // k steps of the expand
    // Issue the first expand group's loads before the shrink?  Measured: no gain on a
    // 4096 x 4096 decode batch, 5% slower on 8192-wide projections (the Y0 rows then
    // compete with the X rows the shrink waits for), so the expand loads follow it.
    static constexpr bool EARLY_EXPAND = false;
};

template <int R>
struct ShrinkOps {
    uint4 x, x8;                // X rows g and g + 8, columns 8t..8t+7 of the block
    uint4 a[RankCfg<R>::NT];    // adapter rows n*8+g, same columns
};

// Element types of the activation X and of the base output Y (the dtype boundary of
// a quantized base model): DT = 3 * XT + YT with XT 0 = bf16, 1 = FP8 e4m3 codes (times
// a per-tensor scale); YT 0 = bf16, 1 = fp16, 2 = fp32.  DT 0 is the all-bf16 path.
__host__ __device__ constexpr int dt_x(int dt) { return dt / 3; }
__host__ __device__ constexpr int dt_y(int dt) { return dt % 3; }
__host__ __device__ constexpr int x_bytes(int dt) { return dt_x(dt) == 1 ? 1 : 2; }
__host__ __device__ constexpr int y_bytes(int dt) { return dt_y(dt) == 2 ? 4 : 2; }

template <int R, int YT = 0>
struct ExpandOps {
    uint2 b[4][RankCfg<R>::KS];  // B rows of the four n8 tiles, this lane's ranks
    uint4 y[2];                  // Y0 rows g, g + 8, columns 8t..8t+7 of the group (bf16 or fp16)
};

template <int R>
struct ExpandOps<R, 2> {
    uint2 b[4][RankCfg<R>::KS];
    uint4 y[2], y2[2];           // fp32 Y0 rows g, g + 8: columns 8t..8t+3, 8t+4..8t+7
};

// Segments whose first-tile indices a CTA keeps after its first metadata scan, so that
// its later tiles are found by a binary search instead of another scan.  Only the
// 128-thread kernels keep the table: they run the batches of several waves of tiles;
// the 256-thread ones run about one wave, where a cluster rarely has a second tile.
// Of those, the fused and rank > 16 ones (measured): in the single-projection rank-16
// kernel the table's registers cost more than the scans it saves.
constexpr int kSegTable = 256;
template <bool KEEP>
struct SegTable {
    int first[kSegTable];   // first tile of each segment (the next segment's, if it has none)
};
template <>
struct SegTable<false> {
    int first[1];
};

struct SharedCtl {
    uint64_t hbar[2];   // partial H tiles of the cluster landed (one per tile parity)
    int fail;           // a partial-H wait ran out: no later tile of this launch is trusted
    int scan[kMaxWarps];
    int rows[kMaxTM];   // original row of each tile position, -1 = absent or invalid
    int tile[5];        // segment, first position, end position, slot, rank from metadata
    int stale;          // the batch was built for an earlier generation of the slot
    float seg_scale;
    int slot_rank;
    float slot_scale;
};

struct Tile {
    int seg, p0, nvalid, slot;
};

__device__ __forceinline__ void report(const TileParams &p, unsigned flag)
{
    atomicOr(p.status, flag);
}

__device__ __forceinline__ void report(const ProjView &v, unsigned flag)
{
    atomicOr(v.status, flag);
}

__device__ __forceinline__ uint4 ldg_nc(const void *p)
{
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

__device__ __forceinline__ uint2 ldg_nc2(const void *p)
{
    return __ldg(reinterpret_cast<const uint2 *>(p));
}

// L2 prefetch, by one thread, of this CTA's slices of an adapter's A and B blocks
// (slot, rank bucket R): every address stays inside the pool.
template <int MODE>
__device__ __forceinline__ void prefetch_slices_one(const TileParams &p, const ProjView &v, int slot, int R,
                                                    uint32_t crank)
{
    constexpr uint32_t kChunk = 32768;
    const char *slotA = reinterpret_cast<const char *>(v.pool + (int64_t)slot * v.slot_stride);
    if (MODE != MODE_EXPAND) {
        const int k0 = min(p.d_in, (int)crank * p.k_slice);
        const int k1 = min(p.d_in, k0 + p.k_slice);
        const int64_t beg = (int64_t)k0 * R * 2, len = (int64_t)(k1 - k0) * R * 2;
        for (int64_t off = 0; off < len; off += kChunk)
            prefetch_l2_bulk(slotA + beg + off, (uint32_t)(len - off < kChunk ? len - off : kChunk));
    }
    if (MODE != MODE_SHRINK) {
        const int n0 = min(v.d_out, (int)crank * v.n_slice);
        const int n1 = min(v.d_out, n0 + v.n_slice);
        const int64_t len = (int64_t)(n1 - n0) * 16;
        for (int j = 0; j < R / 8; ++j) {
            const char *b = slotA + (v.b_offset + ((int64_t)j * v.d_out + n0) * 8) * 2;
            for (int64_t off = 0; off < len; off += kChunk)
                prefetch_l2_bulk(b + off, (uint32_t)(len - off < kChunk ? len - off : kChunk));
        }
    }
}

// Block-wide scan of per-segment tile counts.  Returns the number of tiles; if
// tile `want` exists, its segment and first position are left in ctl.tile.
// SPEC: a speculative pass made before the grids this launch depends on have
// finished (the metadata may still change): relaxed loads, nothing reported.
// slot_gen: generations of the pool the tile will read (ctl.stale).
// want2 (-1: none): the cluster's next tile, of projection v2.  In early launches
// (batches of about one wave of tiles) the thread that finds it prefetches this CTA's
// slices of that tile's adapter into L2, so that they travel while the current tile
// runs.  Batches of several waves skip it: there the prefetches thrashed L2
// (measured 11% slower on 2048 decode rows of 8192-wide projections).
// first (may be null): filled with each segment's first tile (see find_tile).
template <bool SPEC, int NT, int MODE, int RMAX, int TM>
__device__ int scan_tiles(const TileParams &p, const uint32_t *slot_gen, int want, int want2,
                          const ProjView &v2, SharedCtl &ctl, bool reporter, int *first = nullptr)
{
    constexpr int kThreads = NT, kWarps = NT / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) ctl.tile[0] = -1;
    __syncthreads();
    int running = 0;
    for (int base = 0; base < p.n_segments; base += kThreads) {
        const int g = base + tid;
        int cnt = 0, p0 = 0, p1 = 0, a = -1, rk = -1;
        float sc = 0.f;
        if (g < p.n_segments) {
            if constexpr (SPEC) {
                a = ld_relaxed_s32(p.slots + g);
                p0 = ld_relaxed_s32(p.offsets + g);
                p1 = ld_relaxed_s32(p.offsets + g + 1);
                if (p.ranks) rk = ld_relaxed_s32(p.ranks + g);
                reporter = false;
            } else {
                a = p.slots[g];
                p0 = p.offsets[g];
                p1 = p.offsets[g + 1];
                if (p.ranks) rk = p.ranks[g];
                if (p.scales) sc = p.scales[g];
            }
            if (a != -1) {
                if (a < -1 || a >= p.n_slots) {
                    if (reporter) report(p, kFlagBadSlot);
                } else if (p0 < 0 || p1 < p0 || p1 > p.n_tokens) {
                    if (reporter) report(p, kFlagBadOffsets);
                } else if (!long_segment(p, p0, p1)) {
                    cnt = (p1 - p0 + TM - 1) / TM;
                }
            }
        }
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) ctl.scan[warp] = incl;
        __syncthreads();
        int before = 0, total = 0;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const int v = ctl.scan[w];
            before += (w < warp) ? v : 0;
            total += v;
        }
        incl += before;
        const int lo = running + incl - cnt;
        if (!SPEC && first != nullptr && g < p.n_segments && g < kSegTable) first[g] = lo;
        if (cnt > 0 && want >= lo && want < running + incl) {
            ctl.tile[0] = g;
            ctl.tile[1] = p0 + (want - lo) * TM;
            ctl.tile[2] = p1;
            ctl.tile[3] = a;
            ctl.tile[4] = rk;
            ctl.seg_scale = sc;
            if constexpr (!SPEC) ctl.stale = p.generations && slot_gen[a] != p.generations[g];
        }
        if constexpr (RMAX <= 16) {   // (larger pools: more register spills than it saved)
            if (p.early && cnt > 0 && want2 >= lo && want2 < running + incl && p.ranks != nullptr) {
                const int R2 = rank_bucket(rk);
                if (R2 > 0 && R2 <= RMAX) prefetch_slices_one<MODE>(p, v2, a, R2, cluster_rank());
            }
        }
        running += total;
        __syncthreads();   // ctl.scan is rewritten by the next chunk
    }
    return running;
}

// Tile `want` (< the launch's tile count) after a full scan_tiles of the same
// metadata by this CTA (at most kSegTable segments): its segment is the last one whose
// first tile is <= want (segments without tiles of this kernel share the next one's
// first tile, so the last such index is a segment with tiles), found by binary search
// in first; the rest as scan_tiles leaves it in ctl.  want2 (-1: none, else a
// valid tile) as in scan_tiles.
template <int MODE, int RMAX, int TM>
__device__ void find_tile(const TileParams &p, const uint32_t *slot_gen, int want, int want2, const ProjView &v2,
                          SharedCtl &ctl, const int *first)
{
    const int tid = threadIdx.x;
    auto segment_of = [&](int t) {
        int lo = 0, hi = p.n_segments - 1;   // ctl.first[lo] <= t
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (first[mid] <= t) lo = mid;
            else hi = mid - 1;
        }
        return lo;
    };
    if (tid == 0) {
        const int g = segment_of(want);
        const int a = p.slots[g];
        ctl.tile[0] = g;
        ctl.tile[1] = p.offsets[g] + (want - first[g]) * TM;
        ctl.tile[2] = p.offsets[g + 1];
        ctl.tile[3] = a;
        ctl.tile[4] = p.ranks ? p.ranks[g] : -1;
        ctl.seg_scale = p.scales ? p.scales[g] : 0.f;
        ctl.stale = p.generations && slot_gen[a] != p.generations[g];
    }
    if constexpr (RMAX <= 16) {   // as in scan_tiles
        if (tid == 32 && p.early && want2 >= 0 && p.ranks != nullptr) {
            const int g2 = segment_of(want2);
            const int R2 = rank_bucket(p.ranks[g2]);
            const int a2 = p.slots[g2];
            if (R2 > 0 && R2 <= RMAX && a2 >= 0 && a2 < p.n_slots) prefetch_slices_one<MODE>(p, v2, a2, R2, cluster_rank());
        }
    }
    __syncthreads();
}

// Geometry of this CTA's part of a tile.
struct Slices {
    int k_begin, k_end, nblk;   // d_in slice, 32-column blocks
    int n_begin, n_end, ngrp;   // d_out slice, 32-column groups
};

template <int R>
__device__ __forceinline__ void load_a(ShrinkOps<R> &o, const __nv_bfloat16 *slotA, const Slices &sl,
                                       int blk, int g, int t)
{
    const int k = sl.k_begin + blk * 32 + 8 * t;   // this thread's 8 columns
    const bool kin = blk < sl.nblk && k < sl.k_end;
#pragma unroll
    for (int n = 0; n < RankCfg<R>::NT; ++n)
        o.a[n] = kin ? ldg_nc(slotA + ((int64_t)(k / 8) * R + n * 8 + g) * 8) : make_uint4(0, 0, 0, 0);
}

// Two FP8 e4m3 codes (low byte first) as the bf16x2 of their values: exact, since every
// e4m3 value is a bf16 value.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two)
{
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xffffu), __NV_E4M3);
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h));
    return pack_bf16x2(f.x, f.y);
}

// X's element type: bf16 values or FP8 e4m3 codes (bytes).
template <int XT>
using XElem = typename std::conditional<XT == 1, const uint8_t, const __nv_bfloat16>::type;
// Y's element type: bf16, fp16 or fp32.
template <int YT>
using YElem =
    typename std::conditional<YT == 2, float, typename std::conditional<YT == 1, __half, __nv_bfloat16>::type>::type;

template <int XT>
__device__ __forceinline__ uint4 load_x_row(XElem<XT> *xrow, bool in, int k)
{
    if constexpr (XT == 0) {
        return in ? ldg_nc(xrow + k) : make_uint4(0, 0, 0, 0);
    } else {
        // eight e4m3 codes, widened to bf16 (the per-tensor scale is applied to H)
        const uint2 c = in ? __ldg(reinterpret_cast<const uint2 *>(xrow + k)) : make_uint2(0u, 0u);
        return make_uint4(e4m3x2_to_bf16x2(c.x), e4m3x2_to_bf16x2(c.x >> 16), e4m3x2_to_bf16x2(c.y),
                          e4m3x2_to_bf16x2(c.y >> 16));
    }
}

// X rows g (xrow) and g + 8 (xrow8) of the tile, this thread's 8 columns of the block.
template <int R, int XT, int TM>
__device__ __forceinline__ void load_x(ShrinkOps<R> &o, XElem<XT> *xrow, bool row_ok, XElem<XT> *xrow8,
                                       bool row_ok8, const Slices &sl, int blk, int t)
{
    const int k = sl.k_begin + blk * 32 + 8 * t;
    const bool kin = blk < sl.nblk && k < sl.k_end;
    o.x = load_x_row<XT>(xrow, row_ok && kin, k);
    if constexpr (TM == 16) o.x8 = load_x_row<XT>(xrow8, row_ok8 && kin, k);
}

template <int R, int TM>
__device__ __forceinline__ void mma_shrink(float (&acc)[RankCfg<R>::NT][4], const ShrinkOps<R> &o)
{
#pragma unroll
    for (int n = 0; n < RankCfg<R>::NT; ++n) {
        if constexpr (TM == 16) {
            mma_16816(acc[n], o.x.x, o.x8.x, o.x.y, o.x8.y, o.a[n].x, o.a[n].y);
            mma_16816(acc[n], o.x.z, o.x8.z, o.x.w, o.x8.w, o.a[n].z, o.a[n].w);
        } else {   // rows g + 8 of an 8-row tile are zero
            mma_16816(acc[n], o.x.x, 0u, o.x.y, 0u, o.a[n].x, o.a[n].y);
            mma_16816(acc[n], o.x.z, 0u, o.x.w, 0u, o.a[n].z, o.a[n].w);
        }
    }
}

// B row fed by lane (g, t) in n8 tile i of a group: base + 8 (g / 2) + (g % 2) + 2 i, so
// that thread (g, t) accumulates columns base + 8t .. base + 8t + 7 of row g.
template <int R, int YT>
__device__ __forceinline__ void load_b(ExpandOps<R, YT> &o, const __nv_bfloat16 *slotB, int d_out,
                                       const Slices &sl, int grp, int g, int t)
{
    const int base = sl.n_begin + grp * 32;
    const bool bin = grp < sl.ngrp && base + 8 * (g >> 1) < sl.n_end;
    const int brow = base + 8 * (g >> 1) + (g & 1);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int s = 0; s < RankCfg<R>::KS; ++s) {
            if constexpr (R == 8) {
                const uint32_t v =
                    bin ? __ldg(reinterpret_cast<const uint32_t *>(slotB + (int64_t)(brow + 2 * i) * 8 + 2 * t))
                        : 0u;
                o.b[i][s] = make_uint2(v, 0u);
            } else {
                o.b[i][s] = bin ? ldg_nc2(slotB + ((int64_t)(2 * s + (t >> 1)) * d_out + brow + 2 * i) * 8 +
                                          (t & 1) * 4)
                                : make_uint2(0u, 0u);
            }
        }
}

// Y0 rows g (yrow) and g + 8 (yrow8, 16-row tiles), this thread's 8 columns of the group.
template <int R, int YT, int TM>
__device__ __forceinline__ void load_y(ExpandOps<R, YT> &o, const YElem<YT> *yrow, bool row_ok,
                                       const YElem<YT> *yrow8, bool row_ok8, const Slices &sl, int grp, int t)
{
    const int c = sl.n_begin + grp * 32 + 8 * t;
    const bool cin = grp < sl.ngrp && c < sl.n_end;
#pragma unroll
    for (int h = 0; h < TM / 8; ++h) {
        const YElem<YT> *row = h ? yrow8 : yrow;
        const bool in = cin && (h ? row_ok8 : row_ok);
        if constexpr (YT == 2) {   // eight fp32
            const uint4 *src = reinterpret_cast<const uint4 *>(row + c);
            o.y[h] = in ? src[0] : make_uint4(0, 0, 0, 0);
            o.y2[h] = in ? src[1] : make_uint4(0, 0, 0, 0);
        } else {                   // eight bf16 or fp16
            o.y[h] = in ? *reinterpret_cast<const uint4 *>(row + c) : make_uint4(0, 0, 0, 0);
        }
    }
}

// y = y0 + s (H B^T), rounded once to Y's type, for one group; thread (g, t) stores rows
// g and g + 8, columns 8t..8t+7.  ah / al: H rows g and g + 8 ([.][0..1] row g, [.][2..3]
// row g + 8, as the m16 A fragment wants them).
template <int R, int YT, int TM>
__device__ __forceinline__ void mma_expand_store(const ExpandOps<R, YT> &o,
                                                 const uint32_t (&ah)[RankCfg<R>::KS][TM / 4],
                                                 const uint32_t (&al)[RankCfg<R>::KS][TM / 4], float scale, YElem<YT> *yrow,
                                                 bool store, YElem<YT> *yrow8, bool store8, const Slices &sl, int grp,
                                                 int t)
{
    float d[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        d[i][0] = d[i][1] = d[i][2] = d[i][3] = 0.f;
#pragma unroll
        for (int s = 0; s < RankCfg<R>::KS; ++s) {
            if constexpr (TM == 16) {
                if constexpr (R == 8) {
                    mma_1688(d[i], ah[0][0], ah[0][2], o.b[i][0].x);
                    mma_1688(d[i], al[0][0], al[0][2], o.b[i][0].x);
                } else {
                    mma_16816(d[i], ah[s][0], ah[s][2], ah[s][1], ah[s][3], o.b[i][s].x, o.b[i][s].y);
                    mma_16816(d[i], al[s][0], al[s][2], al[s][1], al[s][3], o.b[i][s].x, o.b[i][s].y);
                }
            } else {   // rows g + 8 of an 8-row tile are zero
                if constexpr (R == 8) {
                    mma_1688(d[i], ah[0][0], 0u, o.b[i][0].x);
                    mma_1688(d[i], al[0][0], 0u, o.b[i][0].x);
                } else {
                    mma_16816(d[i], ah[s][0], 0u, ah[s][1], 0u, o.b[i][s].x, o.b[i][s].y);
                    mma_16816(d[i], al[s][0], 0u, al[s][1], 0u, o.b[i][s].x, o.b[i][s].y);
                }
            }
        }
    }
    const int c = sl.n_begin + grp * 32 + 8 * t;
    if (grp >= sl.ngrp || c >= sl.n_end) return;
#pragma unroll
    for (int h = 0; h < TM / 8; ++h) {
        if (!(h ? store8 : store)) continue;
        YElem<YT> *row = h ? yrow8 : yrow;
        if constexpr (YT == 2) {
            const float4 a = *reinterpret_cast<const float4 *>(&o.y[h]);
            const float4 b = *reinterpret_cast<const float4 *>(&o.y2[h]);
            float4 *dst = reinterpret_cast<float4 *>(row + c);
            dst[0] = make_float4(fmaf(scale, d[0][2 * h], a.x), fmaf(scale, d[0][2 * h + 1], a.y),
                                 fmaf(scale, d[1][2 * h], a.z), fmaf(scale, d[1][2 * h + 1], a.w));
            dst[1] = make_float4(fmaf(scale, d[2][2 * h], b.x), fmaf(scale, d[2][2 * h + 1], b.y),
                                 fmaf(scale, d[3][2 * h], b.z), fmaf(scale, d[3][2 * h + 1], b.w));
        } else {
            uint4 out;
            uint32_t *w = reinterpret_cast<uint32_t *>(&out);
            if constexpr (YT == 0) {
                const __nv_bfloat162 *y0 = reinterpret_cast<const __nv_bfloat162 *>(&o.y[h]);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = __bfloat1622float2(y0[i]);
                    w[i] = pack_bf16x2(fmaf(scale, d[i][2 * h], f.x), fmaf(scale, d[i][2 * h + 1], f.y));
                }
            } else {
                const __half2 *y0 = reinterpret_cast<const __half2 *>(&o.y[h]);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = __half22float2(y0[i]);
                    const __half2 hv = __floats2half2_rn(fmaf(scale, d[i][2 * h], f.x), fmaf(scale, d[i][2 * h + 1], f.y));
                    w[i] = *reinterpret_cast<const uint32_t *>(&hv);
                }
            }
            *reinterpret_cast<uint4 *>(row + c) = out;
        }
    }
}

// One tile, specialised for rank bucket R.  Loads are issued as early as their
// addresses are known: adapter blocks right away, rows once their indices land,
// the expand's operands before the cluster reduction.
// Speculative L2 prefetch of this CTA's share of its first tile's adapter (A slice
// and B slice), made before the launch's dependencies have finished: adapter
// weights do not change between loads, so their fetch overlaps the end of the
// previous kernel.  The metadata read here may be stale; a wrong guess only costs
// bandwidth (every address stays inside the pool), never correctness, since the
// tile's real loads come after griddep_wait.
// L2 prefetch of this CTA's slices of one tile's adapter (slot, rank bucket R) and
// of the line of token_indices at its first position: every address is inside the
// pool or the metadata whatever the values, so the caller may pass a guess.
template <int MODE>
__device__ void prefetch_slices(const TileParams &p, const ProjView &v, int slot, int R, int p0,
                                uint32_t crank)
{
    const int tid = threadIdx.x;
    if (tid == 32 && p.token_indices != nullptr && p0 >= 0 && p0 < p.n_tokens)
        prefetch_l2_line(p.token_indices + p0);
    const char *slotA = reinterpret_cast<const char *>(v.pool + (int64_t)slot * v.slot_stride);
    constexpr uint32_t kChunk = 16384;
    if (MODE != MODE_EXPAND && tid < 8) {
        // A block [d_in/8][R][8]: the slice [k_begin, k_end) is one contiguous run
        const int k0 = min(p.d_in, (int)crank * p.k_slice);
        const int k1 = min(p.d_in, k0 + p.k_slice);
        const int64_t beg = (int64_t)k0 * R * 2, len = (int64_t)(k1 - k0) * R * 2;
        for (int64_t off = (int64_t)tid * kChunk; off < len; off += 8 * kChunk)
            prefetch_l2_bulk(slotA + beg + off, (uint32_t)(len - off < kChunk ? len - off : kChunk));
    }
    if (MODE != MODE_SHRINK && tid >= 64 && tid < 64 + R / 8) {
        // B block [R/8][d_out][8]: rows [n_begin, n_end) of rank group j, contiguous
        const int j = tid - 64;
        const int n0 = min(v.d_out, (int)crank * v.n_slice);
        const int n1 = min(v.d_out, n0 + v.n_slice);
        const char *b = slotA + (v.b_offset + ((int64_t)j * v.d_out + n0) * 8) * 2;
        const int64_t len = (int64_t)(n1 - n0) * 16;
        for (int64_t off = 0; off < len; off += kChunk)
            prefetch_l2_bulk(b + off, (uint32_t)(len - off < kChunk ? len - off : kChunk));
    }
}

template <int RMAX, int MODE, int NT, int DT, int TM>
__device__ void prefetch_first_tile(const TileParams &p, const ProjView &v, int want, SharedCtl &ctl,
                                    uint32_t crank)
{
    if (want >= scan_tiles<true, NT, MODE, RMAX, TM>(p, v.slot_gen, want, -1, v, ctl, false)) return;
    const int tid = threadIdx.x;
    const int slot = ctl.tile[3];
    if (slot < 0 || slot >= p.n_slots) return;
    int R = rank_bucket(ctl.tile[4]);
    if (p.ranks == nullptr || R == 0 || R > RMAX) R = rank_bucket(ld_relaxed_s32(v.slot_rank + slot));
    if (R == 0 || R > RMAX) return;
    const int p0 = ctl.tile[1];
    prefetch_slices<MODE>(p, v, slot, R, p0, crank);
    // the tile's rows from a speculative read of token_indices (checked against n_rows,
    // so a stale guess still stays inside X and Y): this CTA's slices of their X and
    // Y0 rows.  L2 is the point of coherence, so lines the previous kernel is still
    // writing are never served stale.
    if (tid >= 96 && tid < 96 + TM) {
        const int pos = p0 + (tid - 96);
        if (pos >= 0 && pos < ctl.tile[2] && pos < p.n_tokens) {
            const int row = p.token_indices ? ld_relaxed_s32(p.token_indices + pos) : pos;
            if (row >= 0 && row < p.n_rows) {
                if (MODE != MODE_EXPAND) {
                    const int k0 = min(p.d_in, (int)crank * p.k_slice);
                    const int k1 = min(p.d_in, k0 + p.k_slice);
                    using XE = typename std::conditional<dt_x(DT) == 1, const uint8_t, const __nv_bfloat16>::type;
                    if (k1 > k0)
                        prefetch_l2_bulk(reinterpret_cast<XE *>(p.X) + (int64_t)row * p.ldx + k0,
                                         (uint32_t)(k1 - k0) * x_bytes(DT));
                }
                if (MODE != MODE_SHRINK) {
                    const int n0 = min(v.d_out, (int)crank * v.n_slice);
                    const int n1 = min(v.d_out, n0 + v.n_slice);
                    using YE = typename std::conditional<dt_y(DT) == 2, const float, const __nv_bfloat16>::type;
                    if (n1 > n0)
                        prefetch_l2_bulk(reinterpret_cast<YE *>(v.Y) + (int64_t)row * v.ldy + n0,
                                         (uint32_t)(n1 - n0) * y_bytes(DT));
                }
            }
        }
    }
}

template <int RMAX, int MODE, int R, int NT, int DT, int TM>
__device__ void run_tile(const TileParams &p, const ProjView &v, const Tile &tl, int r_meta,
                         float seg_scale, SharedCtl &ctl, float *smem_f, uint32_t crank,
                         uint32_t csize, uint32_t nt)
{
    constexpr int kThreads = NT, kWarps = NT / 32;
    using RC = RankCfg<R>;
    using DC = DecodeCfg<RMAX, NT, TM>;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    float *wpart = smem_f;
    float *recv = wpart + DC::WPART_FLOATS + (nt & 1) * (kMaxCluster * TM * RMAX);
    float *hfull = wpart + DC::WPART_FLOATS + DC::RECV_FLOATS;
    const __nv_bfloat16 *slotA = v.pool + (int64_t)tl.slot * v.slot_stride;
    const __nv_bfloat16 *slotB = slotA + v.b_offset;

    Slices sl;
    sl.k_begin = min(p.d_in, (int)crank * p.k_slice);
    sl.k_end = min(p.d_in, sl.k_begin + p.k_slice);
    sl.nblk = (MODE == MODE_EXPAND) ? 0 : (sl.k_end - sl.k_begin + 31) / 32;
    sl.n_begin = min(v.d_out, (int)crank * v.n_slice);
    sl.n_end = min(v.d_out, sl.n_begin + v.n_slice);
    sl.ngrp = (MODE == MODE_SHRINK) ? 0 : (sl.n_end - sl.n_begin + 31) / 32;
    // blocks w, w + 8, ... and groups w, w + 8, ... of this warp, as local indices 0, 1, ...
    const int nb = sl.nblk > warp ? (sl.nblk - warp + kWarps - 1) / kWarps : 0;
    const int ng = sl.ngrp > warp ? (sl.ngrp - warp + kWarps - 1) / kWarps : 0;

    // ---- requests that need only the segment's slot
    int row_g = -1, row_g8 = -1;   // original rows of tile positions g and g + 8
    if (g < tl.nvalid) row_g = p.token_indices ? __ldg(p.token_indices + tl.p0 + g) : tl.p0 + g;
    if (TM == 16 && g + 8 < tl.nvalid)
        row_g8 = p.token_indices ? __ldg(p.token_indices + tl.p0 + g + 8) : tl.p0 + g + 8;
    int srank = 0;
    float sscale = 0.f;
    if (tid == 0) {
        srank = v.slot_rank[tl.slot];
        sscale = v.slot_scale[tl.slot];
        if (ctl.stale) srank = -1;   // rank -1 marks a stale generation
    }
    constexpr int XT = dt_x(DT), YT = dt_y(DT);
    ShrinkOps<R> s0, s1;
    ExpandOps<R, YT> e0, e1;
    if constexpr (MODE != MODE_EXPAND) {
        load_a<R>(s0, slotA, sl, warp, g, t);
        load_a<R>(s1, slotA, sl, warp + kWarps, g, t);
    }
    if constexpr (MODE != MODE_SHRINK && RC::EARLY_EXPAND) load_b<R, YT>(e0, slotB, v.d_out, sl, warp, g, t);

    // ---- requests that need the row
    if (g < tl.nvalid && (row_g < 0 || row_g >= p.n_rows)) {
        if (crank == 0 && warp == 0 && t == 0) report(v, kFlagBadRow);
        row_g = -1;
    }
    if (TM == 16 && g + 8 < tl.nvalid && (row_g8 < 0 || row_g8 >= p.n_rows)) {
        if (crank == 0 && warp == 0 && t == 0) report(v, kFlagBadRow);
        row_g8 = -1;
    }
    const bool row_ok = row_g >= 0, row_ok8 = row_g8 >= 0;
    // row pointers in X's and Y's element types
    XElem<XT> *xrow = reinterpret_cast<XElem<XT> *>(p.X) + (int64_t)(row_ok ? row_g : 0) * p.ldx;
    YElem<YT> *yrow = reinterpret_cast<YElem<YT> *>(v.Y) + (int64_t)(row_ok ? row_g : 0) * v.ldy;
    XElem<XT> *xrow8 = reinterpret_cast<XElem<XT> *>(p.X) + (int64_t)(row_ok8 ? row_g8 : 0) * p.ldx;
    YElem<YT> *yrow8 = reinterpret_cast<YElem<YT> *>(v.Y) + (int64_t)(row_ok8 ? row_g8 : 0) * v.ldy;
    if constexpr (MODE != MODE_EXPAND) {
        load_x<R, XT, TM>(s0, xrow, row_ok, xrow8, row_ok8, sl, warp, t);
        load_x<R, XT, TM>(s1, xrow, row_ok, xrow8, row_ok8, sl, warp + kWarps, t);
    }
    if constexpr (MODE != MODE_SHRINK && RC::EARLY_EXPAND)
        load_y<R, YT, TM>(e0, yrow, row_ok, yrow8, row_ok8, sl, warp, t);

    // ---- shrink: this CTA's d_in slice, two blocks in flight per warp
    if constexpr (MODE != MODE_EXPAND) {
        float acc[RC::NT][4];
#pragma unroll
        for (int n = 0; n < RC::NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
        for (int i = 0; i < nb; i += 2) {
            mma_shrink<R, TM>(acc, s0);
            if (i + 2 < nb) {
                const int b = warp + (i + 2) * kWarps;
                load_a<R>(s0, slotA, sl, b, g, t);
                load_x<R, XT, TM>(s0, xrow, row_ok, xrow8, row_ok8, sl, b, t);
            }
            if (i + 1 < nb) {
                mma_shrink<R, TM>(acc, s1);
                if (i + 3 < nb) {
                    const int b = warp + (i + 3) * kWarps;
                    load_a<R>(s1, slotA, sl, b, g, t);
                    load_x<R, XT, TM>(s1, xrow, row_ok, xrow8, row_ok8, sl, b, t);
                }
            }
        }
        if constexpr (MODE != MODE_SHRINK) {
            // the expand's first groups travel while the cluster sums H
            if constexpr (!RC::EARLY_EXPAND) {
                load_b<R, YT>(e0, slotB, v.d_out, sl, warp, g, t);
                load_y<R, YT, TM>(e0, yrow, row_ok, yrow8, row_ok8, sl, warp, t);
            }
            load_b<R, YT>(e1, slotB, v.d_out, sl, warp + kWarps, g, t);
            load_y<R, YT, TM>(e1, yrow, row_ok, yrow8, row_ok8, sl, warp + kWarps, t);
        }
#pragma unroll
        for (int n = 0; n < RC::NT; ++n) {
            wpart[(warp * TM + g) * R + n * 8 + 2 * t] = acc[n][0];
            wpart[(warp * TM + g) * R + n * 8 + 2 * t + 1] = acc[n][1];
            if constexpr (TM == 16) {
                wpart[(warp * TM + g + 8) * R + n * 8 + 2 * t] = acc[n][2];
                wpart[(warp * TM + g + 8) * R + n * 8 + 2 * t + 1] = acc[n][3];
            }
        }
    } else {
        load_b<R, YT>(e1, slotB, v.d_out, sl, warp + kWarps, g, t);
        load_y<R, YT, TM>(e1, yrow, row_ok, yrow8, row_ok8, sl, warp + kWarps, t);
        if constexpr (!RC::EARLY_EXPAND) {
            load_b<R, YT>(e0, slotB, v.d_out, sl, warp, g, t);
            load_y<R, YT, TM>(e0, yrow, row_ok, yrow8, row_ok8, sl, warp, t);
        }
    }
    if (tid == 0) {
        ctl.slot_rank = srank;
        ctl.slot_scale = sscale;
    }
    if (warp == 0 && t == 0) {
        ctl.rows[g] = row_g;
        if constexpr (TM == 16) ctl.rows[g + 8] = row_g8;
    }
    __syncthreads();
    const int r = ctl.slot_rank;
    const bool ok = r > 0 && (p.ranks == nullptr || r_meta == r) && rank_bucket(r) == R;
    if (tid == 0 && crank == 0 && !ok)
        report(v, r < 0 ? kFlagStaleSlot : r == 0 ? kFlagSlotEmpty : kFlagBadRank);
    const int rank = ok ? r : 0;   // a rejected tile reads and writes no H
    const float scale = p.scales ? seg_scale : ctl.slot_scale;
    bool h_ok = true;

    if constexpr (MODE != MODE_EXPAND) {
        // This CTA's partial tile (summed over its warps) is pushed into every CTA of
        // the cluster with st.async, which counts its bytes on the receiver's mbarrier:
        // no cluster barrier with release semantics (which would first wait for the
        // expand operands still in flight) stands between the shrink and the expand.
        uint64_t *bar = &ctl.hbar[nt & 1];
        if (tid == 0) mbar_arrive_expect_tx(bar, csize * TM * R * 4);
        const uint32_t slot_s = smem_addr(recv + crank * TM * R);
        const uint32_t bar_s = smem_addr(bar);
        for (int e4 = tid; e4 < TM * R / 4; e4 += kThreads) {
            float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                const float4 v = *reinterpret_cast<const float4 *>(wpart + w * TM * R + 4 * e4);
                sum.x += v.x;
                sum.y += v.y;
                sum.z += v.z;
                sum.w += v.w;
            }
            for (uint32_t c = 0; c < csize; ++c)
                st_async_f32x4(map_to_rank(slot_s + 16u * e4, c), sum, map_to_rank(bar_s, c));
        }
        // the cluster's partials, summed in CTA order.  After a wait has run out, the
        // barriers' phases no longer match the tiles (late bytes may complete a later
        // phase), so no later tile of this launch writes anything either (ctl.fail).
        const bool landed = mbar_wait_bounded(bar, (nt >> 1) & 1u, 1000000000ull);
        if (!landed) {
            ctl.fail = 1;
            report(v, kFlagTimeout);
        }
        for (int e = tid; e < TM * R; e += kThreads) {
            const int i = e / R, j = e % R;
            if (MODE == MODE_SHRINK &&
                ((uint32_t)i % csize != crank || i >= tl.nvalid || j >= rank || ctl.rows[i] < 0 || !landed ||
                 ctl.fail))
                continue;
            float v[kMaxCluster];
#pragma unroll
            for (int c = 0; c < kMaxCluster; ++c) v[c] = (c < (int)csize) ? recv[c * TM * R + e] : 0.f;
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < kMaxCluster; ++c) sum += v[c];
            if (!landed) sum = 0.f;   // (the tile's rows are then left alone)
            if constexpr (XT == 1) sum *= p.x_scale;   // the FP8 codes' per-tensor scale
            if constexpr (MODE == MODE_APPLY) {
                hfull[i * DC::HPITCH + j] = sum;
            } else {
                p.H[(int64_t)(tl.p0 + i) * p.ldh + j] = sum;
            }
        }
        h_ok = landed;
        cluster_arrive_relaxed();   // paired with the wait at the end of the tile
    } else {
        for (int e = tid; e < TM * R; e += kThreads) {
            const int i = e / R, j = e % R;
            float v = 0.f;
            if (i < tl.nvalid && j < rank) v = p.H[(int64_t)(tl.p0 + i) * p.ldh + j];
            hfull[i * DC::HPITCH + j] = v;
        }
    }

    // ---- expand: this CTA's d_out slice, two groups in flight per warp
    if constexpr (MODE != MODE_SHRINK) {
        __syncthreads();
        // H rows g ([.][0..1]) and g + 8 ([.][2..3]) as bf16 hi + lo fragments; step s
        // covers rank 16s + 4t .. 16s + 4t + 3 (rank bucket 8: 2t, 2t + 1)
        uint32_t ah[RC::KS][TM / 4], al[RC::KS][TM / 4];
#pragma unroll
        for (int s = 0; s < RC::KS; ++s) {
#pragma unroll
            for (int q = 0; q < TM / 4; ++q) {
                const int col = (R == 8) ? 2 * t : 16 * s + 4 * t + 2 * (q & 1);
                const int hr = g + 8 * (q >> 1);
                float h0, l0, h1, l1;
                split_bf16(hfull[hr * DC::HPITCH + col], h0, l0);
                split_bf16(hfull[hr * DC::HPITCH + col + 1], h1, l1);
                ah[s][q] = pack_bf16x2(h0, h1);
                al[s][q] = pack_bf16x2(l0, l1);
            }
        }
        const bool live = ok && h_ok && (MODE == MODE_EXPAND || ctl.fail == 0);
        const bool store = live && row_ok, store8 = live && row_ok8;
        for (int i = 0; i < ng; i += 2) {
            mma_expand_store<R, YT, TM>(e0, ah, al, scale, yrow, store, yrow8, store8, sl, warp + i * kWarps, t);
            if (i + 2 < ng) {
                const int q = warp + (i + 2) * kWarps;
                load_b<R, YT>(e0, slotB, v.d_out, sl, q, g, t);
                load_y<R, YT, TM>(e0, yrow, row_ok, yrow8, row_ok8, sl, q, t);
            }
            if (i + 1 < ng) {
                mma_expand_store<R, YT, TM>(e1, ah, al, scale, yrow, store, yrow8, store8, sl, warp + (i + 1) * kWarps,
                                        t);
                if (i + 3 < ng) {
                    const int q = warp + (i + 3) * kWarps;
                    load_b<R, YT>(e1, slotB, v.d_out, sl, q, g, t);
                    load_y<R, YT, TM>(e1, yrow, row_ok, yrow8, row_ok8, sl, q, t);
                }
            }
        }
    }
    if constexpr (MODE != MODE_EXPAND) cluster_wait_acquire();
}

// FUSED: the launch applies p.n_proj projections that share X and the metadata.  A
// work item is (tile, projection), projection fastest, so the clusters working on one
// tile's projections run side by side and its X rows come from HBM once (the later
// reads hit L2).  Otherwise the only projection is p.proj[0].
template <int RMAX, int MODE, int NT, bool FUSED, int DT = 0, int TM = kTileRows>
__global__ void __launch_bounds__(NT, (DecodeCfg<RMAX, NT, TM>::MIN_BLOCKS))
    lora_decode_kernel(const __grid_constant__ TileParams p)
{
    extern __shared__ __align__(16) float smem_f[];
    __shared__ SharedCtl ctl;
    constexpr bool kTable = NT == 128 && (FUSED || RMAX > 16);
    __shared__ SegTable<kTable> segtab;
    const int tid = threadIdx.x;
    const uint32_t crank = cluster_rank();
    const uint32_t csize = cluster_size();
    const int n_clusters = (int)(gridDim.x / csize);
    const bool reporter = blockIdx.x == 0;
    const int np = FUSED ? p.n_proj : 1;

    int item = (int)cluster_index();
    int tile = FUSED ? item / np : item;
    int k = FUSED ? item - tile * np : 0;
    // the next launch may start its CTAs now (they wait before touching our results)
    griddep_launch_dependents();
    if constexpr (MODE != MODE_EXPAND) {
        // receive barriers of the partial-H exchange, initialised before any peer pushes
        if (tid == 0) {
            mbar_init(&ctl.hbar[0], 1);
            mbar_init(&ctl.hbar[1], 1);
            fence_mbar_init();
            ctl.fail = 0;
        }
        cluster_arrive_release();
        cluster_wait_acquire();
    }
    if (p.early) prefetch_first_tile<RMAX, MODE, NT, DT, TM>(p, p.proj[k], tile, ctl, crank);
    griddep_wait();
    const int item2 = item + n_clusters;   // this cluster's next work item
    const int total = scan_tiles<false, NT, MODE, RMAX, TM>(p, p.proj[k].slot_gen, tile, item2 / np,
                                                        p.proj[FUSED ? item2 % np : 0], ctl, reporter,
                                                        kTable ? segtab.first : nullptr) *
                      np;
    uint32_t nt = 0;   // tiles done by this CTA (parity of the exchange buffers and barriers)
    for (; item < total; item += n_clusters, ++nt) {
        if constexpr (FUSED) {
            tile = item / np;
            k = item - tile * np;
        } else {
            tile = item;
        }
        const ProjView &v = p.proj[k];
        if (item != (int)cluster_index()) {
            const int next = item + n_clusters;
            // later tiles: a binary search in the first scan's table, else another scan
            if (kTable && p.n_segments <= kSegTable)
                find_tile<MODE, RMAX, TM>(p, v.slot_gen, tile, next < total ? next / np : -1,
                                          p.proj[FUSED ? next % np : 0], ctl, segtab.first);
            else
                scan_tiles<false, NT, MODE, RMAX, TM>(p, v.slot_gen, tile, next / np, p.proj[FUSED ? next % np : 0],
                                                  ctl, false);
        }
        // every CTA of the cluster reads the same metadata and reaches the same tile
        Tile tl;
        tl.seg = ctl.tile[0];
        tl.p0 = ctl.tile[1];
        tl.nvalid = min(TM, ctl.tile[2] - tl.p0);
        tl.slot = ctl.tile[3];
        const int r_meta = ctl.tile[4];
        const float seg_scale = ctl.seg_scale;
        // rank bucket from the metadata when it is given and in range, else from the slot
        int R = rank_bucket(r_meta);
        if (p.ranks == nullptr || R == 0 || R > RMAX) {
            __syncthreads();
            if (tid == 0) ctl.slot_rank = v.slot_rank[tl.slot];
            __syncthreads();
            R = rank_bucket(ctl.slot_rank);
            if (R == 0 || R > RMAX) R = 8;   // rejected inside; moves rank-8 bytes
        }
        if (R == 8) {
            run_tile<RMAX, MODE, 8, NT, DT, TM>(p, v, tl, r_meta, seg_scale, ctl, smem_f, crank, csize, nt);
        } else if (R == 16) {
            if constexpr (RMAX >= 16)
                run_tile<RMAX, MODE, 16, NT, DT, TM>(p, v, tl, r_meta, seg_scale, ctl, smem_f, crank, csize, nt);
        } else if (R == 32) {
            if constexpr (RMAX >= 32)
                run_tile<RMAX, MODE, 32, NT, DT, TM>(p, v, tl, r_meta, seg_scale, ctl, smem_f, crank, csize, nt);
        } else {
            if constexpr (RMAX >= 64)
                run_tile<RMAX, MODE, 64, NT, DT, TM>(p, v, tl, r_meta, seg_scale, ctl, smem_f, crank, csize, nt);
        }
        __syncthreads();   // ctl and the H buffers are rewritten by the next tile
    }
}

// Clusters of `cluster` CTAs of this kernel resident at once (cached per device).
template <int RMAX, int MODE, int NT, bool FUSED, int DT = 0, int TM = kTileRows>
cudaError_t active_clusters(int cluster, int &active)
{
    static std::mutex mu;
    static int cached[64][kMaxCluster + 1] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    active = cached[dev][cluster];
    if (active > 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cluster, 1, 1);
    cfg.blockDim = dim3(NT, 1, 1);
    cfg.dynamicSmemBytes = DecodeCfg<RMAX, NT, TM>::SMEM;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e =
        cudaOccupancyMaxActiveClusters(&active, lora_decode_kernel<RMAX, MODE, NT, FUSED, DT, TM>, &cfg);
    if (e != cudaSuccess) return e;
    if (active <= 0) return cudaErrorInvalidConfiguration;
    cached[dev][cluster] = active;
    return cudaSuccess;
}

template <int RMAX, int MODE, int NT, bool FUSED, int DT = 0, int TM = kTileRows>
cudaError_t launch_one(const TileParams &p, int cluster, int64_t max_tiles, int active,
                       cudaStream_t stream)
{
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(NT, 1, 1);
    cfg.dynamicSmemBytes = DecodeCfg<RMAX, NT, TM>::SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // programmatic dependent launch: CTAs may start while the previous kernel in the
    // stream finishes; the kernel waits (griddepcontrol.wait) before reading inputs
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = p.early ? 2 : 1;
    const int64_t n = max_tiles < active ? max_tiles : active;
    cfg.gridDim = dim3((unsigned)(n * cluster), 1, 1);
    return cudaLaunchKernelEx(&cfg, lora_decode_kernel<RMAX, MODE, NT, FUSED, DT, TM>, p);
}

// CTA width.  256 threads keep each warp's operands in one round of loads; when the
// batch has clearly more tiles than 256-thread clusters fit at once (many adapters or
// long decode segments), 128-thread CTAs let twice as many tiles be in flight, which
// hides more latency than their second round of loads costs (measured: a 4096 x 4096
// batch of 60 tiles is 36% slower with 128 threads, batches of 300+ tiles 3-6% faster).
template <int RMAX, int MODE, bool FUSED = false, int DT = 0, int TM = kTileRows>
cudaError_t launch_mode(const TileParams &p, int cluster, int64_t max_tiles, cudaStream_t stream)
{
    int active = 0;
    cudaError_t e = active_clusters<RMAX, MODE, 256, FUSED, DT, TM>(cluster, active);
    if (e != cudaSuccess) return e;
    if (2 * max_tiles > 3 * (int64_t)active) {
        int active128 = 0;
        e = active_clusters<RMAX, MODE, 128, FUSED, DT, TM>(cluster, active128);
        if (e != cudaSuccess) return e;
        // Early launch with adapter prefetch only pays for batches of about one wave of
        // tiles: with many more, the prefetched slices thrash L2 and the early CTAs
        // hold slots (measured 16% slower on 2048 decode rows over 128 adapters).
        TileParams q = p;
        q.early = 0;
        return launch_one<RMAX, MODE, 128, FUSED, DT, TM>(q, cluster, max_tiles, active128, stream);
    }
    return launch_one<RMAX, MODE, 256, FUSED, DT, TM>(p, cluster, max_tiles, active, stream);
}

// 16-row tiles for batches of long decode segments at small rank (see kMaxTM).
// max_tiles counts 8-row tiles; a 16-row tile takes about two of them.
template <int RMAX, bool FUSED>
cudaError_t launch_apply(const TileParams &p, int cluster, int64_t max_tiles, cudaStream_t stream)
{
    if constexpr (RMAX <= 16) {
        if ((int64_t)p.n_tokens >= 8 * (int64_t)p.n_segments)
            return launch_mode<RMAX, MODE_APPLY, FUSED, 0, 16>(p, cluster, (max_tiles + 1) / 2 + 1, stream);
    }
    return launch_mode<RMAX, MODE_APPLY, FUSED>(p, cluster, max_tiles, stream);
}

// The fused apply with another dtype boundary (DT != 0: FP8 X codes and / or an fp16 or
// fp32 base output).
template <int RMAX>
cudaError_t launch_dt(int dt, const TileParams &p, int cluster, int64_t max_tiles, cudaStream_t stream)
{
    switch (dt) {
    case 1: return launch_mode<RMAX, MODE_APPLY, false, 1>(p, cluster, max_tiles, stream);
    case 2: return launch_mode<RMAX, MODE_APPLY, false, 2>(p, cluster, max_tiles, stream);
    case 3: return launch_mode<RMAX, MODE_APPLY, false, 3>(p, cluster, max_tiles, stream);
    case 4: return launch_mode<RMAX, MODE_APPLY, false, 4>(p, cluster, max_tiles, stream);
    case 5: return launch_mode<RMAX, MODE_APPLY, false, 5>(p, cluster, max_tiles, stream);
    default: return cudaErrorInvalidValue;
    }
}

template <int RMAX>
cudaError_t launch_rmax(int mode, const TileParams &p, int cluster, int64_t max_tiles,
                        cudaStream_t stream)
{
    switch (mode) {
    case MODE_APPLY: return launch_apply<RMAX, false>(p, cluster, max_tiles, stream);
    case MODE_SHRINK: return launch_mode<RMAX, MODE_SHRINK>(p, cluster, max_tiles, stream);
    case MODE_EXPAND: return launch_mode<RMAX, MODE_EXPAND>(p, cluster, max_tiles, stream);
    default: return cudaErrorInvalidValue;
    }
}

// The shared-memory carveout is left to the driver: a preference for more L1
// starves the kernel of resident CTAs, one for more shared memory shrinks the L1
// through which its register operands stream (both measured slower).
template <int RMAX, int NT>
cudaError_t set_attrs_nt()
{
    cudaError_t e;
    if constexpr (RMAX <= 16) {
        e = cudaFuncSetAttribute(lora_decode_kernel<RMAX, MODE_APPLY, NT, false, 0, 16>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, DecodeCfg<RMAX, NT, 16>::SMEM);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(lora_decode_kernel<RMAX, MODE_APPLY, NT, true, 0, 16>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, DecodeCfg<RMAX, NT, 16>::SMEM);
        if (e != cudaSuccess) return e;
    }
    e = cudaFuncSetAttribute(lora_decode_kernel<RMAX, MODE_APPLY, NT, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, DecodeCfg<RMAX, NT>::SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(lora_decode_kernel<RMAX, MODE_APPLY, NT, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, DecodeCfg<RMAX, NT>::SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(lora_decode_kernel<RMAX, MODE_SHRINK, NT, false>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, DecodeCfg<RMAX, NT>::SMEM);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(lora_decode_kernel<RMAX, MODE_EXPAND, NT, false>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, DecodeCfg<RMAX, NT>::SMEM);
}

template <int RMAX, int NT, int DT>
cudaError_t set_attrs_dt()
{
    return cudaFuncSetAttribute(lora_decode_kernel<RMAX, MODE_APPLY, NT, false, DT>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, DecodeCfg<RMAX, NT>::SMEM);
}

template <int RMAX, int NT>
cudaError_t set_attrs_dts()
{
    cudaError_t e;
    if ((e = set_attrs_dt<RMAX, NT, 1>()) != cudaSuccess) return e;
    if ((e = set_attrs_dt<RMAX, NT, 2>()) != cudaSuccess) return e;
    if ((e = set_attrs_dt<RMAX, NT, 3>()) != cudaSuccess) return e;
    if ((e = set_attrs_dt<RMAX, NT, 4>()) != cudaSuccess) return e;
    return set_attrs_dt<RMAX, NT, 5>();
}

template <int RMAX>
cudaError_t set_attrs()
{
    cudaError_t e = set_attrs_nt<RMAX, 256>();
    if (e != cudaSuccess) return e;
    if ((e = set_attrs_nt<RMAX, 128>()) != cudaSuccess) return e;
    if ((e = set_attrs_dts<RMAX, 256>()) != cudaSuccess) return e;
    return set_attrs_dts<RMAX, 128>();
}

// Repack: A [rank, d_in] -> [d_in/8][R][8]; B [d_out, rank] -> [R/8][d_out][8]; zero
// beyond rank.  One thread per 16-byte destination group, written in order.
__global__ void repack_slot_kernel(__nv_bfloat16 *slot, int64_t b_offset, int R, int rank,
                                   int d_in, int d_out, const __nv_bfloat16 *A,
                                   const __nv_bfloat16 *B, int32_t *rank_entry,
                                   float *scale_entry, float scale, uint32_t *gen_entry,
                                   uint32_t generation)
{
    const int na = R * (d_in / 8);    // 16-byte groups of the A block
    const int nb = (R / 8) * d_out;   // 16-byte groups of the B block
    const __nv_bfloat16 zero = __float2bfloat16_rn(0.f);
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < na + nb; e += gridDim.x * blockDim.x) {
        __align__(16) __nv_bfloat16 v[8];
        __nv_bfloat16 *dst;
        if (e < na) {
            const int kg = e / R, j = e - kg * R;          // group [kg][j][0..7]
#pragma unroll
            for (int c = 0; c < 8; ++c)
                v[c] = j < rank ? A[(int64_t)j * d_in + kg * 8 + c] : zero;
            dst = slot + (int64_t)e * 8;
        } else {
            const int f = e - na;
            const int jg = f / d_out, o = f - jg * d_out;   // group [jg][o][0..7]
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const int j = jg * 8 + c;
                v[c] = j < rank ? B[(int64_t)o * rank + j] : zero;
            }
            dst = slot + b_offset + (int64_t)f * 8;
        }
        *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(v);
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        *rank_entry = rank;
        *scale_entry = scale;
        *gen_entry = generation;
    }
}

__global__ void publish_slot_kernel(int32_t *rank_entry, float *scale_entry, uint32_t *gen_entry,
                                    int rank, float scale, uint32_t generation)
{
    *rank_entry = rank;
    *scale_entry = scale;
    *gen_entry = generation;
}

}  // namespace

cudaError_t launch_tile_kernel_dt(int dt, int rmax_bucket, const TileParams &p, int cluster, int64_t max_tiles,
                                  cudaStream_t stream)
{
    if (cluster < 1 || cluster > kMaxCluster || max_tiles < 1) return cudaErrorInvalidValue;
    switch (rmax_bucket) {
    case 8: return launch_dt<8>(dt, p, cluster, max_tiles, stream);
    case 16: return launch_dt<16>(dt, p, cluster, max_tiles, stream);
    case 32: return launch_dt<32>(dt, p, cluster, max_tiles, stream);
    case 64: return launch_dt<64>(dt, p, cluster, max_tiles, stream);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_tile_kernel(int mode, int rmax_bucket, const TileParams &p, int cluster,
                               int64_t max_tiles, cudaStream_t stream)
{
    if (cluster < 1 || cluster > kMaxCluster || max_tiles < 1) return cudaErrorInvalidValue;
    switch (rmax_bucket) {
    case 8: return launch_rmax<8>(mode, p, cluster, max_tiles, stream);
    case 16: return launch_rmax<16>(mode, p, cluster, max_tiles, stream);
    case 32: return launch_rmax<32>(mode, p, cluster, max_tiles, stream);
    case 64: return launch_rmax<64>(mode, p, cluster, max_tiles, stream);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_tile_kernel_fused(int rmax_bucket, const TileParams &p, int cluster,
                                     int64_t max_items, cudaStream_t stream)
{
    if (cluster < 1 || cluster > kMaxCluster || max_items < 1) return cudaErrorInvalidValue;
    if (p.n_proj < 1 || p.n_proj > kMaxFused) return cudaErrorInvalidValue;
    switch (rmax_bucket) {
    case 8: return launch_apply<8, true>(p, cluster, max_items, stream);
    case 16: return launch_apply<16, true>(p, cluster, max_items, stream);
    case 32: return launch_mode<32, MODE_APPLY, true>(p, cluster, max_items, stream);
    case 64: return launch_mode<64, MODE_APPLY, true>(p, cluster, max_items, stream);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t prepare_tile_kernels()
{
    cudaError_t e;
    if ((e = set_attrs<8>()) != cudaSuccess) return e;
    if ((e = set_attrs<16>()) != cudaSuccess) return e;
    if ((e = set_attrs<32>()) != cudaSuccess) return e;
    return set_attrs<64>();
}

cudaError_t launch_repack_slot(__nv_bfloat16 *slot_base, int64_t b_offset, int R, int rank,
                               int d_in, int d_out, const __nv_bfloat16 *A_src,
                               const __nv_bfloat16 *B_src, int32_t *slot_rank_entry,
                               float *slot_scale_entry, float scale, uint32_t *slot_gen_entry,
                               uint32_t generation, cudaStream_t stream)
{
    const int64_t groups = (int64_t)R * (d_in / 8) + (int64_t)(R / 8) * d_out;
    const int threads = 256;
    const int64_t blocks64 = (groups + threads - 1) / threads;
    const int blocks = (int)(blocks64 < 2048 ? blocks64 : 2048);
    repack_slot_kernel<<<blocks, threads, 0, stream>>>(slot_base, b_offset, R, rank, d_in, d_out,
                                                       A_src, B_src, slot_rank_entry,
                                                       slot_scale_entry, scale, slot_gen_entry,
                                                       generation);
    return cudaGetLastError();
}

cudaError_t launch_publish_slot(int32_t *slot_rank_entry, float *slot_scale_entry,
                                uint32_t *slot_gen_entry, int rank, float scale,
                                uint32_t generation, cudaStream_t stream)
{
    publish_slot_kernel<<<1, 1, 0, stream>>>(slot_rank_entry, slot_scale_entry, slot_gen_entry, rank,
                                             scale, generation);
    return cudaGetLastError();
}

}  // namespace mlora
