// base_gemm.cu -- the base projection and the LoRA delta in one tensor-core pass.
//
// Y = X W^T + s_a (X A_a^T) B_a^T for the rows of adapter segments and Y = X W^T for
// every other row (page "Multi-LoRA serving", ybb.press ai-applications, section 3.3
// on fusing W0 x + B(A x) into one kernel, and its paragraph on cuBLASLt epilogue
// fusion after section 5.3: the low-rank product goes into the base GEMM's accumulator, so Y is
// written once, in bf16, and never read).
//
// Order of work.  The shrink H = X A_a^T is the library's segmented shrink (the
// decode-shaped kernel, and the tensor-memory kernel for long segments) into an fp32
// workspace in grouped order.  row_map_kernel then gives each row its grouped
// position, slot, scale and rank (rows outside every valid segment keep position -1:
// base only), and block_slots_kernel lists the distinct slots of each 256-row block.
// Last, the persistent GEMM below.
//
// GEMM tile: 256 rows x 256 columns of Y, computed by a pair of CTAs (a cluster of
// two on neighbouring SMs) with tcgen05.mma.cta_group::2: CTA c holds rows
// [128 c, +128) of the tile's X and rows [128 c, +128) of its W columns, so each SM
// streams half of what a one-CTA 128 x 256 tile needs per flop, and its tensor
// memory holds its 128 rows of the fp32 accumulator (two accumulators of 256 columns,
// so that a tile's epilogue overlaps the next tile's main loop).  Warp roles, in both
// CTAs, which meet only at mbarriers:
//   warp 0     TMA: per 64-wide K block the CTA's X tile (128 x 64) and W half
//              (128 x 64), 128-byte swizzle, into a 6-stage ring; after the K blocks,
//              per distinct slot of the tile's rows the CTA's half (128 columns x all
//              rank groups) of that slot's B chunk.  Both CTAs' copies complete on the
//              even CTA's mbarriers, which its MMA thread waits on.
//   warp 1     tensor memory (allocated for the pair); in the even CTA one thread
//              issues the pair's tcgen05.mma (M=256, N=256, K=16): four per K block,
//              then per slot (s H)_hi B^T + (s H)_lo B^T; its commits arrive on the
//              mbarriers of both CTAs
//   warps 2-5  epilogue: tcgen05.ld of the CTA's 128 rows, one rounding to bf16,
//              16-byte stores of Y
//   warps 6-9  LoRA operand: the CTA's rows of s H for one slot (rows of other slots
//              and base rows zero), as bf16 hi + lo in the tensor core's K-major
//              no-swizzle layout; the masking makes one M=256 product per slot exact
//              for the rows of that slot and zero for the others
// Every mbarrier wait is bounded; on expiry the kernel flags a timeout (in both CTAs
// of the pair), stores nothing more, lets copies in flight land and frees its tensor
// memory before it leaves.
#include <algorithm>
#include <mutex>

#include "kernels.cuh"
#include "ptx.cuh"

namespace mlora {

namespace {

constexpr int GM = 128;                // rows per CTA (one tensor-memory lane each)
constexpr int PM = kGemmRows;          // 256 rows per pair tile
constexpr int UN = 256;                // columns of Y per unit (one 256-column slab of tensor memory)
constexpr int NH = UN / 2;             // W rows (and B columns) per CTA per unit
constexpr int GK = 64;                 // K columns per stage (one 128-byte swizzled row)
constexpr int X_BYTES = GM * GK * 2;   // 16 KB
constexpr int W_BYTES = NH * GK * 2;   // 16 KB per unit
constexpr int B_BYTES = NH * 64 * 2;   // one B copy (128 columns) at rank bucket 64
constexpr int HOP = GM * 64 * 2;       // one of hi / lo at rank bucket 64: [8][16][8][8] bf16
constexpr int HOP_BUF = 2 * HOP;       // one operand buffer (hi, lo); two of them
// Rank bucket 8 runs as K=16: its second operand half is read from 2 KB of zeros
// placed in the part of the hi buffer that bucket 8 leaves unused.
constexpr int ZERO_OFF = 8192;
constexpr int G_WARPS = 10;
constexpr int GT = G_WARPS * 32;
constexpr int kEpiBar = 1;             // named barrier of the epilogue warps
constexpr int kStgBar = 2;             // named barrier of the operand warps
constexpr int G_TMEM = 2 * UN;         // two slabs: all of tensor memory
constexpr uint16_t kPairMask = 0x3;    // both CTAs of the cluster
constexpr uint64_t kGemmWaitNs = 1000000000ull;

static_assert(ZERO_OFF >= 2 * (GM / 8) * 128 && ZERO_OFF + NH * 16 <= HOP, "zero block placement");
static_assert(PM == 2 * GM, "a pair tile is two CTAs' rows");
static_assert(kExpandChunk == NH, "B copies are the pool's 128-column view");

// A pair tile is NSUB units of 256 columns.  NSUB = 1: each tile takes one slab of
// tensor memory, alternating, so a tile's epilogue overlaps the next tile's main loop.
// NSUB = 2: a tile takes both slabs; per K block each CTA copies 128 rows of X and
// 2 x 128 rows of W for twice the tensor-core work, a third fewer bytes per flop --
// the main loop of NSUB = 1 is bound by its copies on B200, that of NSUB = 2 by the
// tensor core -- and the epilogue hands each slab back as soon as it has read it.
template <int NSUB>
struct Shape {
    static constexpr int GN = NSUB * UN;
    static constexpr int STAGE = X_BYTES + NSUB * W_BYTES;   // also holds NSUB B copies
    static constexpr int GS = NSUB == 1 ? 5 : 3;             // ring stages
    static constexpr int SMEM = 1024 + GS * STAGE + 2 * HOP_BUF;
    static_assert(NSUB * B_BYTES <= STAGE && STAGE % 1024 == 0, "stage layout");
    static_assert(SMEM + 1024 <= 227 * 1024, "shared memory");
};
constexpr int kMaxStages = 5;

struct GemmCtl {
    uint64_t full[kMaxStages], empty[kMaxStages];
    uint64_t slab_full[2], slab_empty[2];
    uint64_t hop_full[2], hop_empty[2];
    uint32_t tmem;
    volatile int fail;
};

__device__ __forceinline__ uint8_t *align_1024(uint8_t *p)
{
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Bounded wait (acquire at cluster scope: the partner CTA and the tensor-core
// commits of the pair arrive on these barriers).  On expiry both CTAs of the pair
// are told to stop.
__device__ __forceinline__ bool gwait(const GemmParams &p, GemmCtl &ctl, uint64_t *bar, uint32_t parity)
{
    if (ctl.fail) return false;
    if (!mbar_wait_bounded_cluster(bar, parity, kGemmWaitNs)) {
        ctl.fail = 1;
        st_cluster_u32(map_to_rank(smem_addr((const void *)&ctl.fail), cluster_rank() ^ 1u), 1u);
        atomicOr(p.status, kFlagTimeout);
        return false;
    }
    return true;
}

// Tile t -> (256-row block mb, column block nb).  Tiles run in groups of
// kGroupRows row blocks, column-major inside a group, so that the pairs working at
// the same time share a few row blocks of X and a few column blocks of W in L2.
constexpr int kGroupRows = 8;

__device__ __forceinline__ void tile_coords(const GemmParams &p, int t, int &mb, int &nb)
{
    const int per_group = kGroupRows * p.n_nblk;
    const int first_mb = (t / per_group) * kGroupRows;
    const int rows = min(kGroupRows, p.n_mblk - first_mb);
    const int local = t % per_group;
    mb = first_mb + local % rows;
    nb = local / rows;
}

// Cluster address of `bar` in the even CTA of the pair (rank 0 of the cluster).
__device__ __forceinline__ uint32_t leader_bar(const uint64_t *bar) { return map_to_rank(smem_addr(bar), 0); }

__device__ __forceinline__ int bucket_index(int R) { return R <= 8 ? 0 : R <= 16 ? 1 : R <= 32 ? 2 : 3; }

}  // namespace

// ------------------------------------------------------------------ row map
// The problems of segment g (status bits as the other kernels report them), 0 if it
// is a valid adapter segment; *rank and *scale are set for a valid one.
__device__ __forceinline__ unsigned segment_problem(const TileParams &p, int g, int a, int p0, int p1, int &rank,
                                                    float &scale)
{
    if (a < -1 || a >= p.n_slots) return kFlagBadSlot;
    if (p0 < 0 || p1 < p0 || p1 > p.n_tokens) return kFlagBadOffsets;
    if (a < 0) return 0;
    rank = p.slot_rank[a];
    scale = p.scales ? p.scales[g] : p.slot_scale[a];
    if (p.generations && p.slot_gen[a] != p.generations[g]) return kFlagStaleSlot;
    if (rank <= 0) return kFlagSlotEmpty;
    if ((p.ranks && p.ranks[g] != rank) || rank_bucket(rank) == 0) return kFlagBadRank;
    return 0;
}

// Grid-stride over segments (their problems are reported once each) and over
// grouped positions: position q belongs to the segment g with offsets[g] <= q <
// offsets[g + 1] (binary search over the offsets); when that segment is a valid
// adapter segment, row_info[token_indices[q]] = {q, slot, scale, rank}.  A row
// claimed twice keeps its first claim and is reported; rows of base or rejected
// segments and uncovered rows keep position -1 (base only).
__global__ void __launch_bounds__(256) row_map_kernel(const __grid_constant__ TileParams p, int4 *row_info)
{
    const int stride = (int)(gridDim.x * blockDim.x);
    const int i0 = (int)(blockIdx.x * blockDim.x + threadIdx.x);
    for (int g = i0; g < p.n_segments; g += stride) {
        int rank = 0;
        float scale = 0.f;
        const unsigned f = segment_problem(p, g, p.slots[g], p.offsets[g], p.offsets[g + 1], rank, scale);
        if (f) atomicOr(p.status, f);
    }
    if (p.n_segments <= 0) return;
    for (int q = i0; q < p.n_tokens; q += stride) {
        int lo = 0, hi = p.n_segments - 1;   // last g with offsets[g] <= q
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (p.offsets[mid] <= q) lo = mid;
            else hi = mid - 1;
        }
        const int g = lo, a = p.slots[g], p0 = p.offsets[g], p1 = p.offsets[g + 1];
        if (a < 0 || q < p0 || q >= p1) continue;
        int rank = 0;
        float scale = 0.f;
        if (segment_problem(p, g, a, p0, p1, rank, scale)) continue;
        const int t = p.token_indices ? p.token_indices[q] : q;
        if (t < 0 || t >= p.n_rows || atomicCAS(&row_info[t].x, -1, q) != -1) {
            atomicOr(p.status, kFlagBadRow);
            continue;
        }
        row_info[t].y = a;
        row_info[t].z = __float_as_int(scale);
        row_info[t].w = rank;
    }
}

// One CTA of 256 threads per 256-row block: the distinct slots of the block's rows in
// order of first appearance, as out[0] = count, then (slot, rank bucket) pairs.
__global__ void __launch_bounds__(PM) block_slots_kernel(const int4 *row_info, int n_rows, int32_t *out)
{
    __shared__ int s_slot[PM];
    __shared__ int s_count[PM / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int row = blockIdx.x * PM + tid;
    int slot = -1, rank = 0;
    if (row < n_rows) {
        const int4 v = row_info[row];
        if (v.x >= 0) {
            slot = v.y;
            rank = v.w;
        }
    }
    s_slot[tid] = slot;
    __syncthreads();
    bool first = slot >= 0;
    for (int j = 0; j < tid && first; ++j)
        if (s_slot[j] == slot) first = false;
    const unsigned m = __ballot_sync(0xffffffffu, first);
    if (lane == 0) s_count[warp] = __popc(m);
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < PM / 32; ++w) {
        before += w < warp ? s_count[w] : 0;
        total += s_count[w];
    }
    int32_t *o = out + (int64_t)blockIdx.x * kBlockSlotsPitch;
    if (first) {
        const int idx = before + __popc(m & ((1u << lane) - 1u));
        o[1 + 2 * idx] = slot;
        o[2 + 2 * idx] = rank_bucket(rank);
    }
    if (tid == 0) o[0] = total;
}

// One row of the LoRA operand: s * H[row, 0:rank) (zeros past rank, all zeros for
// rank 0) as bf16 hi + lo parts in the K-major no-swizzle layout [RK/8][16][8][8].
// The row's loads are all issued before any is used.
template <int RK>
__device__ __forceinline__ void stage_operand(uint8_t *hi, uint8_t *lo, const float *hsrc, int rank, float sc, int r)
{
    float h[RK];
    if (rank == RK) {
#pragma unroll
        for (int i = 0; i < RK / 4; ++i) {
            const float4 v = reinterpret_cast<const float4 *>(hsrc)[i];
            h[4 * i] = v.x;
            h[4 * i + 1] = v.y;
            h[4 * i + 2] = v.z;
            h[4 * i + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int c = 0; c < RK; ++c) h[c] = c < rank ? hsrc[c] : 0.f;
    }
#pragma unroll
    for (int cg = 0; cg < RK / 8; ++cg) {
        uint4 vh, vl;
        uint32_t *ph = reinterpret_cast<uint32_t *>(&vh);
        uint32_t *pl = reinterpret_cast<uint32_t *>(&vl);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float h0, l0, h1, l1;
            split_bf16(sc * h[8 * cg + 2 * c], h0, l0);
            split_bf16(sc * h[8 * cg + 2 * c + 1], h1, l1);
            ph[c] = pack_bf16x2(h0, h1);
            pl[c] = pack_bf16x2(l0, l1);
        }
        const int off = (cg * (GM / 8) + r / 8) * 128 + (r % 8) * 16;
        *reinterpret_cast<uint4 *>(hi + off) = vh;
        *reinterpret_cast<uint4 *>(lo + off) = vl;
    }
}

// ------------------------------------------------------------------ GEMM
// Pair tiles t = cluster index, + number of clusters, ...; tile t covers rows
// [256 mb, +256) and columns [GN nb, +GN) with (mb, nb) from tile_coords.  Every role
// of both CTAs walks the same tiles and reads the same slot lists, so the ring, the
// slabs and the operand buffers are used in the same order on both sides of each
// mbarrier.  Unit u of a tile (columns [256 u, +256) of it) accumulates in slab
// unit_slab(tc, u) of tensor memory; that slab's use count is slab_use(tc).
template <int NSUB>
__device__ __forceinline__ int unit_slab(uint32_t tc, int u) { return NSUB == 2 ? u : (int)(tc & 1); }
template <int NSUB>
__device__ __forceinline__ uint32_t slab_use(uint32_t tc) { return NSUB == 2 ? tc : tc >> 1; }

template <int NSUB>
__global__ void __launch_bounds__(GT, 1) base_gemm_kernel(const __grid_constant__ GemmParams p)
{
    using S = Shape<NSUB>;
    constexpr int GN = S::GN, STAGE = S::STAGE, GS = S::GS;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ GemmCtl ctl;
    uint8_t *ring = align_1024(smem_raw);
    uint8_t *hop = ring + GS * STAGE;              // [2][hi, lo]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t crank = cluster_rank();        // 0 issues the pair's MMAs
    const bool leader = crank == 0;
    const int n_clusters = (int)(gridDim.x / 2);
    const int first = (int)cluster_index();

    if (warp == 1) {
        tmem_alloc_pair(&ctl.tmem, G_TMEM);
        tmem_relinquish_pair();
    }
    if (tid == 0) {
        for (int s = 0; s < GS; ++s) {
            mbar_init(&ctl.full[s], 1);
            mbar_init(&ctl.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl.slab_full[b], 1);
            mbar_init(&ctl.slab_empty[b], 8);  // four epilogue warps in each CTA
            mbar_init(&ctl.hop_full[b], 2);    // one arrival per CTA
            mbar_init(&ctl.hop_empty[b], 1);
        }
        fence_mbar_init();
        ctl.fail = 0;
    }
    tc_fence_before();
    __syncthreads();
    // both CTAs' barriers exist before either signals the other's
    cluster_arrive_release();
    cluster_wait_acquire();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem;
    const int n_tiles = p.n_mblk * p.n_nblk;
    const int nk = (p.d_in + GK - 1) / GK;

    if (warp == 0) {
        // ---------------------------------------------------------------- copies
        if (lane == 0) {
            uint32_t g = 0;
            for (int t = first; t < n_tiles && !ctl.fail; t += n_clusters) {
                int mb, nb;
                tile_coords(p, t, mb, nb);
                const int m0 = mb * PM + GM * (int)crank;    // this CTA's rows
                const int nc = nb * GN + NH * (int)crank;     // this CTA's first W row / B column
                for (int kb = 0; kb < nk; ++kb, ++g) {
                    const int s = (int)(g % GS);
                    if (g >= GS && !gwait(p, ctl, &ctl.empty[s], ((g / GS) - 1) & 1u)) break;
                    uint8_t *st = ring + s * STAGE;
                    if (leader) mbar_arrive_expect_tx(&ctl.full[s], 2u * STAGE);
                    const uint32_t fb = leader_bar(&ctl.full[s]);
                    tma_load_2d_pair(st, &p.x_map, kb * GK, m0, fb);
#pragma unroll
                    for (int u = 0; u < NSUB; ++u)
                        tma_load_2d_pair(st + X_BYTES + u * W_BYTES, &p.w_map, kb * GK, nc + u * UN, fb);
                }
                const int32_t *bs = p.block_slots + (int64_t)mb * kBlockSlotsPitch;
                const int cnt = bs[0];
                for (int j = 0; j < cnt && !ctl.fail; ++j, ++g) {
                    const int slot = bs[1 + 2 * j], R = bs[2 + 2 * j];
                    const int s = (int)(g % GS);
                    if (g >= GS && !gwait(p, ctl, &ctl.empty[s], ((g / GS) - 1) & 1u)) break;
                    // columns past d_out read as zeros
                    if (leader) mbar_arrive_expect_tx(&ctl.full[s], 2u * NSUB * (uint32_t)R * NH * 2);
                    const uint32_t fb = leader_bar(&ctl.full[s]);
#pragma unroll
                    for (int u = 0; u < NSUB; ++u)
                        tma_load_4d_pair(ring + s * STAGE + u * B_BYTES, &p.b_map[bucket_index(R)], 0,
                                         (nc + u * UN) / p.b_col_div, 0, slot, fb);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- tensor core
        if (leader && lane == 0) {
            uint32_t g = 0, hc = 0, tc = 0;
            const uint32_t idesc = umma_idesc_bf16(PM, UN);
            const uint32_t hop0 = smem_addr(hop);
            for (int t = first; t < n_tiles && !ctl.fail; t += n_clusters, ++tc) {
                int mb, nb;
                tile_coords(p, t, mb, nb);
                const uint32_t use = slab_use<NSUB>(tc);
                bool ok = true;
                for (int kb = 0; kb < nk && ok; ++kb, ++g) {
                    const int s = (int)(g % GS);
                    if (!gwait(p, ctl, &ctl.full[s], (g / GS) & 1u)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t xs = smem_addr(ring + s * STAGE);
#pragma unroll
                    for (int u = 0; u < NSUB; ++u) {
                        const int slab = unit_slab<NSUB>(tc, u);
                        // before the tile's first product into a slab, its last reader
                        // (the epilogue) must be done with it
                        if (kb == 0 && use >= 1) {
                            if (!gwait(p, ctl, &ctl.slab_empty[slab], (use - 1) & 1u)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                        }
                        const uint32_t d = tmem + (uint32_t)(slab * UN);
                        const uint32_t ws = xs + X_BYTES + u * W_BYTES;
#pragma unroll
                        for (int k = 0; k < GK / 16; ++k)
                            umma_bf16_pair(d, umma_desc_sw128(xs + 32 * k), umma_desc_sw128(ws + 32 * k), idesc,
                                           (kb > 0 || k > 0) ? 1u : 0u);
                    }
                    if (!ok) break;
                    umma_commit_pair(&ctl.empty[s], kPairMask);   // stage s is free in both CTAs
                }
                if (!ok) break;
                const int32_t *bs = p.block_slots + (int64_t)mb * kBlockSlotsPitch;
                const int cnt = bs[0];
                for (int j = 0; j < cnt; ++j, ++g, ++hc) {
                    const int R = bs[2 + 2 * j];
                    const int RK = R < 16 ? 16 : R;
                    const int s = (int)(g % GS);
                    const int hb = (int)(hc & 1);
                    if (!gwait(p, ctl, &ctl.hop_full[hb], (hc >> 1) & 1u) ||
                        !gwait(p, ctl, &ctl.full[s], (g / GS) & 1u)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_hi = hop0 + hb * HOP_BUF, a_lo = a_hi + HOP, zero = a_hi + ZERO_OFF;
#pragma unroll
                    for (int u = 0; u < NSUB; ++u) {
                        const uint32_t d = tmem + (uint32_t)(unit_slab<NSUB>(tc, u) * UN);
                        const uint32_t b_s = smem_addr(ring + s * STAGE + u * B_BYTES);
                        for (int st = 0; st < RK / 16; ++st) {
                            const uint32_t b0 = b_s + st * 2 * NH * 16;
                            // bucket 8: the second rank group of B is the zero block
                            const uint32_t lbo = R == 8 ? zero - b0 : NH * 16;
                            const uint64_t bd = umma_desc_kmajor(b0, lbo, 128);
                            const uint32_t koff = st * 2 * (GM / 8) * 128;
                            umma_bf16_pair(d, umma_desc_kmajor(a_hi + koff, (GM / 8) * 128, 128), bd, idesc, 1u);
                            umma_bf16_pair(d, umma_desc_kmajor(a_lo + koff, (GM / 8) * 128, 128), bd, idesc, 1u);
                        }
                    }
                    umma_commit_pair(&ctl.empty[s], kPairMask);
                    umma_commit_pair(&ctl.hop_empty[hb], kPairMask);   // operand buffers free in both CTAs
                }
                if (!ok) break;
#pragma unroll
                for (int u = 0; u < NSUB; ++u) umma_commit_pair(&ctl.slab_full[unit_slab<NSUB>(tc, u)], kPairMask);
            }
        }
        __syncwarp();
    } else if (warp < 6) {
        // ---------------------------------------------------------------- epilogue
        const int quarter = warp & 3;             // tensor-memory lanes 32 quarter .. +31
        const uint32_t empty_bar0 = leader_bar(&ctl.slab_empty[0]), empty_bar1 = leader_bar(&ctl.slab_empty[1]);
        const int k = lane & 7;
        uint32_t tc = 0;
        bool alive = true;
        for (int t = first; t < n_tiles && alive; t += n_clusters, ++tc) {
            int mb, nb;
            tile_coords(p, t, mb, nb);
            const uint32_t use = slab_use<NSUB>(tc);
            // lane 8g + k of the warp ends up with 16-byte piece k of rows 8g .. 8g+7 (of
            // the warp's 32), so each store instruction writes four whole 128-byte rows
            const int row0 = mb * PM + GM * (int)crank + 32 * quarter + 8 * (lane >> 3);
            for (int u = 0; u < NSUB; ++u) {
                const int slab = unit_slab<NSUB>(tc, u);
                // every wait ends in a vote, so the four warps leave together
                if (!named_sync_and(kEpiBar, 128, gwait(p, ctl, &ctl.slab_full[slab], use & 1u))) {
                    alive = false;
                    break;
                }
                tc_fence_after();
                const int n0 = nb * GN + u * UN;
                const int ncols = min(UN, p.d_out - n0);
                const uint32_t tbase = tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(slab * UN);
                for (int c = 0; c < UN / 64 && 64 * c < ncols; ++c) {
                    uint32_t v0[32], v1[32];
                    tmem_ld32(tbase + 64 * c, v0);
                    tmem_ld32(tbase + 64 * c + 32, v1);
                    tmem_wait_ld();
                    if (64 * c + 64 >= ncols || c == UN / 64 - 1) {
                        // the slab's last columns are in registers: hand it back
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(slab ? empty_bar1 : empty_bar0);
                    }
                    uint4 a[8];   // this thread's row, columns [64 c, +64), as eight pieces
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        a[q] = make_uint4(pack_bf16x2(__uint_as_float(v0[8 * q]), __uint_as_float(v0[8 * q + 1])),
                                          pack_bf16x2(__uint_as_float(v0[8 * q + 2]), __uint_as_float(v0[8 * q + 3])),
                                          pack_bf16x2(__uint_as_float(v0[8 * q + 4]), __uint_as_float(v0[8 * q + 5])),
                                          pack_bf16x2(__uint_as_float(v0[8 * q + 6]), __uint_as_float(v0[8 * q + 7])));
                        a[4 + q] = make_uint4(pack_bf16x2(__uint_as_float(v1[8 * q]), __uint_as_float(v1[8 * q + 1])),
                                              pack_bf16x2(__uint_as_float(v1[8 * q + 2]), __uint_as_float(v1[8 * q + 3])),
                                              pack_bf16x2(__uint_as_float(v1[8 * q + 4]), __uint_as_float(v1[8 * q + 5])),
                                              pack_bf16x2(__uint_as_float(v1[8 * q + 6]), __uint_as_float(v1[8 * q + 7])));
                    }
                    // 8 x 8 transpose of the pieces across the eight lanes of each group
#pragma unroll
                    for (int sh = 4; sh >= 1; sh >>= 1) {
#pragma unroll
                        for (int jj = 0; jj < 8; ++jj) {
                            if (jj & sh) continue;
                            const bool upper = (k & sh) != 0;
                            const uint4 send = upper ? a[jj] : a[jj | sh];
                            uint4 recv;
                            recv.x = __shfl_xor_sync(0xffffffffu, send.x, sh);
                            recv.y = __shfl_xor_sync(0xffffffffu, send.y, sh);
                            recv.z = __shfl_xor_sync(0xffffffffu, send.z, sh);
                            recv.w = __shfl_xor_sync(0xffffffffu, send.w, sh);
                            if (upper) a[jj] = recv;
                            else a[jj | sh] = recv;
                        }
                    }
                    if (64 * c + 8 * k < ncols) {   // d_out is a multiple of 8
                        __nv_bfloat16 *ycol = p.Y + n0 + 64 * c + 8 * k;
#pragma unroll
                        for (int jj = 0; jj < 8; ++jj)
                            if (row0 + jj < p.n_rows)
                                *reinterpret_cast<uint4 *>(ycol + (int64_t)(row0 + jj) * p.ldy) = a[jj];
                    }
                }
                if (ncols <= 0) {   // a unit wholly past d_out: nothing to read
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(slab ? empty_bar1 : empty_bar0);
                }
            }
        }
    } else {
        // ---------------------------------------------------------------- LoRA operand
        const int r = tid - 6 * 32;               // row 0..127 of this CTA's half
        const uint32_t full_bar0 = leader_bar(&ctl.hop_full[0]), full_bar1 = leader_bar(&ctl.hop_full[1]);
        // H comes from the shrink launched just before this kernel (which may still be
        // running when launched with programmatic dependent launch); nothing else here
        // reads what it writes
        griddep_wait();
        uint32_t hc = 0;
        bool alive = true;
        for (int t = first; t < n_tiles && alive; t += n_clusters) {
            int mb, nb;
            tile_coords(p, t, mb, nb);
            const int32_t *bs = p.block_slots + (int64_t)mb * kBlockSlotsPitch;
            const int cnt = bs[0];
            const int row = mb * PM + GM * (int)crank + r;
            int4 info = make_int4(-1, -1, 0, 0);
            if (cnt > 0 && row < p.n_rows) info = p.row_info[row];
            for (int j = 0; j < cnt; ++j, ++hc) {
                const int slot = bs[1 + 2 * j], R = bs[2 + 2 * j];
                const int hb = (int)(hc & 1);
                // the use of this buffer two slots back must have left the tensor core
                if (hc >= 2 &&
                    !named_sync_and(kStgBar, 128, gwait(p, ctl, &ctl.hop_empty[hb], ((hc >> 1) - 1) & 1u))) {
                    alive = false;
                    break;
                }
                const bool mine = info.x >= 0 && info.y == slot;
                const int rank = mine ? info.w : 0;
                const float sc = mine ? __int_as_float(info.z) : 0.f;   // other rows: exact zeros
                const float *hsrc = p.H + (int64_t)(mine ? info.x : 0) * p.ldh;
                uint8_t *hi = hop + hb * HOP_BUF;
                if (R <= 16) stage_operand<16>(hi, hi + HOP, hsrc, rank, sc, r);
                else if (R == 32) stage_operand<32>(hi, hi + HOP, hsrc, rank, sc, r);
                else stage_operand<64>(hi, hi + HOP, hsrc, rank, sc, r);
                if (R == 8) reinterpret_cast<uint4 *>(hi + ZERO_OFF)[r] = make_uint4(0, 0, 0, 0);
                fence_proxy_async_smem();   // the operand is read by the tensor core
                named_sync(kStgBar, 128);
                if (r == 0) mbar_arrive_cluster(hb ? full_bar1 : full_bar0);
            }
        }
    }

    // leave: tensor-core work done, copies landed, neither CTA still signals the
    // other, tensor memory freed
    __syncthreads();
    if (ctl.fail && tid == 0) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 2000000ull) {
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_arrive_release();
    cluster_wait_acquire();
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem, G_TMEM);
}

// ------------------------------------------------------------------ launches
cudaError_t launch_row_map(const TileParams &p, int4 *row_info, cudaStream_t stream)
{
    if (p.n_rows > 0) {
        cudaError_t e = cudaMemsetAsync(row_info, 0xff, (size_t)p.n_rows * sizeof(int4), stream);
        if (e != cudaSuccess) return e;
    }
    if (p.n_segments <= 0) return cudaSuccess;
    const int64_t items = std::max<int64_t>(p.n_segments, p.n_tokens);
    const int blocks = (int)std::min<int64_t>((items + 255) / 256, 1184);
    row_map_kernel<<<blocks, 256, 0, stream>>>(p, row_info);
    return cudaGetLastError();
}

cudaError_t launch_block_slots(const int4 *row_info, int n_rows, int32_t *block_slots, cudaStream_t stream)
{
    const int n_mblk = (n_rows + PM - 1) / PM;
    if (n_mblk <= 0) return cudaSuccess;
    block_slots_kernel<<<n_mblk, PM, 0, stream>>>(row_info, n_rows, block_slots);
    return cudaGetLastError();
}

namespace {

template <int NSUB>
cudaLaunchConfig_t gemm_config(unsigned pairs, cudaStream_t stream, cudaLaunchAttribute *attr, bool pdl = false)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    cfg.blockDim = dim3(GT, 1, 1);
    cfg.dynamicSmemBytes = Shape<NSUB>::SMEM;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    return cfg;
}

// Pairs of the GEMM resident at once on the current device (cached per device).
template <int NSUB>
cudaError_t gemm_active_pairs(int &active)
{
    static std::mutex mu;
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (cached[dev] > 0) {
        active = cached[dev];
        return cudaSuccess;
    }
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = gemm_config<NSUB>(1, nullptr, attr);
    cudaError_t e = cudaOccupancyMaxActiveClusters(&active, base_gemm_kernel<NSUB>, &cfg);
    if (e != cudaSuccess) return e;
    if (active <= 0) return cudaErrorInvalidConfiguration;
    cached[dev] = active;
    return cudaSuccess;
}

template <int NSUB>
cudaError_t launch_units(const GemmParams &p, cudaStream_t stream, bool pdl)
{
    const int64_t tiles = (int64_t)p.n_mblk * p.n_nblk;
    if (tiles <= 0) return cudaSuccess;
    int active = 0;
    cudaError_t e = gemm_active_pairs<NSUB>(active);
    if (e != cudaSuccess) return e;
    const unsigned pairs = (unsigned)std::min<int64_t>(tiles, active);   // persistent
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = gemm_config<NSUB>(pairs, stream, attr, pdl);
    return cudaLaunchKernelEx(&cfg, base_gemm_kernel<NSUB>, p);
}

template <int NSUB>
cudaError_t prepare_units()
{
    cudaError_t e = cudaFuncSetAttribute(base_gemm_kernel<NSUB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Shape<NSUB>::SMEM);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(base_gemm_kernel<NSUB>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
}

}  // namespace

int choose_gemm_cols(int n_mblk, int d_out)
{
    // Time per 256-column unit, relative (measured on B200): 1.15 for 256-column
    // tiles, whose main loop is bound by its copies, 1.03 for 512-column tiles (tensor
    // core bound, plus the part of the epilogue the next tile cannot hide).  The cost
    // of a width is waves of resident pairs x units per tile x that time.
    int a1 = 0, a2 = 0;
    if (gemm_active_pairs<1>(a1) != cudaSuccess || gemm_active_pairs<2>(a2) != cudaSuccess) return UN;
    const int64_t t1 = (int64_t)n_mblk * ((d_out + UN - 1) / UN);
    const int64_t t2 = (int64_t)n_mblk * ((d_out + 2 * UN - 1) / (2 * UN));
    const int64_t c1 = (t1 + a1 - 1) / a1 * 115, c2 = (t2 + a2 - 1) / a2 * 2 * 103;
    return c2 < c1 ? 2 * UN : UN;
}

cudaError_t launch_base_gemm(int gn, const GemmParams &p, cudaStream_t stream, bool pdl)
{
    switch (gn) {
    case UN: return launch_units<1>(p, stream, pdl);
    case 2 * UN: return launch_units<2>(p, stream, pdl);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t prepare_base_gemm()
{
    cudaError_t e;
    if ((e = prepare_units<1>()) != cudaSuccess) return e;
    return prepare_units<2>();
}

}  // namespace mlora
