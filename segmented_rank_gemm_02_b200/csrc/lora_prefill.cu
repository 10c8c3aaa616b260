// lora_prefill.cu -- long segments (prefill-shaped): TMA + tcgen05 tensor-core tiles.
//
// The computation is the same as the decode family's (page "Multi-LoRA Serving:
// adapter batching", sections "What metadata a segmented kernel needs" and
// "Prefill and decode have different LoRA shapes": a prefill segment holds hundreds
// to thousands of rows, so its two low-rank products are real matrix
// multiplications).  A work tile is (segment, 128 consecutive grouped positions),
// one M=128 tensor-memory tile.
//
// Shrink (long_shrink_kernel).  A thread-block cluster of `ksplit` CTAs owns a tile;
// CTA c covers one part of d_in.  Warp 0 streams the part through an 8-stage ring:
// per 64-column block (two per stage) one TMA tile load of X (128 rows
// x 64 columns, 128-byte swizzle) when the tile's rows are consecutive in X, else
// one four-row TMA gather per lane, plus the adapter's A blocks (one bulk copy)
// (pool layout [8 groups][R][8] is already the tensor core's no-swizzle K-major
// layout).  One thread of warp 1 issues tcgen05.mma (M=128, N=rank bucket, K=16
// each) into an fp32 accumulator in tensor memory as stages land.  The epilogue
// reads the accumulator with tcgen05.ld; the cluster sums its partial tiles through
// distributed shared memory in a fixed order, each CTA a contiguous share written
// to H (fp32) with coalesced stores.
//
// Expand (long_expand_kernel).  Warp-specialised and persistent: the (tile,
// 128-column chunk) pairs of all long tiles are cut into one contiguous range per
// CTA.  A producer warp streams each chunk's B rows (one 4-D TMA load: 128 columns
// x all rank groups of the slot) and Y0 rows (TMA tile, or four-row gathers) into a
// ring of stages; an MMA warp multiplies H_hi B^T + H_lo B^T (M=128, N=128, H read
// from tensor memory) into one of two fp32 accumulators in tensor memory; eight
// epilogue warps (two threads per row) add s * acc to Y0 in shared memory and stage
// the next unit's H as bf16 hi + lo parts in tensor memory (two buffers, written
// with tcgen05.st) ahead of its chunks, which leaves shared memory to the ring (four
// stages at rank 64 instead of three: qkv_prefill 67.7 -> 65.7-66.1 us); a store warp writes full tiles
// of consecutive rows back with TMA stores (the epilogue writes other tiles with
// coalesced 16-byte stores) and releases the stages.  The roles meet only at
// mbarriers, so copies, tensor-core work, epilogue and stores overlap.
//
// Fused projections (mlora_apply_multi): one shrink launch serves up to four
// projections that share X and whose pools hold every slot at the same rank, with
// one A block per projection in each stage and one accumulator per projection in
// tensor memory, so the prefill rows of X are read once; each projection's H goes to
// its own workspace and its own expand follows.
//
// Which segments come here: those of at least 128 grouped positions whose rows are
// consecutive in X and Y (prefill requests); see long_segment().  The shrink is
// launched after the decode-shaped kernel and the expand after the shrink with
// programmatic dependent launch, so each one's launch and set-up overlap the
// kernel before it; the expand's epilogue waits for the shrink before reading H.
//
// Rank buckets: kernels are compiled for the pool's largest bucket and dispatch each
// tile to code for its own bucket (bucket 8 runs as 16; its missing operand half is
// read from a block of zeros).  Every mbarrier wait is bounded; on expiry the kernel
// flags a timeout, stores nothing more, waits again (bounded) for its tensor-core
// work and frees its tensor memory before it leaves.
#include <mutex>

#include "kernels.cuh"
#include "ptx.cuh"

namespace mlora {

namespace {

constexpr int PT = 256;               // threads per CTA: two per tile row
constexpr int PM = kLongTileRows;     // 128 rows per tile
constexpr int KB = 64;                // d_in columns per shrink block (one 128-byte row)
constexpr int NCH = kExpandChunk;     // d_out columns per expand chunk
// shrink pipeline stages: the shrink streams X from HBM with one CTA per SM (what the
// occupancy calculation grants it), so it keeps as many blocks in flight as fit
// (qkv_prefill step 70.8 -> 66.8 us with 8 stages instead of 4)
constexpr int NS = 8;
// 64-column blocks per shrink stage where four stages of two still fit (qkv_prefill
// step 68.3-69.0 -> 67.1-67.6 us): each X row is then read in runs of 256 bytes
constexpr int kShrinkBoxes = 2;
constexpr int kMaxExpandStages = 6;  // expand chunk ring, as deep as shared memory allows
constexpr int kExpandSmemCap = 224 * 1024;   // dynamic shared memory of one expand CTA
constexpr int kMaxSplit = 8;          // CTAs per shrink cluster
constexpr int kZeroBytes = 2048;      // zero operand half for rank bucket 8
constexpr uint64_t kWaitNs = 1000000000ull;

__host__ __device__ constexpr int padded_rank(int r) { return r < 16 ? 16 : r; }

// Shrink of NP projections that share X (one A block per projection per stage, one
// accumulator of RK columns per projection in tensor memory).
template <int RMAX, int NP = 1>
struct ShrinkCfg {
    static constexpr int RK = padded_rank(RMAX);
    static constexpr int X_BOX = PM * KB * 2;            // 16 KB, 128-byte swizzle
    static constexpr int A_BOX = 8 * RK * 16;            // [8][RK][8]
    static constexpr int NBOX = 4 * (2 * X_BOX + NP * 2 * A_BOX) <= 200 * 1024 ? kShrinkBoxes : 1;
    static constexpr int X_STAGE = NBOX * X_BOX;
    static constexpr int A_STAGE = (NBOX * A_BOX + 1023) / 1024 * 1024;
    static constexpr int S_STAGE = X_STAGE + NP * A_STAGE;   // multiple of 1024
    static constexpr int NSTAGE_FIT = (200 * 1024) / S_STAGE;
    static constexpr int NSTAGE = NSTAGE_FIT < NS ? NSTAGE_FIT : NS;
    static constexpr int RED_PITCH = RK + 4;             // floats per row of a partial tile
    static constexpr int S_SMEM = 1024 + NSTAGE * S_STAGE + kZeroBytes;   // + alignment slack
    static_assert(NSTAGE >= 3, "shrink ring");
    static_assert(PM * RED_PITCH * 4 <= NSTAGE * S_STAGE, "partial tile must fit in the ring");
    static constexpr int S_TMEM = NP * RK <= 32 ? 32 : NP * RK <= 64 ? 64 : NP * RK <= 128 ? 128 : 256;
};

template <int RMAX>
struct LongCfg {
    static constexpr int RK = padded_rank(RMAX);
    static constexpr int B_BYTES = (NCH * RK * 2 + 1023) / 1024 * 1024;  // [RK/8][128][8]
    static constexpr int Y_BYTES = PM * NCH * 2;         // two 64-column halves, swizzled
    static constexpr int E_STAGE = B_BYTES + Y_BYTES;    // one 128-column chunk
    static constexpr int E_FIXED = 1024 + kZeroBytes;    // alignment slack + zero block
    static constexpr int E_NB_FIT = (kExpandSmemCap - E_FIXED) / E_STAGE;
    static constexpr int E_NB = E_NB_FIT < kMaxExpandStages ? E_NB_FIT : kMaxExpandStages;
    static_assert(E_NB >= 2, "expand stage ring");
    static constexpr int E_SMEM = E_FIXED + E_NB * E_STAGE;
    // tensor memory: two fp32 accumulators of NCH columns, then two H buffers of RK
    // columns (bf16 hi in the first RK / 2, lo in the next, two values per column)
    static constexpr int H_TCOL = 2 * NCH;
    static constexpr int E_TMEM = H_TCOL + 2 * RK <= 256 ? 256 : 512;
};

struct LongCtl {
    uint64_t bar[NS];   // stage free (its MMAs ended)
    uint64_t full[NS];  // operands of a stage landed
    uint64_t done;      // the tile's accumulator is complete
    uint32_t tmem;
    int scan[PT / 32];
    int tile[5];        // segment, first position, end position, slot, rank from metadata
    float seg_scale;
    int slot_rank;
    float slot_scale;
    int rows[PM];
    int contiguous;     // the tile's rows are consecutive in X / Y
    volatile int fail;
};

__device__ __forceinline__ void report(const TileParams &p, unsigned flag) { atomicOr(p.status, flag); }

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Block-wide scan of the long segments' tile counts; returns the number of tiles
// and leaves tile `want` (if it exists) in ctl.tile.
__device__ int scan_long(const TileParams &p, int want, LongCtl &ctl)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) ctl.tile[0] = -1;
    __syncthreads();
    int running = 0;
    for (int base = 0; base < p.n_segments; base += PT) {
        const int g = base + tid;
        int cnt = 0, p0 = 0, p1 = 0, a = -1, rk = -1;
        float sc = 0.f;
        if (g < p.n_segments) {
            a = p.slots[g];
            p0 = p.offsets[g];
            p1 = p.offsets[g + 1];
            if (p.ranks) rk = p.ranks[g];
            if (p.scales) sc = p.scales[g];
            // malformed segments are reported by the decode-shaped kernel's scan
            if (a >= 0 && a < p.n_slots && p0 >= 0 && p1 >= p0 && p1 <= p.n_tokens &&
                long_segment(p, p0, p1))
                cnt = (p1 - p0 + PM - 1) / PM;
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
        for (int w = 0; w < PT / 32; ++w) {
            const int v = ctl.scan[w];
            before += (w < warp) ? v : 0;
            total += v;
        }
        incl += before;
        const int lo = running + incl - cnt;
        if (cnt > 0 && want >= lo && want < running + incl) {
            ctl.tile[0] = g;
            ctl.tile[1] = p0 + (want - lo) * PM;
            ctl.tile[2] = p1;
            ctl.tile[3] = a;
            ctl.tile[4] = rk;
            ctl.seg_scale = sc;
        }
        running += total;
        __syncthreads();
    }
    return running;
}

// Rows of the current tile, whether they are consecutive, the slot's rank and scale;
// returns the rank bucket to run (0 if the tile must be skipped) and sets ok.
__device__ int tile_setup(const TileParams &p, LongCtl &ctl, int nvalid, bool reporter, bool &ok,
                          int &rank)
{
    const int tid = threadIdx.x;
    const int p0 = ctl.tile[1], slot = ctl.tile[3], r_meta = ctl.tile[4];
    int t = -1;
    if (tid < PM && tid < nvalid) {
        t = p.token_indices ? p.token_indices[p0 + tid] : p0 + tid;
        if (t < 0 || t >= p.n_rows) {
            if (reporter) report(p, kFlagBadRow);
            t = -1;
        }
    }
    if (tid < PM) ctl.rows[tid] = t;
    if (tid == 0) {
        ctl.slot_rank = p.slot_rank[slot];
        ctl.slot_scale = p.slot_scale[slot];
        // a batch built for an earlier generation of the slot: rank -1 marks it stale
        if (p.generations && p.slot_gen[slot] != p.generations[ctl.tile[0]]) ctl.slot_rank = -1;
    }
    __syncthreads();
    // consecutive rows, all present: one TMA tile covers the tile's X / Y rows
    const bool mine = tid >= PM || tid >= nvalid ||
                      (ctl.rows[tid] >= 0 && ctl.rows[tid] == ctl.rows[0] + tid);
    const int contiguous = __syncthreads_and(mine ? 1 : 0);
    if (tid == 0) ctl.contiguous = contiguous;
    __syncthreads();
    const int r = ctl.slot_rank;
    ok = r > 0 && (p.ranks == nullptr || r_meta == r) && rank_bucket(r) != 0;
    if (reporter && tid == 0 && !ok)
        report(p, r < 0 ? kFlagStaleSlot : r == 0 ? kFlagSlotEmpty : kFlagBadRank);
    rank = ok ? r : 0;
    return ok ? rank_bucket(r) : 0;
}

__device__ __forceinline__ bool wait_or_fail(const TileParams &p, LongCtl &ctl, uint64_t *bar,
                                             uint32_t parity)
{
    if (ctl.fail) return false;
    if (!mbar_wait_bounded(bar, parity, kWaitNs)) {
        ctl.fail = 1;
        report(p, kFlagTimeout);
        return false;
    }
    return true;
}

// ------------------------------------------------------------------ shrink
// One tile per cluster iteration.  Warp 0 streams this CTA's part of d_in (X rows by
// TMA tile or lane-parallel four-row gathers, the adapter's A block by one bulk copy
// per 64-column block) through an NS-stage ring; lane 0 of warp 1 issues the
// tensor-core work as stages land and frees each stage with tcgen05.commit.  Then
// the CTA's partial tile goes from tensor memory to shared memory, and the cluster
// sums its partials through distributed shared memory, each CTA one contiguous
// share of the tile, written to H with coalesced 16-byte stores.
// Projection j of a shrink launch: j = 0 is the launch's own pool and H workspace,
// j >= 1 the further projections of a fused launch (same X, same slot numbering).
__device__ __forceinline__ const __nv_bfloat16 *proj_slot_a(const TileParams &p, int j, int slot)
{
    return j == 0 ? p.pool + (int64_t)slot * p.slot_stride : p.proj[j].pool + (int64_t)slot * p.proj[j].slot_stride;
}

// RAGGED: d_in is not a multiple of 64 (its last block is partial); a separate
// instantiation, so that the common case runs the same instructions as without it.
template <int RMAX, int R, int NP, bool RAGGED>
__device__ void shrink_tile(const TileParams &p, LongCtl &ctl, uint8_t *ring, uint8_t *zero,
                            uint32_t tmem, uint32_t &gb, uint32_t &tc, uint32_t crank, uint32_t csize,
                            int nvalid, int rank, bool ok)
{
    using C = ShrinkCfg<RMAX, NP>;
    constexpr int NSTAGE = C::NSTAGE;
    constexpr int RK = padded_rank(R);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int p0 = ctl.tile[1], slot = ctl.tile[3];
    const int k0 = min(p.d_in, (int)crank * p.k_part);
    const int k1 = min(p.d_in, k0 + p.k_part);
    const int nkb = (k1 - k0 + KB - 1) / KB;            // 64-column blocks
    constexpr bool ragged = RAGGED;
    constexpr int NBOX = C::NBOX;
    const int nst = (nkb + NBOX - 1) / NBOX;             // stages

    if (warp == 0) {
        // ---- copies: X block (tile or gathers) + one A block per projection per stage
        const bool contiguous = ctl.contiguous != 0;
        int r[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int t = ctl.rows[4 * lane + q];
            r[q] = t >= 0 ? t : p.n_rows;   // absent rows read as zeros
        }
        for (int b = 0; b < nst; ++b) {
            const uint32_t G = gb + b;
            const int s = (int)(G % NSTAGE);
            bool go = true;
            if (lane == 0 && G >= (uint32_t)NSTAGE)
                go = wait_or_fail(p, ctl, &ctl.bar[s], ((G / NSTAGE) - 1) & 1u);
            if (__shfl_sync(0xffffffffu, go ? 1 : 0, 0) == 0) break;
            uint8_t *xs = ring + s * C::S_STAGE;
            uint8_t *as = xs + C::X_STAGE;
            const int kb0 = k0 + b * NBOX * KB;
            const int nb = min(NBOX, nkb - b * NBOX);   // blocks in this stage
            // A bytes of the stage: fewer than nb blocks' only in the last block of a d_in
            // that is not a multiple of 64 (the X copies read zeros past d_in)
            uint32_t a_bytes = (uint32_t)nb * R * 128;
            const int valid = ragged ? min(k1, kb0 + nb * KB) - kb0 : nb * KB;
            if (ragged) a_bytes = (uint32_t)(valid / 8) * R * 16;
            if (ragged && valid % 16 != 0) {
                // the last K=16 step reads one 8-column group past d_in: zero it (X is
                // zero there too, and stale shared memory may hold any bits)
                for (int j = 0; j < NP; ++j)
                    for (int o = lane * 16; o < R * 16; o += 32 * 16)
                        *reinterpret_cast<uint4 *>(as + j * C::A_STAGE + a_bytes + o) = make_uint4(0, 0, 0, 0);
                fence_proxy_async_smem();   // read by the tensor core
                __syncwarp();
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(&ctl.full[s], (uint32_t)nb * C::X_BOX + NP * a_bytes);
                // the blocks of a stage go out back to back
                if (contiguous)
                    for (int i = 0; i < nb; ++i)
                        tma_load_2d(xs + i * C::X_BOX, &p.x_tile, kb0 + i * KB, ctl.rows[0], &ctl.full[s]);
#pragma unroll
                for (int j = 0; j < NP; ++j)
                    bulk_load(as + j * C::A_STAGE, proj_slot_a(p, j, slot) + (int64_t)(kb0 / 8) * R * 8, a_bytes,
                              &ctl.full[s]);
            }
            __syncwarp();
            if (!contiguous)
                for (int i = 0; i < nb; ++i)
                    tma_gather4(xs + i * C::X_BOX + lane * 4 * 128, &p.x_rows, kb0 + i * KB, r[0], r[1], r[2], r[3],
                                &ctl.full[s]);
        }
    } else if (warp == 1 && lane == 0) {
        // ---- tensor core: 4 K=16 steps per block into one fp32 accumulator per projection
        const uint32_t idesc = umma_idesc_bf16(PM, RK);
        for (int b = 0; b < nst; ++b) {
            const uint32_t G = gb + b;
            const int s = (int)(G % NSTAGE);
            if (!wait_or_fail(p, ctl, &ctl.full[s], (G / NSTAGE) & 1u)) break;
            tc_fence_after();
            const uint32_t xs = smem_addr(ring + s * C::S_STAGE);
            const uint32_t as = xs + C::X_STAGE;
            const int nb = min(NBOX, nkb - b * NBOX);
            const int valid = ragged ? min(k1, k0 + b * NBOX * KB + nb * KB) - (k0 + b * NBOX * KB) : nb * KB;
            // one K=16 step of block i for every projection
            auto step = [&](int i, int st) {
                const uint64_t ad = umma_desc_sw128(xs + i * C::X_BOX + st * 32);
#pragma unroll
                for (int j = 0; j < NP; ++j) {
                    const uint32_t a0 = as + j * C::A_STAGE + (i * (KB / 16) + st) * 2 * R * 16;
                    // adapter rows 8 .. 15 of bucket 8 come from the zero block
                    const uint32_t sbo = (R == 8) ? smem_addr(zero) - a0 : 128;
                    const uint64_t bd = umma_desc_kmajor(a0, R * 16, sbo);
                    umma_bf16(tmem + (uint32_t)(j * RK), ad, bd, idesc, (b > 0 || i > 0 || st > 0) ? 1u : 0u);
                }
            };
            if (valid == nb * KB) {
                for (int i = 0; i < nb; ++i) {
#pragma unroll
                    for (int st = 0; st < KB / 16; ++st) step(i, st);
                }
            } else {   // the last block of d_in: steps up to d_in only
                for (int i = 0; i < nb; ++i)
                    for (int st = 0; st < KB / 16 && i * KB + st * 16 < valid; ++st) step(i, st);
            }
            umma_commit(&ctl.bar[s]);   // stage s is free once these MMAs end
        }
        umma_commit(&ctl.done);         // the partial tiles are complete
    }
    gb += nst;
    // the other threads (and lanes 1..31 of warp 1) wait here, at a hardware barrier,
    // instead of spinning beside the copy and MMA loops
    __syncthreads();
    // everyone: the accumulators are final (bounded wait; a timeout leaves zeros)
    // (warp-uniform: tcgen05.ld below is a warp-wide instruction)
    const bool acc_ok = __all_sync(0xffffffffu, wait_or_fail(p, ctl, &ctl.done, tc & 1u));
    ++tc;
    tc_fence_after();

    for (int j = 0; j < NP; ++j) {
        // projection j: its pool must hold the slot at the same rank (a pool that does
        // not is rejected by that projection's expand, which reads its own slot table)
        bool ok_j = ok;
        if (j > 0 && ok_j) ok_j = p.proj[j].slot_rank[slot] == rank;
        float *ws = j == 0 ? p.ws : p.proj[j].ws;
        const int64_t ws_ld = j == 0 ? p.ws_ld : p.proj[j].ws_ld;
        // this CTA's partial tile from tensor memory: warp w holds rows 32 (w % 4) .. +31
        // and columns [(w / 4) * RK/2, +RK/2) of projection j's accumulator
        constexpr int HC = RK / 2;
        float h[HC];
        const int col0 = (warp / 4) * HC;
        if (nkb > 0 && acc_ok) {
            const uint32_t taddr = tmem + ((uint32_t)(32 * (warp % 4)) << 16) + (uint32_t)(j * RK) + col0;
            if constexpr (HC == 8) {
                uint32_t v0[8];
                tmem_ld8(taddr, v0);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 8; ++c) h[c] = __uint_as_float(v0[c]);
            } else if constexpr (HC == 16) {
                uint32_t v0[8], v1[8];
                tmem_ld8(taddr, v0);
                tmem_ld8(taddr + 8, v1);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    h[c] = __uint_as_float(v0[c]);
                    h[8 + c] = __uint_as_float(v1[c]);
                }
            } else {
                uint32_t v[32];
                tmem_ld32(taddr, v);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) h[c] = __uint_as_float(v[c]);
            }
        } else {
#pragma unroll
            for (int c = 0; c < HC; ++c) h[c] = 0.f;
        }
        // every block of this tile has been consumed, so the ring holds the partial tile
        float *red = reinterpret_cast<float *>(ring);
        const int trow = 32 * (warp % 4) + (tid & 31);
#pragma unroll
        for (int c = 0; c < HC; c += 4)
            *reinterpret_cast<float4 *>(red + trow * C::RED_PITCH + col0 + c) =
                make_float4(h[c], h[c + 1], h[c + 2], h[c + 3]);
        tc_fence_before();
        cluster_arrive_release();
        cluster_wait_acquire();
        // CTA crank sums the cluster's partials (in CTA order) for its share of the tile's
        // float4 slots, row-major, and writes them to H: consecutive threads write
        // consecutive columns of a row
        if (ok_j && !ctl.fail) {
            constexpr int F4 = RK / 4;                       // float4 slots per row
            const int total = PM * F4;
            const int per = (total + (int)csize - 1) / (int)csize;
            const int f_lo = (int)crank * per, f_hi = min(total, f_lo + per);
            for (int f = f_lo + tid; f < f_hi; f += PT) {
                const int row = f / F4, c4 = f % F4;
                if (row >= nvalid || ctl.rows[row] < 0 || 4 * c4 >= rank) continue;
                const uint32_t addr = smem_addr(red + row * C::RED_PITCH + 4 * c4);
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (uint32_t c = 0; c < csize; ++c) {
                    const float4 v = ld_dsmem_f32x4(map_to_rank(addr, c));
                    acc.x += v.x;
                    acc.y += v.y;
                    acc.z += v.z;
                    acc.w += v.w;
                }
                float *dst = ws + (int64_t)(p0 + row) * ws_ld + 4 * c4;
                if (4 * c4 + 4 <= rank) {
                    *reinterpret_cast<float4 *>(dst) = acc;
                } else {   // columns >= rank are left alone
                    const int n = rank - 4 * c4;
                    dst[0] = acc.x;
                    if (n > 1) dst[1] = acc.y;
                    if (n > 2) dst[2] = acc.z;
                }
            }
        }
        // peers are done reading this CTA's partial tile before it is overwritten (next
        // projection) or the ring is refilled
        cluster_arrive_release();
        cluster_wait_acquire();
    }
    fence_proxy_async_smem();   // the ring is next written by TMA
    __syncthreads();
    tc_fence_after();
}

template <int RMAX, int NP, bool RAGGED>
__global__ void __launch_bounds__(PT) long_shrink_kernel(const __grid_constant__ TileParams p)
{
    using C = ShrinkCfg<RMAX, NP>;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ LongCtl ctl;
    uint8_t *ring = align1024(smem_raw);
    uint8_t *zero = ring + C::NSTAGE * C::S_STAGE;
    const int tid = threadIdx.x, warp = tid >> 5;
    const uint32_t crank = cluster_rank(), csize = cluster_size();
    const int n_clusters = (int)(gridDim.x / csize);
    // the expand kernel may start its CTAs now, on SMs this grid leaves free
    griddep_launch_dependents();
    if (warp == 0) {
        tmem_alloc(&ctl.tmem, C::S_TMEM);
        tmem_relinquish();
    }
    for (int i = tid; i < kZeroBytes / 16; i += PT) reinterpret_cast<uint4 *>(zero)[i] = make_uint4(0, 0, 0, 0);
    if (tid == 0) {
#pragma unroll
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(&ctl.bar[s], 1);
            mbar_init(&ctl.full[s], 1);
        }
        mbar_init(&ctl.done, 1);
        fence_mbar_init();
        ctl.fail = 0;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem;
    uint32_t gb = 0, tc = 0;
    // every CTA of a cluster reads the same metadata and takes the same tiles
    for (int tile = (int)cluster_index();; tile += n_clusters) {
        const int ntiles = scan_long(p, tile, ctl);
        if (tile >= ntiles) break;
        const int nvalid = min(PM, ctl.tile[2] - ctl.tile[1]);
        bool ok;
        int rank;
        const int R = tile_setup(p, ctl, nvalid, crank == 0, ok, rank);
        if (R == 8) {
            shrink_tile<RMAX, 8, NP, RAGGED>(p, ctl, ring, zero, tmem, gb, tc, crank, csize, nvalid, rank, ok);
        } else if (R == 16) {
            shrink_tile<RMAX, 16, NP, RAGGED>(p, ctl, ring, zero, tmem, gb, tc, crank, csize, nvalid, rank, ok);
        } else if (R == 32) {
            if constexpr (RMAX >= 32)
                shrink_tile<RMAX, 32, NP, RAGGED>(p, ctl, ring, zero, tmem, gb, tc, crank, csize, nvalid, rank, ok);
        } else if (R == 64) {
            if constexpr (RMAX >= 64)
                shrink_tile<RMAX, 64, NP, RAGGED>(p, ctl, ring, zero, tmem, gb, tc, crank, csize, nvalid, rank, ok);
        }
        __syncthreads();
    }
    // Nothing here reads what the decode-shaped kernel before us writes (other rows of
    // Y and H), so the wait for it comes only now: this grid ends after it.
    griddep_wait();
    // leave: tensor-core work done, tensor memory freed
    if (ctl.fail && tid == 0) {
        // let copies still in flight land before shared memory is released
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 2000000ull) {
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, C::S_TMEM);
}

// ------------------------------------------------------------------ expand
// Warp roles.  Warp 0 copies (one lane issues the B-row bulk copies and Y0 tile
// loads; every lane issues its own four-row gathers), warp 1 owns tensor memory and
// issues the tensor-core work, warps 2..9 stage H and run the epilogue (two threads
// per tile row, one 64-column half each), warp 10 writes finished chunks of full
// tiles back with TMA stores and releases the stages.  The roles meet only at
// mbarriers:
//   full[s] / empty[s]      stage ring (B rows + Y0 rows of one 128-column chunk)
//   res[s]                  the epilogue is done with stage s (results in place)
//   acc_full[a] / acc_empty[a]  two fp32 accumulators of 128 columns in tensor memory
//   h_full[b] / h_empty[b]  two H buffers (hi + lo, tensor memory), one per work unit in flight
constexpr int E_WARPS = 11;
constexpr int ET = E_WARPS * 32;     // threads per expand CTA
constexpr int E_EPI = 256;           // epilogue threads (warps 2..9)
constexpr int kEpiBar = 1;           // named barrier of the epilogue warps
constexpr int kMaxUnits = 64;        // work units per CTA (the host sizes the grid)

struct ExpUnit {
    int seg;           // segment of the tile
    int p0, p1;        // first grouped position of the tile, end of its segment
    int slot, r_meta;  // slot and rank from the metadata (-1 if none)
    float seg_scale;   // scale from the metadata
    int c_begin, c_end;   // 128-column chunks [c_begin, c_end) of d_out
    int full, row0;       // set when staged: 128 consecutive rows from row0
};

struct ExpCtl {
    uint64_t full[kMaxExpandStages], empty[kMaxExpandStages], res[kMaxExpandStages];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t h_full[2], h_empty[2];
    uint32_t tmem;
    volatile int fail;
    int scan[E_WARPS];
    int rows[2][PM];   // original row of each tile position (epilogue), -1 = none
    ExpUnit unit[kMaxUnits];
};

// Rank and scale of a unit's slot; every role derives the same values.
struct UnitInfo {
    int nvalid, R, rank, ok, n_lo, n_hi, nch;
    int slot_rank;   // as read (-1 if the segment's generation is stale)
    float scale;
};

__device__ __forceinline__ UnitInfo unit_info(const TileParams &p, const ExpUnit &u)
{
    UnitInfo i;
    i.nvalid = min(PM, u.p1 - u.p0);
    int r = p.slot_rank[u.slot];
    // a batch built for an earlier generation of the slot: rank -1 marks it stale
    if (p.generations && p.slot_gen[u.slot] != p.generations[u.seg]) r = -1;
    i.slot_rank = r;
    i.ok = r > 0 && (p.ranks == nullptr || u.r_meta == r) && rank_bucket(r) != 0;
    i.rank = i.ok ? r : 0;
    i.R = i.ok ? rank_bucket(r) : 8;
    i.scale = p.scales ? u.seg_scale : p.slot_scale[u.slot];
    i.n_lo = u.c_begin * NCH;
    i.n_hi = min(p.d_out, u.c_end * NCH);
    i.nch = u.c_end - u.c_begin;
    return i;
}

__device__ __forceinline__ bool exp_wait(const TileParams &p, ExpCtl &ctl, uint64_t *bar, uint32_t parity)
{
    if (ctl.fail) return false;
    if (!mbar_wait_bounded(bar, parity, kWaitNs)) {
        ctl.fail = 1;
        report(p, kFlagTimeout);
        return false;
    }
    return true;
}

// One thread's part of a tile row of H for the expand: HC columns of H (the first
// ncols read from src, the rest zero) as bf16 hi + lo parts, two per 32-bit column, to
// tensor memory at columns hi_col .. and lo_col .. of the thread's lane.  The row's
// loads all go out before any is used.
template <int HC>
__device__ __forceinline__ void stage_h_tmem(const float *src, int ncols, uint32_t hi_col, uint32_t lo_col)
{
    float h[HC];
#pragma unroll
    for (int c = 0; c < HC; c += 4) {
        if (c + 4 <= ncols) {
            const float4 v = *reinterpret_cast<const float4 *>(src + c);
            h[c] = v.x;
            h[c + 1] = v.y;
            h[c + 2] = v.z;
            h[c + 3] = v.w;
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) h[c + e] = c + e < ncols ? src[c + e] : 0.f;
        }
    }
#pragma unroll
    for (int c = 0; c < HC; c += 8) {
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float h0, l0, h1, l1;
            split_bf16(h[c + 2 * e], h0, l0);
            split_bf16(h[c + 2 * e + 1], h1, l1);
            hw[e] = pack_bf16x2(h0, h1);
            lw[e] = pack_bf16x2(l0, l1);
        }
        tmem_st4(hi_col + c / 2, hw);
        tmem_st4(lo_col + c / 2, lw);
    }
}

// Work split.  The (tile, 128-column chunk) pairs of all long tiles, tile-major, are
// cut into gridDim.x equal contiguous ranges; CTA b takes range b.  A unit is the run
// of one tile's chunks inside the range, so a CTA stages H once per tile it touches.
//
// Pass over the segments: with want_lo < 0 it only counts the long tiles; otherwise it
// also fills ctl.unit[t - want_lo] for every tile t in [want_lo, want_hi].
__device__ int scan_units(const TileParams &p, ExpCtl &ctl, int want_lo, int want_hi)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int running = 0;
    for (int base = 0; base < p.n_segments; base += ET) {
        const int g = base + tid;
        int cnt = 0, p0 = 0, p1 = 0, a = -1, rk = -1;
        float sc = 0.f;
        if (g < p.n_segments) {
            a = p.slots[g];
            p0 = p.offsets[g];
            p1 = p.offsets[g + 1];
            if (want_lo >= 0) {
                if (p.ranks) rk = p.ranks[g];
                if (p.scales) sc = p.scales[g];
            }
            if (a >= 0 && a < p.n_slots && p0 >= 0 && p1 >= p0 && p1 <= p.n_tokens &&
                long_segment(p, p0, p1))
                cnt = (p1 - p0 + PM - 1) / PM;
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
        for (int w = 0; w < E_WARPS; ++w) {
            const int v = ctl.scan[w];
            before += (w < warp) ? v : 0;
            total += v;
        }
        if (want_lo >= 0 && cnt > 0) {
            const int lo = running + before + incl - cnt;   // this segment's first tile
            const int t0 = max(lo, want_lo), t1 = min(lo + cnt - 1, want_hi);
            for (int t = t0; t <= t1; ++t) {
                ExpUnit &e = ctl.unit[t - want_lo];
                e.seg = g;
                e.p0 = p0 + (t - lo) * PM;
                e.p1 = p1;
                e.slot = a;
                e.r_meta = rk;
                e.seg_scale = sc;
            }
        }
        running += total;
        __syncthreads();
    }
    return running;
}

template <int RMAX, int MODE>
__global__ void __launch_bounds__(ET, 1) long_expand_kernel(const __grid_constant__ TileParams p)
{
    using C = LongCfg<RMAX>;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ ExpCtl ctl;
    uint8_t *stages = align1024(smem_raw);
    uint8_t *zero = stages + C::E_NB * C::E_STAGE;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (warp == 1) {
        tmem_alloc(&ctl.tmem, C::E_TMEM);
        tmem_relinquish();
    }
    for (int i = tid; i < kZeroBytes / 16; i += ET) reinterpret_cast<uint4 *>(zero)[i] = make_uint4(0, 0, 0, 0);
    if (tid == 0) {
        for (int s = 0; s < C::E_NB; ++s) {
            mbar_init(&ctl.full[s], 1);
            mbar_init(&ctl.empty[s], 1);
            mbar_init(&ctl.res[s], E_EPI / 32);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl.acc_full[b], 1);
            mbar_init(&ctl.acc_empty[b], E_EPI / 32);
            mbar_init(&ctl.h_full[b], 1);
            mbar_init(&ctl.h_empty[b], 1);
        }
        fence_mbar_init();
        ctl.fail = 0;
    }
    // this CTA's share of the (tile, chunk) pairs
    const int cpt = (p.d_out + NCH - 1) / NCH;   // chunks per tile
    const int ntiles = scan_units(p, ctl, -1, -1);
    const int64_t total = (int64_t)ntiles * cpt;
    const int64_t lo = total * blockIdx.x / gridDim.x, hi = total * (blockIdx.x + 1) / gridDim.x;
    int n_my = 0;
    if (hi > lo) {
        const int t_lo = (int)(lo / cpt), t_hi = (int)((hi - 1) / cpt);
        n_my = t_hi - t_lo + 1;
        if (n_my > kMaxUnits) {   // the host sizes the grid so that this never happens
            if (tid == 0) report(p, kFlagTimeout);
            n_my = 0;
        } else {
            scan_units(p, ctl, t_lo, t_hi);
            for (int k = tid; k < n_my; k += ET) {
                const int64_t t = t_lo + k;
                ctl.unit[k].c_begin = (int)((lo > t * cpt ? lo : t * cpt) - t * cpt);
                ctl.unit[k].c_end = (int)((hi < (t + 1) * cpt ? hi : (t + 1) * cpt) - t * cpt);
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem;

    if (warp == 0) {
        // ---------------------------------------------------------------- copies
        uint32_t g = 0;
        for (int k = 0; k < n_my; ++k) {
            if (__shfl_sync(0xffffffffu, ctl.fail, 0)) break;
            const ExpUnit u = ctl.unit[k];
            const UnitInfo ui = unit_info(p, u);
            // this lane's four rows of the tile: gathers and the contiguity test
            int t[4];
            bool mine = true;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int i = 4 * lane + q;
                t[q] = -1;
                if (i < ui.nvalid) {
                    const int v = p.token_indices ? p.token_indices[u.p0 + i] : u.p0 + i;
                    t[q] = (v >= 0 && v < p.n_rows) ? v : -1;
                }
            }
            const int row0 = __shfl_sync(0xffffffffu, t[0], 0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int i = 4 * lane + q;
                if (i < ui.nvalid) mine = mine && t[q] >= 0 && t[q] == row0 + i;
            }
            const bool contiguous = __all_sync(0xffffffffu, mine);
            for (int ci = 0; ci < ui.nch; ++ci, ++g) {
                const int s = (int)(g % C::E_NB);
                bool go = true;
                if (lane == 0 && g >= (uint32_t)C::E_NB)
                    go = exp_wait(p, ctl, &ctl.empty[s], ((g / C::E_NB) - 1) & 1u);
                go = __shfl_sync(0xffffffffu, go ? 1 : 0, 0) != 0;
                if (!go) break;
                uint8_t *bs = stages + s * C::E_STAGE;
                uint8_t *ys = bs + C::B_BYTES;
                const int c0 = ui.n_lo + ci * NCH;
                const int len = min(NCH, ui.n_hi - c0);
                const int halves = len > 64 ? 2 : 1;
                if (lane == 0) {
                    // B: one box of 128 columns x all rank groups (columns past d_out read
                    // as zeros); Y0: one or two 64-column halves of the tile's rows
                    uint32_t bytes = (uint32_t)ui.R * NCH * 2;
                    if (ui.ok) bytes += (uint32_t)halves * PM * 64 * 2;
                    mbar_arrive_expect_tx(&ctl.full[s], bytes);
                    const int bi = ui.R == 8 ? 0 : ui.R == 16 ? 1 : ui.R == 32 ? 2 : 3;
                    tma_load_4d(bs, &p.b_map[bi], 0, c0 / p.b_col_div, 0, u.slot, &ctl.full[s]);
                    if (ui.ok && contiguous)
                        for (int h = 0; h < halves; ++h)
                            tma_load_2d(ys + h * PM * 128, &p.y_tile, c0 + 64 * h, row0, &ctl.full[s]);
                }
                __syncwarp();
                if (ui.ok && !contiguous) {
                    int r[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) r[q] = t[q] >= 0 ? t[q] : p.n_rows;   // absent: zeros
                    for (int h = 0; h < halves; ++h)
                        tma_gather4(ys + h * PM * 128 + lane * 4 * 128, &p.y_rows, c0 + 64 * h, r[0], r[1],
                                    r[2], r[3], &ctl.full[s]);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- tensor core
        if (lane == 0) {
            uint32_t g = 0, a = 0;
            const uint32_t idesc = umma_idesc_bf16(PM, NCH);
            for (int k = 0; k < n_my && !ctl.fail; ++k) {
                const UnitInfo ui = unit_info(p, ctl.unit[k]);
                const int hb = k & 1;
                if (!exp_wait(p, ctl, &ctl.h_full[hb], (uint32_t)(k >> 1) & 1u)) break;
                const uint32_t a_hi = tmem + (uint32_t)(C::H_TCOL + hb * C::RK);
                const uint32_t a_lo = a_hi + C::RK / 2;
                const int RK = padded_rank(ui.R);
                for (int ci = 0; ci < ui.nch; ++ci, ++g, ++a) {
                    const int s = (int)(g % C::E_NB);
                    const int ab = (int)(a & 1);
                    if (!exp_wait(p, ctl, &ctl.full[s], (g / C::E_NB) & 1u)) break;
                    if (a >= 2 && !exp_wait(p, ctl, &ctl.acc_empty[ab], ((a >> 1) - 1) & 1u)) break;
                    tc_fence_after();
                    const uint32_t b_s = smem_addr(stages + s * C::E_STAGE);
                    const uint32_t d = tmem + ab * NCH;
                    for (int st = 0; st < RK / 16; ++st) {
                        const uint32_t b0 = b_s + st * 2 * NCH * 16;
                        // bucket 8: the second rank group of B is the zero block
                        const uint32_t lbo = (ui.R == 8) ? smem_addr(zero) - b0 : NCH * 16;
                        const uint64_t bd = umma_desc_kmajor(b0, lbo, 128);
                        // H from tensor memory: 16 ranks = 8 columns per step
                        umma_bf16_tmem_a(d, a_hi + st * 8, bd, idesc, st > 0 ? 1u : 0u);
                        umma_bf16_tmem_a(d, a_lo + st * 8, bd, idesc, 1u);
                    }
                    umma_commit(&ctl.acc_full[ab]);
                }
                umma_commit(&ctl.h_empty[hb]);   // this unit's H buffer is free once its MMAs end
            }
        }
        __syncwarp();
    } else if (warp < 2 + E_EPI / 32) {
        // ---------------------------------------------------------------- H staging + epilogue
        const int et = tid - 64;
        const int quarter = warp & 3, half = (warp - 2) >> 2;
        const int row = 32 * quarter + lane;                 // tensor-memory lane = tile row
        // Every wait of the epilogue warps ends in a vote, so they all leave together
        // (a named barrier has no time limit).
        auto wait_all = [&](uint64_t *bar, uint32_t parity) -> bool {
            const bool ok = exp_wait(p, ctl, bar, parity);
            return named_sync_and(kEpiBar, E_EPI, ok);
        };
        // Stage unit k: its rows, whether they form one full run, and H as bf16 hi + lo
        // in buffer k & 1 (free once unit k - 2's tensor-core work has ended).
        auto stage = [&](int k) -> bool {
            const ExpUnit u = ctl.unit[k];
            const UnitInfo ui = unit_info(p, u);
            const int hb = k & 1;
            int t = -1;
            if (row < ui.nvalid) {
                const int v = p.token_indices ? p.token_indices[u.p0 + row] : u.p0 + row;
                if (v >= 0 && v < p.n_rows) t = v;
                else if (MODE == MODE_EXPAND && u.c_begin == 0 && half == 0) report(p, kFlagBadRow);
            }
            if (MODE == MODE_EXPAND && u.c_begin == 0 && et == 0 && !ui.ok)
                report(p, ui.slot_rank < 0 ? kFlagStaleSlot : ui.slot_rank == 0 ? kFlagSlotEmpty : kFlagBadRank);
            if (k >= 2 && !wait_all(&ctl.h_empty[hb], (uint32_t)((k >> 1) - 1) & 1u)) return false;
            tc_fence_after();   // the tensor core's reads of buffer hb came before these writes
            if (half == 0) ctl.rows[hb][row] = t;
            const int RK = padded_rank(ui.R);
            const int HC = RK / 2;                            // H columns of this thread
            const bool hrow = ui.ok && row < ui.nvalid;
            const float *hsrc = p.ws + (int64_t)(u.p0 + (hrow ? row : 0)) * p.ws_ld + half * HC;
            const int ncols = hrow ? min(HC, max(0, ui.rank - half * HC)) : 0;
            // this thread's row of buffer hb: hi at column half * HC / 2, lo RK_max / 2 on
            const uint32_t tcol = tmem + ((uint32_t)(32 * quarter) << 16) +
                                  (uint32_t)(C::H_TCOL + hb * C::RK + half * HC / 2);
            if (HC == 8) stage_h_tmem<8>(hsrc, ncols, tcol, tcol + C::RK / 2);
            if constexpr (RMAX >= 32)
                if (HC == 16) stage_h_tmem<16>(hsrc, ncols, tcol, tcol + C::RK / 2);
            if constexpr (RMAX >= 64)
                if (HC == 32) stage_h_tmem<32>(hsrc, ncols, tcol, tcol + C::RK / 2);
            tmem_wait_st();
            tc_fence_before();   // the H tile is read by the tensor core
            named_sync(kEpiBar, E_EPI);
            const bool run = named_sync_and(kEpiBar, E_EPI, ui.nvalid == PM && ctl.rows[hb][row] >= 0 &&
                                                                ctl.rows[hb][row] == ctl.rows[hb][0] + row);
            if (et == 0) {
                ctl.unit[k].full = run ? 1 : 0;
                ctl.unit[k].row0 = ctl.rows[hb][0];
                mbar_arrive(&ctl.h_full[hb]);
            }
            // every epilogue thread reads the run flag (right away when the CTA has one unit)
            named_sync(kEpiBar, E_EPI);
            return true;
        };

        uint32_t g = 0, a = 0;
        // H comes from the shrink kernel launched just before this one
        griddep_wait();
        bool alive = n_my > 0 ? stage(0) : false;
        for (int k = 0; k < n_my && alive; ++k) {
            // the next unit's H is staged before this unit's chunks, so the tensor core
            // never waits for it
            if (k + 1 < n_my && !stage(k + 1)) break;
            const ExpUnit u = ctl.unit[k];
            const UnitInfo ui = unit_info(p, u);
            const int hb = k & 1;
            const bool full_tile = ctl.unit[k].full != 0;
            const bool compute = ui.ok && row < ui.nvalid && ctl.rows[hb][row] >= 0;

            for (int ci = 0; ci < ui.nch; ++ci, ++g, ++a) {
                const int s = (int)(g % C::E_NB);
                const int ab = (int)(a & 1);
                const int c0 = ui.n_lo + ci * NCH;
                const int len = min(NCH, ui.n_hi - c0);
                uint8_t *ys = stages + s * C::E_STAGE + C::B_BYTES;
                if (!wait_all(&ctl.acc_full[ab], (a >> 1) & 1u) || !wait_all(&ctl.full[s], (g / C::E_NB) & 1u)) {
                    alive = false;
                    break;
                }
                tc_fence_after();
                constexpr int CT = NCH / 2;                  // columns per thread
                const uint32_t taddr = tmem + ((uint32_t)(32 * quarter) << 16) + ab * NCH + CT * half;
                uint32_t v0[32], v1[32];
                tmem_ld32(taddr, v0);
                if constexpr (CT == 64) tmem_ld32(taddr + 32, v1);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl.acc_empty[ab]);
                if (compute && CT * half < len) {
                    // this thread's columns [CT * half, +CT): 64-column swizzled block and
                    // first 16-byte chunk inside its 128-byte row
                    const int blk = (CT * half) / 64, q0 = ((CT * half) % 64) / 8;
                    uint8_t *yh = ys + blk * PM * 128 + row * 128;
#pragma unroll
                    for (int q = 0; q < CT / 8; ++q) {
                        uint4 *yp = reinterpret_cast<uint4 *>(yh + (((q0 + q) ^ (row & 7)) * 16));
                        const uint4 y0 = *yp;
                        const __nv_bfloat162 *y2 = reinterpret_cast<const __nv_bfloat162 *>(&y0);
                        uint4 out;
                        uint32_t *o = reinterpret_cast<uint32_t *>(&out);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = __bfloat1622float2(y2[e]);
                            const uint32_t a0 = q < 4 ? v0[8 * q + 2 * e] : v1[8 * (q - 4) + 2 * e];
                            const uint32_t a1 = q < 4 ? v0[8 * q + 2 * e + 1] : v1[8 * (q - 4) + 2 * e + 1];
                            o[e] = pack_bf16x2(fmaf(ui.scale, __uint_as_float(a0), f.x),
                                               fmaf(ui.scale, __uint_as_float(a1), f.y));
                        }
                        *yp = out;
                    }
                }
                if (full_tile && ui.ok) {
                    // the store warp writes the chunk back with TMA and frees the stage
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&ctl.res[s]);
                } else {
                    named_sync(kEpiBar, E_EPI);
                    // coalesced stores: sixteen threads per row, 16 bytes each
                    if (ui.ok) {
#pragma unroll
                        for (int it = 0; it < (PM * NCH / 8) / E_EPI; ++it) {
                            const int i = et + it * E_EPI;
                            const int r = i / (NCH / 8), q = i % (NCH / 8);
                            const int tr = ctl.rows[hb][r];
                            if (r < ui.nvalid && tr >= 0 && 8 * q < len) {
                                const uint8_t *src = ys + (q / 8) * PM * 128 + r * 128 + (((q % 8) ^ (r & 7)) * 16);
                                *reinterpret_cast<uint4 *>(p.Y + (int64_t)tr * p.ldy + c0 + 8 * q) =
                                    *reinterpret_cast<const uint4 *>(src);
                            }
                        }
                    }
                    fence_proxy_async_smem();   // the stage is next written by TMA
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&ctl.res[s]);
                }
            }
        }
    } else {
        // ---------------------------------------------------------------- stores (warp 10)
        if (lane == 0) {
            uint32_t g = 0;
            for (int k = 0; k < n_my && !ctl.fail; ++k) {
                const UnitInfo ui = unit_info(p, ctl.unit[k]);
                for (int ci = 0; ci < ui.nch; ++ci, ++g) {
                    const int s = (int)(g % C::E_NB);
                    if (!exp_wait(p, ctl, &ctl.res[s], (g / C::E_NB) & 1u)) break;
                    // the epilogue staged unit k (its run flag and first row) before it
                    // released any of the unit's chunks
                    if (ctl.unit[k].full && ui.ok) {
                        const int c0 = ui.n_lo + ci * NCH;
                        const int len = min(NCH, ui.n_hi - c0);
                        uint8_t *ys = stages + s * C::E_STAGE + C::B_BYTES;
                        const int row0 = ctl.unit[k].row0;
                        tma_store_2d(&p.y_tile, c0, row0, ys);
                        if (len > 64) tma_store_2d(&p.y_tile, c0 + 64, row0, ys + PM * 128);
                        bulk_commit();
                        bulk_wait_read<0>();   // the stage is free once the store has read it
                    }
                    mbar_arrive(&ctl.empty[s]);
                }
            }
            bulk_wait_all();
        }
        __syncwarp();
    }

    // leave: tensor-core work done, copies landed, tensor memory freed
    __syncthreads();
    if (ctl.fail && tid == 0) {
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < 2000000ull) {
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::E_TMEM);
}

// ------------------------------------------------------------------ launches
// CTAs of `kernel` resident per SM with `smem` bytes, limited by tensor memory.
template <typename K>
int resident_per_sm(K kernel, int threads, int smem, int tmem_cols)
{
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) != cudaSuccess)
        per_sm = 0;
    if (per_sm <= 0) per_sm = 1;
    return per_sm < 512 / tmem_cols ? per_sm : 512 / tmem_cols;
}

// Clusters of `cluster` shrink CTAs resident at once on the current device (cached).
template <int RMAX, int NP = 1>
cudaError_t shrink_active(int cluster, int &active)
{
    using C = ShrinkCfg<RMAX, NP>;
    static std::mutex mu;
    static int cached[64][kMaxSplit + 1] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    active = cached[dev][cluster];
    if (active > 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cluster, 1, 1);
    cfg.blockDim = dim3(PT, 1, 1);
    cfg.dynamicSmemBytes = C::S_SMEM;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaOccupancyMaxActiveClusters(&active, long_shrink_kernel<RMAX, NP, false>, &cfg);
    if (e != cudaSuccess) return e;
    if (active <= 0) return cudaErrorInvalidConfiguration;
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // tensor memory: at most 512 / S_TMEM CTAs per SM
    const int cap = sms * (512 / C::S_TMEM) / cluster;
    if (cap > 0 && active > cap) active = cap;
    cached[dev][cluster] = active;
    return cudaSuccess;
}

template <int RMAX, int NP = 1>
cudaError_t shrink_rmax(const TileParams &p, int64_t max_tiles, cudaStream_t stream)
{
    using C = ShrinkCfg<RMAX, NP>;
    const int cluster = p.ksplit;
    int active = 0;
    cudaError_t e = shrink_active<RMAX, NP>(cluster, active);
    if (e != cudaSuccess) return e;
    const int64_t n = max_tiles < active ? max_tiles : active;
    if (n <= 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(n * cluster), 1, 1);
    cfg.blockDim = dim3(PT, 1, 1);
    cfg.dynamicSmemBytes = C::S_SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // programmatic dependent launch after the decode-shaped kernel of the same call
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return (p.d_in % KB) ? cudaLaunchKernelEx(&cfg, long_shrink_kernel<RMAX, NP, true>, p)
                         : cudaLaunchKernelEx(&cfg, long_shrink_kernel<RMAX, NP, false>, p);
}

template <int RMAX, int MODE>
cudaError_t expand_rmax(const TileParams &p, int64_t max_tiles, cudaStream_t stream)
{
    using C = LongCfg<RMAX>;
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int per_sm = resident_per_sm(long_expand_kernel<RMAX, MODE>, ET, C::E_SMEM, C::E_TMEM);
    int64_t n = (int64_t)sms * per_sm;
    // a CTA's share of the (tile, chunk) pairs spans at most kMaxUnits tiles
    const int64_t need = (max_tiles + kMaxUnits - 3) / (kMaxUnits - 2);
    if (n < need) n = need;
    const int64_t chunks = max_tiles * ((p.d_out + NCH - 1) / NCH);
    if (n > chunks) n = chunks;
    if (n <= 0) return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)n, 1, 1);
    cfg.blockDim = dim3(ET, 1, 1);
    cfg.dynamicSmemBytes = C::E_SMEM;
    cfg.stream = stream;
    // programmatic dependent launch after the shrink: copies of B and Y0 start while
    // it finishes; the epilogue waits for it before reading H
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, long_expand_kernel<RMAX, MODE>, p);
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes)
{
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
}

template <int RMAX, int NP>
cudaError_t set_shrink_attrs()
{
    cudaError_t e;
    for (auto k : {long_shrink_kernel<RMAX, NP, false>, long_shrink_kernel<RMAX, NP, true>}) {
        if ((e = set_smem(k, ShrinkCfg<RMAX, NP>::S_SMEM)) != cudaSuccess) return e;
        if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1)) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template <int RMAX>
cudaError_t set_long_attrs()
{
    using C = LongCfg<RMAX>;
    cudaError_t e;
    if ((e = set_shrink_attrs<RMAX, 1>()) != cudaSuccess) return e;
    if ((e = set_shrink_attrs<RMAX, 2>()) != cudaSuccess) return e;
    if ((e = set_shrink_attrs<RMAX, 3>()) != cudaSuccess) return e;
    if ((e = set_shrink_attrs<RMAX, 4>()) != cudaSuccess) return e;
    if ((e = set_smem(long_expand_kernel<RMAX, MODE_APPLY>, C::E_SMEM)) != cudaSuccess) return e;
    return set_smem(long_expand_kernel<RMAX, MODE_EXPAND>, C::E_SMEM);
}

}  // namespace

int long_shrink_split(int rmax_bucket, int d_in, int64_t tiles)
{
    // cost of a split: waves of resident clusters x 64-column blocks per CTA
    int best = 1;
    int64_t best_cost = -1;
    for (int k = 1; k <= kMaxSplit; ++k) {
        int active = 0;
        cudaError_t e = rmax_bucket <= 16 ? shrink_active<16>(k, active)
                        : rmax_bucket <= 32 ? shrink_active<32>(k, active)
                                            : shrink_active<64>(k, active);
        if (e != cudaSuccess || active <= 0) continue;
        const int k_part = (((d_in + k - 1) / k) + KB - 1) / KB * KB;
        if ((d_in + k_part - 1) / k_part != k) continue;   // k parts would not all be used
        const int64_t waves = (tiles + active - 1) / active;
        const int64_t cost = waves * (k_part / KB);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = k;
        }
    }
    return best;
}

namespace {

template <int NP>
cudaError_t launch_shrink_np(int rmax_bucket, const TileParams &p, int64_t max_tiles, cudaStream_t stream)
{
    switch (rmax_bucket) {
    case 8:
    case 16: return shrink_rmax<16, NP>(p, max_tiles, stream);
    case 32: return shrink_rmax<32, NP>(p, max_tiles, stream);
    case 64: return shrink_rmax<64, NP>(p, max_tiles, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_long_shrink(int rmax_bucket, const TileParams &p, int64_t max_tiles,
                               cudaStream_t stream, int np)
{
    if (p.ksplit < 1 || p.ksplit > kMaxSplit) return cudaErrorInvalidValue;
    switch (np) {
    case 1: return launch_shrink_np<1>(rmax_bucket, p, max_tiles, stream);
    case 2: return launch_shrink_np<2>(rmax_bucket, p, max_tiles, stream);
    case 3: return launch_shrink_np<3>(rmax_bucket, p, max_tiles, stream);
    case 4: return launch_shrink_np<4>(rmax_bucket, p, max_tiles, stream);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_long_expand(int rmax_bucket, int mode, const TileParams &p, int64_t max_tiles,
                               cudaStream_t stream)
{
    const bool apply = mode == MODE_APPLY;
    switch (rmax_bucket) {
    case 8:
    case 16: return apply ? expand_rmax<16, MODE_APPLY>(p, max_tiles, stream)
                          : expand_rmax<16, MODE_EXPAND>(p, max_tiles, stream);
    case 32: return apply ? expand_rmax<32, MODE_APPLY>(p, max_tiles, stream)
                          : expand_rmax<32, MODE_EXPAND>(p, max_tiles, stream);
    case 64: return apply ? expand_rmax<64, MODE_APPLY>(p, max_tiles, stream)
                          : expand_rmax<64, MODE_EXPAND>(p, max_tiles, stream);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t prepare_long_kernels()
{
    cudaError_t e;
    if ((e = set_long_attrs<16>()) != cudaSuccess) return e;
    if ((e = set_long_attrs<32>()) != cudaSuccess) return e;
    return set_long_attrs<64>();
}

}  // namespace mlora
