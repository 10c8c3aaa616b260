// lora_tiles.cu -- segmented LoRA shrink / expand / fused apply for sm_100a.
//
// The computation (page "Multi-LoRA Serving: adapter batching", section "What
// metadata a segmented kernel needs"): for each adapter segment g with slot a
// and each grouped position p of it, with t = token_indices[p],
//     H[p, :] = X[t, :] A_a^T                  (shrink, rank r)
//     Y[t, :] = bf16(Y[t, :] + s_g H[p, :] B_a^T)   (expand + scatter)
//
// Work decomposition.  A work tile is (segment, up to 16 consecutive grouped
// positions).  One thread-block cluster of C CTAs owns one tile: CTA c streams
// its slice of d_in for the shrink (split-K) and its slice of d_out for the
// expand.  The C partial H tiles (16 x R fp32) are summed through distributed
// shared memory, so in the fused mode H never leaves the chip.
//
// Data movement.  Each CTA is a small pipeline: thread 0 issues bulk (TMA)
// copies for up to NSTAGES jobs ahead -- the adapter's A or B block for one
// chunk of columns (one contiguous copy per 8-column group, thanks to the
// pool's [cols/8][rows][8] layout) and one copy per activation row (gathered
// through token_indices) -- and the 8 warps consume them in order with bf16
// mma.sync.  The expand's B and Y0 chunks do not depend on H, so they are
// prefetched while the shrink runs.  Results are written back into the staged
// Y0 rows in shared memory and leave with per-row bulk stores.
//
// Rank buckets.  A kernel is compiled for the pool's largest bucket RMAX and
// dispatches every tile to code specialised for its own slot's bucket R <= RMAX,
// so a rank-8 adapter moves and multiplies rank-8 data even in a rank-64 pool.
//
// Precision.  fp32 accumulation throughout.  For the expand, H is split into
// bf16 hi + lo parts and both are multiplied on the tensor cores, so H enters
// the product with about 2^-17 relative error instead of bf16's 2^-9.
//
// Invalid metadata never traps: bad segments and rows are skipped and flagged
// in the status word.  Every mbarrier wait is bounded; a timeout is flagged, the
// tile's results are not stored, and the CTA still takes part in every cluster
// barrier before it leaves.
#include "kernels.cuh"
#include "ptx.cuh"

namespace mlora {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int TM = kTileRows;
constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s per wait
constexpr uint64_t kDrainNs = 2000000ull;          // settle time after a timeout

template <int RMAX>
struct TileCfg {
    static constexpr int KC = 128;                      // d_in columns per shrink job
    static constexpr int NC = 128;                      // d_out columns per expand job
    static constexpr int XPITCH = KC + 8;               // staged X row pitch (elements)
    static constexpr int YPITCH = NC + 8;               // staged Y row pitch (elements)
    static constexpr int A_BYTES = (KC / 8 + 1) * RMAX * 16;  // A chunk + one zero group
    static constexpr int X_BYTES = TM * XPITCH * 2;
    static constexpr int B_BYTES = RMAX * NC * 2;
    static constexpr int Y_BYTES = TM * YPITCH * 2;
    static constexpr int SHRINK_BYTES = A_BYTES + X_BYTES;
    static constexpr int EXPAND_BYTES = B_BYTES + Y_BYTES;
    static constexpr int STAGE =
        ((SHRINK_BYTES > EXPAND_BYTES ? SHRINK_BYTES : EXPAND_BYTES) + 127) / 128 * 128;
    static constexpr int NSTAGES = RMAX <= 8 ? 8 : RMAX <= 16 ? 7 : RMAX <= 32 ? 5 : 4;
    static constexpr int HPITCH = RMAX + 4;             // fp32 pitch of the full H tile
    static constexpr int WPART_FLOATS = kWarps * TM * 8;  // one 16x8 partial per warp
    static constexpr int HPART_FLOATS = TM * RMAX;
    static constexpr int HFULL_FLOATS = TM * HPITCH;
    static constexpr int SMEM =
        NSTAGES * STAGE + 4 * (WPART_FLOATS + HPART_FLOATS + HFULL_FLOATS);
};

struct TileState {
    int seg;        // segment index
    int p0;         // first grouped position of the tile
    int nvalid;     // grouped positions in the tile (<= TM)
    int slot;
    int rank;
    float scale;
    uint32_t crank; // CTA rank in the cluster
    uint32_t csize; // CTAs in the cluster
};

struct SharedCtl {
    uint64_t full_bar[8];
    int rows[TM];       // original row of each tile position, -1 = not present
    int scan[kWarps];
    int tile[3];
    int meta[3];
    float scale;
    int timeout;
};

__device__ __forceinline__ void report(const TileParams &p, unsigned flag)
{
    atomicOr(p.status, flag);
}

// Producer: stage the inputs of job j (thread 0 only).
template <int RMAX, int MODE, int R>
__device__ __forceinline__ void issue_job(const TileParams &p, const TileState &ts, SharedCtl &ctl,
                                          uint8_t *smem, int j, int nK, int k_begin, int k_end,
                                          int n_begin, int n_end, uint64_t pol_stream,
                                          uint64_t pol_keep)
{
    using Cfg = TileCfg<RMAX>;
    const int s = j % Cfg::NSTAGES;
    uint8_t *st = smem + s * Cfg::STAGE;
    uint64_t *bar = &ctl.full_bar[s];
    const __nv_bfloat16 *slotA = p.pool + (int64_t)ts.slot * p.slot_stride;
    int present = 0;
    for (int i = 0; i < ts.nvalid; ++i) present += ctl.rows[i] >= 0;
    if (j < nK) {
        const int kc0 = k_begin + j * Cfg::KC;
        const int len = min(Cfg::KC, k_end - kc0);
        const uint32_t a_bytes = (uint32_t)(len / 8) * R * 16;
        mbar_arrive_expect_tx(bar, a_bytes + (uint32_t)present * len * 2);
        bulk_load_hint(st, slotA + (int64_t)(kc0 / 8) * R * 8, a_bytes, bar, pol_keep);
        for (int i = 0; i < ts.nvalid; ++i) {
            const int t = ctl.rows[i];
            if (t >= 0)
                bulk_load_hint(st + Cfg::A_BYTES + i * Cfg::XPITCH * 2,
                               p.X + (int64_t)t * p.ldx + kc0, len * 2, bar, pol_stream);
        }
    } else {
        const int nc0 = n_begin + (j - nK) * Cfg::NC;
        const int len = min(Cfg::NC, n_end - nc0);
        const __nv_bfloat16 *slotB = slotA + p.b_offset;
        mbar_arrive_expect_tx(bar, (uint32_t)R * len * 2 + (uint32_t)present * len * 2);
#pragma unroll
        for (int q = 0; q < R / 8; ++q)
            bulk_load_hint(st + q * Cfg::NC * 16, slotB + ((int64_t)q * p.d_out + nc0) * 8,
                           len * 16, bar, pol_keep);
        for (int i = 0; i < ts.nvalid; ++i) {
            const int t = ctl.rows[i];
            if (t >= 0)
                bulk_load_hint(st + Cfg::B_BYTES + i * Cfg::YPITCH * 2,
                               p.Y + (int64_t)t * p.ldy + nc0, len * 2, bar, pol_stream);
        }
    }
}

// All warps: wait for job j's stage.
template <int RMAX>
__device__ __forceinline__ void wait_job(const TileParams &p, SharedCtl &ctl, int j, bool &timed_out)
{
    using Cfg = TileCfg<RMAX>;
    if (timed_out) return;
    const int s = j % Cfg::NSTAGES;
    const uint32_t parity = (uint32_t)(j / Cfg::NSTAGES) & 1u;
    if (!mbar_wait_bounded(&ctl.full_bar[s], parity, kWaitLimitNs)) {
        timed_out = true;
        ctl.timeout = 1;
        report(p, kFlagTimeout);
    }
}

// Shrink one staged chunk: warp (nt, ks) accumulates the 16x8 block nt of the
// partial H over every KS-th k16 step.
template <int RMAX, int R>
__device__ __forceinline__ void shrink_chunk(uint8_t *st, int len, float (&acc)[4], int warp,
                                             int lane, int tid)
{
    using Cfg = TileCfg<RMAX>;
    constexpr int NT = R / 8;
    constexpr int KS = kWarps / NT;
    if (len & 15) {
        // d_in ends on an odd 8-column group: zero the 8 columns after it in A and X
        // so the last k16 step adds nothing.
        uint4 *za = reinterpret_cast<uint4 *>(st + (len / 8) * R * 16);
        for (int i = tid; i < R; i += kThreads) za[i] = make_uint4(0, 0, 0, 0);
        if (tid < TM)
            *reinterpret_cast<uint4 *>(st + Cfg::A_BYTES + tid * Cfg::XPITCH * 2 + len * 2) =
                make_uint4(0, 0, 0, 0);
        __syncthreads();
    }
    const int nt = warp % NT;
    const int ks = warp / NT;
    const int nsteps = (len + 15) / 16;
    const uint32_t as = smem_addr(st);
    const uint32_t xs = smem_addr(st + Cfg::A_BYTES);
    const int m = lane >> 3, i = lane & 7;
    const int xrow = i + ((m & 1) << 3);
    const int xcol = (m >> 1) << 3;
    for (int step = ks; step < nsteps; step += KS) {
        uint32_t a0, a1, a2, a3, b0, b1;
        ldsm_x4(xs + (xrow * Cfg::XPITCH + step * 16 + xcol) * 2, a0, a1, a2, a3);
        const int kg = step * 2 + (m & 1);
        ldsm_x2(as + (kg * R + nt * 8 + i) * 16, b0, b1);
        mma_16816(acc, a0, a1, a2, a3, b0, b1);
    }
}

// Expand one staged chunk and write the bf16 results over the staged Y0 rows.
// k16 steps of the expand (one k8 step for rank bucket 8)
template <int R>
__host__ __device__ constexpr int expand_ksteps() { return (R + 15) / 16; }

template <int RMAX, int R>
__device__ __forceinline__ void expand_chunk(uint8_t *st, int len,
                                             const uint32_t (&ah)[expand_ksteps<R>()][4],
                                             const uint32_t (&al)[expand_ksteps<R>()][4],
                                             float scale, int warp, int lane)
{
    using Cfg = TileCfg<RMAX>;
    const uint32_t bs = smem_addr(st);
    uint8_t *ys = st + Cfg::B_BYTES;
    const int ntiles = len / 8;
    const int gq = lane >> 2, tq = lane & 3;
    for (int tn = warp; tn < ntiles; tn += kWarps) {
        const int n0 = tn * 8;
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (R == 8) {
            uint32_t b0;
            ldsm_x1(bs + (n0 + (lane & 7)) * 16, b0);
            mma_1688(d, ah[0][0], ah[0][1], b0);
            mma_1688(d, al[0][0], al[0][1], b0);
        } else {
#pragma unroll
            for (int kk = 0; kk < R / 16; ++kk) {
                uint32_t b0, b1;
                const int kg = 2 * kk + ((lane >> 3) & 1);
                ldsm_x2(bs + (kg * Cfg::NC + n0 + (lane & 7)) * 16, b0, b1);
                mma_16816(d, ah[kk][0], ah[kk][1], ah[kk][2], ah[kk][3], b0, b1);
                mma_16816(d, al[kk][0], al[kk][1], al[kk][2], al[kk][3], b0, b1);
            }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int row = gq + 8 * h;
            __nv_bfloat162 *yp =
                reinterpret_cast<__nv_bfloat162 *>(ys + (row * Cfg::YPITCH + n0 + 2 * tq) * 2);
            const float2 y0 = __bfloat1622float2(*yp);
            *yp = __floats2bfloat162_rn(fmaf(scale, d[2 * h], y0.x), fmaf(scale, d[2 * h + 1], y0.y));
        }
    }
}

template <int RMAX, int MODE, int R>
__device__ __forceinline__ void run_tile(const TileParams &p, const TileState &ts, SharedCtl &ctl,
                                         uint8_t *smem)
{
    using Cfg = TileCfg<RMAX>;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float *wpart = reinterpret_cast<float *>(smem + Cfg::NSTAGES * Cfg::STAGE);
    float *hpart = wpart + Cfg::WPART_FLOATS;
    float *hfull = hpart + Cfg::HPART_FLOATS;

    const int k_begin = min(p.d_in, (int)ts.crank * p.k_slice);
    const int k_end = min(p.d_in, k_begin + p.k_slice);
    const int n_begin = min(p.d_out, (int)ts.crank * p.n_slice);
    const int n_end = min(p.d_out, n_begin + p.n_slice);
    const int nK = (MODE == MODE_EXPAND) ? 0 : (k_end - k_begin + Cfg::KC - 1) / Cfg::KC;
    const int nN = (MODE == MODE_SHRINK) ? 0 : (n_end - n_begin + Cfg::NC - 1) / Cfg::NC;
    const int J = nK + nN;

    uint64_t pol_stream = 0, pol_keep = 0;
    if (tid == 0) {
        pol_stream = policy_evict_first();
        pol_keep = policy_evict_last();
        for (int j = 0; j < J && j < Cfg::NSTAGES; ++j)
            issue_job<RMAX, MODE, R>(p, ts, ctl, smem, j, nK, k_begin, k_end, n_begin, n_end,
                                     pol_stream, pol_keep);
    }
    bool timed_out = false;
    uint32_t store_mask = 0;   // stages with bulk stores still reading them (thread 0)

    // ---------------- shrink: partial H over this CTA's d_in slice
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < nK; ++j) {
        wait_job<RMAX>(p, ctl, j, timed_out);
        const int kc0 = k_begin + j * Cfg::KC;
        shrink_chunk<RMAX, R>(smem + (j % Cfg::NSTAGES) * Cfg::STAGE, min(Cfg::KC, k_end - kc0),
                              acc, warp, lane, tid);
        __syncthreads();
        if (tid == 0 && j + Cfg::NSTAGES < J)
            issue_job<RMAX, MODE, R>(p, ts, ctl, smem, j + Cfg::NSTAGES, nK, k_begin, k_end,
                                     n_begin, n_end, pol_stream, pol_keep);
    }

    if constexpr (MODE != MODE_EXPAND) {
        constexpr int NT = R / 8;
        constexpr int KS = kWarps / NT;
        const int gq = lane >> 2, tq = lane & 3;
        float *wp = wpart + warp * TM * 8;
        wp[gq * 8 + 2 * tq] = acc[0];
        wp[gq * 8 + 2 * tq + 1] = acc[1];
        wp[(gq + 8) * 8 + 2 * tq] = acc[2];
        wp[(gq + 8) * 8 + 2 * tq + 1] = acc[3];
        __syncthreads();
        for (int e = tid; e < TM * R; e += kThreads) {
            const int i = e / R, jj = e % R;
            const int nt = jj / 8, c = jj % 8;
            float sum = 0.f;
#pragma unroll
            for (int k = 0; k < KS; ++k) sum += wpart[(k * NT + nt) * TM * 8 + i * 8 + c];
            hpart[e] = sum;
        }
        // sum the cluster's partial tiles through distributed shared memory
        cluster_arrive_release();
        cluster_wait_acquire();
        const uint32_t hpart_s = smem_addr(hpart);
        if constexpr (MODE == MODE_APPLY) {
            for (int e = tid; e < TM * R; e += kThreads) {
                float sum = 0.f;
                for (uint32_t c = 0; c < ts.csize; ++c)
                    sum += ld_dsmem_f32(map_to_rank(hpart_s + 4u * e, c));
                hfull[(e / R) * Cfg::HPITCH + e % R] = sum;
            }
        } else {
            for (int e = tid; e < TM * R; e += kThreads) {
                const int i = e / R, jj = e % R;
                if ((uint32_t)i % ts.csize != ts.crank || i >= ts.nvalid || jj >= ts.rank ||
                    ctl.rows[i] < 0)
                    continue;
                float sum = 0.f;
                for (uint32_t c = 0; c < ts.csize; ++c)
                    sum += ld_dsmem_f32(map_to_rank(hpart_s + 4u * e, c));
                if (!ctl.timeout) p.H[(int64_t)(ts.p0 + i) * p.ldh + jj] = sum;
            }
        }
        cluster_arrive_relaxed();   // paired with the wait before the CTA leaves
    } else {
        for (int e = tid; e < TM * R; e += kThreads) {
            const int i = e / R, jj = e % R;
            float v = 0.f;
            if (i < ts.nvalid && jj < ts.rank) v = p.H[(int64_t)(ts.p0 + i) * p.ldh + jj];
            hfull[i * Cfg::HPITCH + jj] = v;
        }
    }

    if constexpr (MODE != MODE_SHRINK) {
        __syncthreads();
        // H as bf16 hi + lo A-fragments (rows g, g+8; columns 2t.., 2t+8..)
        constexpr int KSTEPS = expand_ksteps<R>();
        uint32_t ah[KSTEPS][4], al[KSTEPS][4];
        const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int row = gq + ((q & 1) << 3);
                const int col = kk * 16 + 2 * tq + ((q >> 1) << 3);
                float x0 = 0.f, x1 = 0.f;
                if (col < R) {
                    x0 = hfull[row * Cfg::HPITCH + col];
                    x1 = hfull[row * Cfg::HPITCH + col + 1];
                }
                float h0, l0, h1, l1;
                split_bf16(x0, h0, l0);
                split_bf16(x1, h1, l1);
                ah[kk][q] = pack_bf16x2(h0, h1);
                al[kk][q] = pack_bf16x2(l0, l1);
            }
        }
        for (int j = nK; j < J; ++j) {
            wait_job<RMAX>(p, ctl, j, timed_out);
            const int s = j % Cfg::NSTAGES;
            uint8_t *st = smem + s * Cfg::STAGE;
            const int nc0 = n_begin + (j - nK) * Cfg::NC;
            const int len = min(Cfg::NC, n_end - nc0);
            expand_chunk<RMAX, R>(st, len, ah, al, ts.scale, warp, lane);
            fence_proxy_async_smem();
            __syncthreads();
            if (tid == 0) {
                if (!ctl.timeout) {
                    for (int i = 0; i < ts.nvalid; ++i) {
                        const int t = ctl.rows[i];
                        if (t >= 0)
                            bulk_store(p.Y + (int64_t)t * p.ldy + nc0,
                                       st + Cfg::B_BYTES + i * Cfg::YPITCH * 2, len * 2);
                    }
                    bulk_commit();
                    store_mask |= 1u << s;
                }
                if (j + Cfg::NSTAGES < J) {
                    const int s_next = (j + Cfg::NSTAGES) % Cfg::NSTAGES;
                    if (store_mask & (1u << s_next)) {
                        bulk_wait_read_all();
                        store_mask = 0;
                    }
                    issue_job<RMAX, MODE, R>(p, ts, ctl, smem, j + Cfg::NSTAGES, nK, k_begin,
                                             k_end, n_begin, n_end, pol_stream, pol_keep);
                }
            }
        }
    }

    if (tid == 0) bulk_wait_all();
    if constexpr (MODE != MODE_EXPAND) cluster_wait_acquire();
    if (ctl.timeout) {
        // let copies still in flight land before shared memory is released
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < kDrainNs) {
        }
    }
}

template <int RMAX, int MODE>
__global__ void __launch_bounds__(kThreads) lora_tile_kernel(const __grid_constant__ TileParams p)
{
    using Cfg = TileCfg<RMAX>;
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ SharedCtl ctl;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tile = (int)cluster_index();
    const bool reporter = blockIdx.x == 0;

    // ---- find this cluster's tile: per-segment tile counts, block-wide scan
    if (tid == 0) {
        ctl.tile[0] = -1;
        ctl.timeout = 0;
    }
    __syncthreads();
    int running = 0;
    for (int base = 0; base < p.n_segments; base += kThreads) {
        const int g = base + tid;
        int cnt = 0, p0 = 0, p1 = 0;
        if (g < p.n_segments) {
            const int a = p.slots[g];
            p0 = p.offsets[g];
            p1 = p.offsets[g + 1];
            if (a != -1) {
                if (a < -1 || a >= p.n_slots) {
                    if (reporter) report(p, kFlagBadSlot);
                } else if (p0 < 0 || p1 < p0 || p1 > p.n_tokens) {
                    if (reporter) report(p, kFlagBadOffsets);
                } else {
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
        if (cnt > 0 && tile >= lo && tile < running + incl) {
            ctl.tile[0] = g;
            ctl.tile[1] = p0 + (tile - lo) * TM;
            ctl.tile[2] = p1;
        }
        running += total;
        __syncthreads();
        if (ctl.tile[0] >= 0 || running > tile) break;
    }
    if (ctl.tile[0] < 0) return;   // same decision in every CTA of the cluster

    TileState ts;
    ts.seg = ctl.tile[0];
    ts.p0 = ctl.tile[1];
    ts.nvalid = min(TM, ctl.tile[2] - ts.p0);
    ts.crank = cluster_rank();
    ts.csize = cluster_size();

    // ---- tile metadata and row list
    if (tid == 0) {
        const int a = p.slots[ts.seg];
        const int r = p.slot_rank[a];
        int ok = 1;
        if (r <= 0) {
            ok = 0;
            if (ts.crank == 0) report(p, kFlagSlotEmpty);
        } else if ((p.ranks != nullptr && p.ranks[ts.seg] != r) || rank_bucket(r) == 0 ||
                   rank_bucket(r) > RMAX) {
            ok = 0;
            if (ts.crank == 0) report(p, kFlagBadRank);
        }
        ctl.meta[0] = a;
        ctl.meta[1] = r;
        ctl.meta[2] = ok;
        ctl.scale = p.scales ? p.scales[ts.seg] : p.slot_scale[a];
#pragma unroll
        for (int s = 0; s < Cfg::NSTAGES; ++s) mbar_init(&ctl.full_bar[s], 1);
        fence_mbar_init();
    }
    if (tid < TM) {
        int t = -1;
        if (tid < ts.nvalid) {
            t = p.token_indices ? p.token_indices[ts.p0 + tid] : ts.p0 + tid;
            if (t < 0 || t >= p.n_rows) {
                if (ts.crank == 0) report(p, kFlagBadRow);
                t = -1;
            }
        }
        ctl.rows[tid] = t;
    }
    __syncthreads();
    if (!ctl.meta[2]) return;   // same decision in every CTA of the cluster
    ts.slot = ctl.meta[0];
    ts.rank = ctl.meta[1];
    ts.scale = ctl.scale;

    const int R = rank_bucket(ts.rank);
    if (R == 8) {
        run_tile<RMAX, MODE, 8>(p, ts, ctl, smem);
    } else if (R == 16) {
        if constexpr (RMAX >= 16) run_tile<RMAX, MODE, 16>(p, ts, ctl, smem);
    } else if (R == 32) {
        if constexpr (RMAX >= 32) run_tile<RMAX, MODE, 32>(p, ts, ctl, smem);
    } else {
        if constexpr (RMAX >= 64) run_tile<RMAX, MODE, 64>(p, ts, ctl, smem);
    }
}

template <int RMAX, int MODE>
cudaError_t launch_one(const TileParams &p, int cluster, int n_clusters, cudaStream_t stream)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(n_clusters * cluster), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = TileCfg<RMAX>::SMEM;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, lora_tile_kernel<RMAX, MODE>, p);
}

template <int RMAX>
cudaError_t launch_rmax(int mode, const TileParams &p, int cluster, int n_clusters,
                        cudaStream_t stream)
{
    switch (mode) {
    case MODE_APPLY: return launch_one<RMAX, MODE_APPLY>(p, cluster, n_clusters, stream);
    case MODE_SHRINK: return launch_one<RMAX, MODE_SHRINK>(p, cluster, n_clusters, stream);
    case MODE_EXPAND: return launch_one<RMAX, MODE_EXPAND>(p, cluster, n_clusters, stream);
    default: return cudaErrorInvalidValue;
    }
}

template <int RMAX>
cudaError_t set_attrs()
{
    cudaError_t e;
    e = cudaFuncSetAttribute(lora_tile_kernel<RMAX, MODE_APPLY>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, TileCfg<RMAX>::SMEM);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(lora_tile_kernel<RMAX, MODE_SHRINK>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, TileCfg<RMAX>::SMEM);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(lora_tile_kernel<RMAX, MODE_EXPAND>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, TileCfg<RMAX>::SMEM);
}

// Repack: A [rank, d_in] -> [d_in/8][R][8]; B [d_out, rank] -> [R/8][d_out][8]; zero
// beyond rank.  Written destination-contiguous.
__global__ void repack_slot_kernel(__nv_bfloat16 *slot, int64_t b_offset, int R, int rank,
                                   int d_in, int d_out, const __nv_bfloat16 *A,
                                   const __nv_bfloat16 *B, int32_t *rank_entry,
                                   float *scale_entry, float scale)
{
    const int64_t na = (int64_t)R * d_in;
    const int64_t nb = (int64_t)R * d_out;
    const __nv_bfloat16 zero = __float2bfloat16_rn(0.f);
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < na + nb;
         e += (int64_t)gridDim.x * blockDim.x) {
        if (e < na) {
            const int64_t kg = e / (8 * R);
            const int j = (int)((e / 8) % R);
            const int64_t k = kg * 8 + e % 8;
            slot[e] = j < rank ? A[(int64_t)j * d_in + k] : zero;
        } else {
            const int64_t f = e - na;
            const int64_t jg = f / (8 * (int64_t)d_out);
            const int64_t o = (f / 8) % d_out;
            const int j = (int)(jg * 8 + f % 8);
            slot[b_offset + f] = j < rank ? B[o * rank + j] : zero;
        }
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        *rank_entry = rank;
        *scale_entry = scale;
    }
}

}  // namespace

cudaError_t launch_tile_kernel(int mode, int rmax_bucket, const TileParams &p, int cluster,
                               int n_clusters, cudaStream_t stream)
{
    switch (rmax_bucket) {
    case 8: return launch_rmax<8>(mode, p, cluster, n_clusters, stream);
    case 16: return launch_rmax<16>(mode, p, cluster, n_clusters, stream);
    case 32: return launch_rmax<32>(mode, p, cluster, n_clusters, stream);
    case 64: return launch_rmax<64>(mode, p, cluster, n_clusters, stream);
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
                               float *slot_scale_entry, float scale, cudaStream_t stream)
{
    const int64_t total = (int64_t)R * (d_in + d_out);
    const int threads = 256;
    const int64_t blocks64 = (total + threads - 1) / threads;
    const int blocks = (int)(blocks64 < 4096 ? blocks64 : 4096);
    repack_slot_kernel<<<blocks, threads, 0, stream>>>(slot_base, b_offset, R, rank, d_in, d_out,
                                                       A_src, B_src, slot_rank_entry,
                                                       slot_scale_entry, scale);
    return cudaGetLastError();
}

}  // namespace mlora
