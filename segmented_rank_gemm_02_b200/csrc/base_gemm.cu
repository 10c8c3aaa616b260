// base_gemm.cu -- the base projection and the LoRA delta in one tensor-core pass.
//
// Y = X W^T + s_a (X A_a^T) B_a^T for the rows of adapter segments and Y = X W^T for
// every other row (page "LoRA/QLoRA multi-tenant serving", section 3.3 on fusing
// W0 x + B(A x) into one kernel, and the paragraph on cuBLASLt epilogue fusion after
// section 5.3: the low-rank product goes into the base GEMM's accumulator, so Y is
// written once, in bf16, and never read).
//
// Order of work.  The shrink H = X A_a^T is the library's segmented shrink (the
// decode-shaped kernel, and the tensor-memory kernel for long segments) into an fp32
// workspace in grouped order.  row_map_kernel then gives each row its grouped
// position, slot, scale and rank (rows outside every valid segment keep position -1:
// base only), and block_slots_kernel lists the distinct slots of each 128-row block.
// Last, the persistent GEMM below.
//
// GEMM tile: 128 rows x 256 columns of Y in one fp32 tensor-memory accumulator (two
// of them, 512 columns, so that a tile's epilogue overlaps the next tile's main
// loop).  Warp roles, which meet only at mbarriers:
//   warp 0     TMA: per 64-wide K block one X tile (128 x 64) and one W tile
//              (256 x 64), 128-byte swizzle, into a 4-stage ring; after the K blocks,
//              per distinct slot of the tile's rows one chunk of that slot's B (256
//              columns x all its rank groups) into the same ring
//   warp 1     owns tensor memory; one thread issues tcgen05.mma: four K=16 steps per
//              K block (M=128, N=256), then per slot (s H)_hi B^T + (s H)_lo B^T
//   warps 2-5  epilogue: tcgen05.ld, one rounding to bf16, 16-byte stores of Y
//   warps 6-9  LoRA operand: the tile's rows of s H for one slot (rows of other
//              slots and base rows zero), as bf16 hi + lo in the tensor core's K-major
//              no-swizzle layout; the masking makes one M=128 product per slot exact
//              for the rows of that slot and zero for the others
// Every mbarrier wait is bounded; on expiry the kernel flags a timeout, stores nothing
// more, lets copies in flight land and frees its tensor memory before it leaves.
#include <algorithm>

#include "kernels.cuh"
#include "ptx.cuh"

namespace mlora {

namespace {

constexpr int GM = kGemmRows;          // 128 rows per tile
constexpr int GN = kGemmCols;          // 256 columns per tile
constexpr int GK = 64;                 // K columns per stage (one 128-byte swizzled row)
constexpr int GS = 4;                  // ring stages
constexpr int X_BYTES = GM * GK * 2;   // 16 KB
constexpr int W_BYTES = GN * GK * 2;   // 32 KB
constexpr int STAGE = X_BYTES + W_BYTES;   // 48 KB; a B chunk takes at most GN * 64 * 2 = 32 KB
constexpr int HOP = GM * 64 * 2;       // one of hi / lo at rank bucket 64: [8][16][8][8] bf16
// Rank bucket 8 runs as K=16: its second operand half is read from 4 KB of zeros
// placed in the part of the hi buffer that bucket 8 leaves unused.
constexpr int ZERO_OFF = 8192;
constexpr int G_SMEM = 1024 + GS * STAGE + 2 * HOP;
constexpr int G_WARPS = 10;
constexpr int GT = G_WARPS * 32;
constexpr int kEpiBar = 1;             // named barrier of the epilogue warps
constexpr int kStgBar = 2;             // named barrier of the operand warps
constexpr int G_TMEM = 2 * GN;         // two accumulators
constexpr uint64_t kGemmWaitNs = 1000000000ull;

static_assert(GN * 64 * 2 <= STAGE, "a B chunk fits in a ring stage");
static_assert(ZERO_OFF >= 2 * (GM / 8) * 128 && ZERO_OFF + GN * 16 <= HOP, "zero block placement");

struct GemmCtl {
    uint64_t full[GS], empty[GS];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t hop_full, hop_empty;
    uint32_t tmem;
    volatile int fail;
};

__device__ __forceinline__ uint8_t *align_1024(uint8_t *p)
{
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ bool gwait(const GemmParams &p, GemmCtl &ctl, uint64_t *bar, uint32_t parity)
{
    if (ctl.fail) return false;
    if (!mbar_wait_bounded(bar, parity, kGemmWaitNs)) {
        ctl.fail = 1;
        atomicOr(p.status, kFlagTimeout);
        return false;
    }
    return true;
}

__device__ __forceinline__ int bucket_index(int R) { return R <= 8 ? 0 : R <= 16 ? 1 : R <= 32 ? 2 : 3; }

}  // namespace

// ------------------------------------------------------------------ row map
// One warp per segment.  A valid segment (slot in range and loaded at the generation
// the batch expects, rank as declared, offsets inside [0, n_tokens]) writes, for each
// of its grouped positions q, row_info[token_indices[q]] = {q, slot, scale, rank}; a
// row claimed twice keeps its first claim and is reported.  Problems set the same
// status bits as the other kernels; the rows concerned stay base only.
__global__ void __launch_bounds__(256) row_map_kernel(const __grid_constant__ TileParams p, int4 *row_info)
{
    const int lane = threadIdx.x & 31;
    const int w0 = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
    const int nw = (int)((gridDim.x * blockDim.x) >> 5);
    for (int g = w0; g < p.n_segments; g += nw) {
        const int a = p.slots[g], p0 = p.offsets[g], p1 = p.offsets[g + 1];
        if (a == -1) continue;   // base-model rows
        unsigned flag = 0;
        int rank = 0;
        float scale = 0.f;
        if (a < -1 || a >= p.n_slots) {
            flag = kFlagBadSlot;
        } else if (p0 < 0 || p1 < p0 || p1 > p.n_tokens) {
            flag = kFlagBadOffsets;
        } else {
            rank = p.slot_rank[a];
            if (p.generations && p.slot_gen[a] != p.generations[g]) flag = kFlagStaleSlot;
            else if (rank <= 0) flag = kFlagSlotEmpty;
            else if ((p.ranks && p.ranks[g] != rank) || rank_bucket(rank) == 0) flag = kFlagBadRank;
            scale = p.scales ? p.scales[g] : p.slot_scale[a];
        }
        if (flag) {
            if (lane == 0) atomicOr(p.status, flag);
            continue;
        }
        for (int q = p0 + lane; q < p1; q += 32) {
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
}

// One CTA of 128 threads per 128-row block: the distinct slots of the block's rows in
// order of first appearance, as out[0] = count, then (slot, rank bucket) pairs.
__global__ void __launch_bounds__(GM) block_slots_kernel(const int4 *row_info, int n_rows, int32_t *out)
{
    __shared__ int s_slot[GM];
    __shared__ int s_count[GM / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int row = blockIdx.x * GM + tid;
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
    for (int w = 0; w < GM / 32; ++w) {
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

// ------------------------------------------------------------------ GEMM
// Tiles t = blockIdx.x, blockIdx.x + gridDim.x, ...; tile t covers rows
// [128 (t / n_nblk), +128) and columns [256 (t % n_nblk), +256).  Every role walks the
// same tiles and reads the same slot lists, so the ring, the accumulators and the
// operand buffer are used in the same order on both sides of each mbarrier.
__global__ void __launch_bounds__(GT, 1) base_gemm_kernel(const __grid_constant__ GemmParams p)
{
    extern __shared__ __align__(128) uint8_t smem_raw[];
    __shared__ GemmCtl ctl;
    uint8_t *ring = align_1024(smem_raw);
    uint8_t *hop_hi = ring + GS * STAGE;
    uint8_t *hop_lo = hop_hi + HOP;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (warp == 1) {
        tmem_alloc(&ctl.tmem, G_TMEM);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int s = 0; s < GS; ++s) {
            mbar_init(&ctl.full[s], 1);
            mbar_init(&ctl.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl.acc_full[b], 1);
            mbar_init(&ctl.acc_empty[b], 4);   // one arrival per epilogue warp
        }
        mbar_init(&ctl.hop_full, 1);
        mbar_init(&ctl.hop_empty, 1);
        fence_mbar_init();
        ctl.fail = 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl.tmem;
    const int n_tiles = p.n_mblk * p.n_nblk;
    const int nk = (p.d_in + GK - 1) / GK;

    if (warp == 0) {
        // ---------------------------------------------------------------- copies
        if (lane == 0) {
            uint32_t g = 0;
            for (int t = blockIdx.x; t < n_tiles && !ctl.fail; t += gridDim.x) {
                const int mb = t / p.n_nblk, n0 = (t % p.n_nblk) * GN;
                const int m0 = mb * GM;
                for (int kb = 0; kb < nk; ++kb, ++g) {
                    const int s = (int)(g % GS);
                    if (g >= GS && !gwait(p, ctl, &ctl.empty[s], ((g / GS) - 1) & 1u)) break;
                    uint8_t *st = ring + s * STAGE;
                    mbar_arrive_expect_tx(&ctl.full[s], (uint32_t)STAGE);
                    tma_load_2d(st, &p.x_map, kb * GK, m0, &ctl.full[s]);
                    tma_load_2d(st + X_BYTES, &p.w_map, kb * GK, n0, &ctl.full[s]);
                }
                const int32_t *bs = p.block_slots + (int64_t)mb * kBlockSlotsPitch;
                const int cnt = bs[0];
                for (int j = 0; j < cnt && !ctl.fail; ++j, ++g) {
                    const int slot = bs[1 + 2 * j], R = bs[2 + 2 * j];
                    const int s = (int)(g % GS);
                    if (g >= GS && !gwait(p, ctl, &ctl.empty[s], ((g / GS) - 1) & 1u)) break;
                    // columns past d_out read as zeros
                    mbar_arrive_expect_tx(&ctl.full[s], (uint32_t)R * GN * 2);
                    tma_load_4d(ring + s * STAGE, &p.b_map[bucket_index(R)], 0, n0, 0, slot, &ctl.full[s]);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- tensor core
        if (lane == 0) {
            uint32_t g = 0, hc = 0, tc = 0;
            const uint32_t idesc = umma_idesc_bf16(GM, GN);
            const uint32_t a_hi = smem_addr(hop_hi), a_lo = smem_addr(hop_lo);
            const uint32_t zero = a_hi + ZERO_OFF;
            for (int t = blockIdx.x; t < n_tiles && !ctl.fail; t += gridDim.x, ++tc) {
                const int mb = t / p.n_nblk;
                const int ab = (int)(tc & 1);
                if (tc >= 2 && !gwait(p, ctl, &ctl.acc_empty[ab], ((tc >> 1) - 1) & 1u)) break;
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(ab * GN);
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb, ++g) {
                    const int s = (int)(g % GS);
                    if (!gwait(p, ctl, &ctl.full[s], (g / GS) & 1u)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t xs = smem_addr(ring + s * STAGE), ws = xs + X_BYTES;
#pragma unroll
                    for (int k = 0; k < GK / 16; ++k)
                        umma_bf16(d, umma_desc_sw128(xs + 32 * k), umma_desc_sw128(ws + 32 * k), idesc,
                                  (kb > 0 || k > 0) ? 1u : 0u);
                    umma_commit(&ctl.empty[s]);   // stage s is free once these MMAs end
                }
                if (!ok) break;
                const int32_t *bs = p.block_slots + (int64_t)mb * kBlockSlotsPitch;
                const int cnt = bs[0];
                for (int j = 0; j < cnt; ++j, ++g, ++hc) {
                    const int R = bs[2 + 2 * j];
                    const int RK = R < 16 ? 16 : R;
                    const int s = (int)(g % GS);
                    if (!gwait(p, ctl, &ctl.hop_full, hc & 1u) || !gwait(p, ctl, &ctl.full[s], (g / GS) & 1u)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t b_s = smem_addr(ring + s * STAGE);
                    for (int st = 0; st < RK / 16; ++st) {
                        const uint32_t b0 = b_s + st * 2 * GN * 16;
                        // bucket 8: the second rank group of B is the zero block
                        const uint32_t lbo = R == 8 ? zero - b0 : GN * 16;
                        const uint64_t bd = umma_desc_kmajor(b0, lbo, 128);
                        const uint32_t koff = st * 2 * (GM / 8) * 128;
                        umma_bf16(d, umma_desc_kmajor(a_hi + koff, (GM / 8) * 128, 128), bd, idesc, 1u);
                        umma_bf16(d, umma_desc_kmajor(a_lo + koff, (GM / 8) * 128, 128), bd, idesc, 1u);
                    }
                    umma_commit(&ctl.empty[s]);
                    umma_commit(&ctl.hop_empty);   // the operand buffer is free once they end
                }
                if (!ok) break;
                umma_commit(&ctl.acc_full[ab]);
            }
        }
        __syncwarp();
    } else if (warp < 6) {
        // ---------------------------------------------------------------- epilogue
        const int quarter = warp & 3;             // tensor-memory lanes 32 quarter .. +31
        const int r = 32 * quarter + lane;        // tile row of this thread
        uint32_t tc = 0;
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++tc) {
            const int mb = t / p.n_nblk, n0 = (t % p.n_nblk) * GN;
            const int ab = (int)(tc & 1);
            // every wait ends in a vote, so the four warps leave together
            if (!named_sync_and(kEpiBar, 128, gwait(p, ctl, &ctl.acc_full[ab], (tc >> 1) & 1u))) break;
            tc_fence_after();
            const int row = mb * GM + r;
            const int ncols = min(GN, p.d_out - n0);
            __nv_bfloat16 *yrow = p.Y + (int64_t)row * p.ldy + n0;
            const uint32_t tbase = tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(ab * GN);
            for (int c = 0; c < GN / 32 && 32 * c < ncols; ++c) {
                uint32_t v[32];
                tmem_ld32(tbase + 32 * c, v);
                tmem_wait_ld();
                if (row < p.n_rows) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        if (32 * c + 8 * q < ncols) {   // d_out is a multiple of 8
                            uint4 o;
                            o.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
                            o.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
                            o.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
                            o.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
                            *reinterpret_cast<uint4 *>(yrow + 32 * c + 8 * q) = o;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl.acc_empty[ab]);
        }
    } else {
        // ---------------------------------------------------------------- LoRA operand
        const int r = tid - 6 * 32;               // tile row 0..127
        uint32_t hc = 0;
        bool alive = true;
        for (int t = blockIdx.x; t < n_tiles && alive; t += gridDim.x) {
            const int mb = t / p.n_nblk;
            const int32_t *bs = p.block_slots + (int64_t)mb * kBlockSlotsPitch;
            const int cnt = bs[0];
            const int row = mb * GM + r;
            int4 info = make_int4(-1, -1, 0, 0);
            if (cnt > 0 && row < p.n_rows) info = p.row_info[row];
            for (int j = 0; j < cnt; ++j, ++hc) {
                const int slot = bs[1 + 2 * j], R = bs[2 + 2 * j];
                const int RK = R < 16 ? 16 : R;
                // the previous use of the buffer must have left the tensor core
                if (hc >= 1 &&
                    !named_sync_and(kStgBar, 128, gwait(p, ctl, &ctl.hop_empty, (hc - 1) & 1u))) {
                    alive = false;
                    break;
                }
                const bool mine = info.x >= 0 && info.y == slot;
                const int rank = mine ? info.w : 0;
                const float sc = mine ? __int_as_float(info.z) : 0.f;   // other rows: exact zeros
                const float *hsrc = p.H + (int64_t)(mine ? info.x : 0) * p.ldh;
                for (int cg = 0; cg < RK / 8; ++cg) {
                    float h[8];
                    if (8 * cg + 8 <= rank) {
                        const float4 v0 = *reinterpret_cast<const float4 *>(hsrc + 8 * cg);
                        const float4 v1 = *reinterpret_cast<const float4 *>(hsrc + 8 * cg + 4);
                        h[0] = v0.x; h[1] = v0.y; h[2] = v0.z; h[3] = v0.w;
                        h[4] = v1.x; h[5] = v1.y; h[6] = v1.z; h[7] = v1.w;
                    } else {
#pragma unroll
                        for (int c = 0; c < 8; ++c) h[c] = (8 * cg + c < rank) ? hsrc[8 * cg + c] : 0.f;
                    }
                    uint4 hi, lo;
                    uint32_t *ph = reinterpret_cast<uint32_t *>(&hi);
                    uint32_t *pl = reinterpret_cast<uint32_t *>(&lo);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        float h0, l0, h1, l1;
                        split_bf16(sc * h[2 * c], h0, l0);
                        split_bf16(sc * h[2 * c + 1], h1, l1);
                        ph[c] = pack_bf16x2(h0, h1);
                        pl[c] = pack_bf16x2(l0, l1);
                    }
                    const int off = (cg * (GM / 8) + r / 8) * 128 + (r % 8) * 16;
                    *reinterpret_cast<uint4 *>(hop_hi + off) = hi;
                    *reinterpret_cast<uint4 *>(hop_lo + off) = lo;
                }
                if (R == 8) {
                    uint4 *z = reinterpret_cast<uint4 *>(hop_hi + ZERO_OFF);
                    for (int i = r; i < GN; i += GM) z[i] = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();   // the operand is read by the tensor core
                named_sync(kStgBar, 128);
                if (r == 0) mbar_arrive(&ctl.hop_full);
            }
        }
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
    if (warp == 1) tmem_dealloc(tmem, G_TMEM);
}

// ------------------------------------------------------------------ launches
cudaError_t launch_row_map(const TileParams &p, int4 *row_info, cudaStream_t stream)
{
    if (p.n_rows > 0) {
        cudaError_t e = cudaMemsetAsync(row_info, 0xff, (size_t)p.n_rows * sizeof(int4), stream);
        if (e != cudaSuccess) return e;
    }
    if (p.n_segments <= 0) return cudaSuccess;
    const int64_t warps = p.n_segments;
    const int blocks = (int)std::min<int64_t>((warps + 7) / 8, 4096);
    row_map_kernel<<<blocks, 256, 0, stream>>>(p, row_info);
    return cudaGetLastError();
}

cudaError_t launch_block_slots(const int4 *row_info, int n_rows, int32_t *block_slots, cudaStream_t stream)
{
    const int n_mblk = (n_rows + GM - 1) / GM;
    if (n_mblk <= 0) return cudaSuccess;
    block_slots_kernel<<<n_mblk, GM, 0, stream>>>(row_info, n_rows, block_slots);
    return cudaGetLastError();
}

cudaError_t launch_base_gemm(const GemmParams &p, cudaStream_t stream)
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
    cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (int64_t)p.n_mblk * p.n_nblk;
    if (tiles <= 0) return cudaSuccess;
    const int grid = (int)std::min<int64_t>(tiles, sms);   // one CTA per SM
    base_gemm_kernel<<<grid, GT, G_SMEM, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t prepare_base_gemm()
{
    cudaError_t e = cudaFuncSetAttribute(base_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, G_SMEM);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(base_gemm_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
}

}  // namespace mlora
