// mlora.cu -- host side of the C ABI declared in include/mlora.h.
//
// The adapter pool (page "LoRA/QLoRA multi-tenant serving", ybb.press, section 1.1:
// one pre-allocated buffer, fixed per-adapter size, O(1) slot addressing) and the
// argument checks, kernel choice and launches of mlora_shrink / mlora_expand /
// mlora_apply.  The grouping helper mlora_build_segments follows the metadata
// layout of page "Multi-LoRA Serving: adapter batching", section "What metadata a
// segmented kernel needs".
#include "mlora.h"

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>
#include <unordered_map>
#include <vector>

#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "internal.h"
#include "kernels.cuh"

struct mlora_pool {
    int device;
    int32_t d_in, d_out, n_slots, r_max, r_bucket_max;
    int64_t slot_stride;   // elements per slot
    int64_t b_offset;      // elements from a slot's start to its B block
    __nv_bfloat16 *buf;
    int32_t *d_rank;
    float *d_scale;
    uint32_t *d_gen;        // generation of each slot's contents (device copy)
    unsigned int *d_status;
    std::vector<int32_t> h_rank;
    std::vector<float> h_alpha;
    std::vector<uint32_t> h_gen;
    float *ws;              // H partial sums of the long-segment kernels (grown on demand)
    size_t ws_bytes;
    std::mutex ws_mutex;
    // TMA views of the B blocks for rank buckets 8, 16, 32, 64 (those <= r_bucket_max):
    // one load brings one 128-column chunk of one slot's B, all its rank groups
    CUtensorMap b_maps[4];
    // the same blocks viewed as [slot][rank group][d_out / 32][32 columns x 8] (when
    // d_out is a multiple of 32): one box {256, 4, R/8, 1} brings the same 128-column
    // chunk in 512-byte rows instead of 16-byte ones
    CUtensorMap b_maps_wide[4];
    bool b_maps_wide_ok;
    bool b_maps_ok;
};

namespace {

using mlora::rank_bucket;

// Runs the body with the pool's device current, restoring the caller's device.
struct DeviceGuard {
    int prev = -1;
    bool ok = true;
    explicit DeviceGuard(int dev)
    {
        if (cudaGetDevice(&prev) != cudaSuccess) {
            ok = false;
            return;
        }
        if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
    }
    ~DeviceGuard()
    {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

std::mutex g_prep_mutex;
bool g_prepared[128] = {};

mlora_status prepare_device(int dev)
{
    std::lock_guard<std::mutex> lock(g_prep_mutex);
    if (dev < 0 || dev >= 128) return MLORA_ERR_INVALID_ARG;
    if (g_prepared[dev]) return MLORA_OK;
    if (mlora::prepare_tile_kernels() != cudaSuccess) return MLORA_ERR_CUDA;
    if (mlora::prepare_long_kernels() != cudaSuccess) return MLORA_ERR_CUDA;
    if (mlora::prepare_base_gemm() != cudaSuccess) return MLORA_ERR_CUDA;
    g_prepared[dev] = true;
    return MLORA_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

// Cluster size: enough CTAs per tile to spread one adapter's A and B over ~1K
// columns each, at most 8 (the portable cluster size), and every CTA must own at
// least one 32-column block of d_in and one 8-column group of d_out.
int choose_cluster(int d_in, int d_out)
{
    int c = (int)std::min<int64_t>(8, std::max<int64_t>(1, (int64_t)(d_in + d_out + 1023) / 1024));
    while (c > 1 && (round_up((d_in + c - 1) / c, 32) * (c - 1) >= d_in ||
                     round_up((d_out + c - 1) / c, 8) * (c - 1) >= d_out))
        --c;
    return c;
}

mlora_status check_segments(const mlora_pool *pool, const mlora_segments *s)
{
    if (pool == nullptr || s == nullptr) return MLORA_ERR_INVALID_ARG;
    if (s->n_segments < 0 || s->n_rows < 0 || s->n_tokens < 0) return MLORA_ERR_INVALID_ARG;
    if (s->n_segments > 0 && (s->segment_offsets == nullptr || s->adapter_slots == nullptr))
        return MLORA_ERR_INVALID_ARG;
    return MLORA_OK;
}

mlora::TileParams base_params(const mlora_pool *pool, const mlora_segments *s)
{
    mlora::TileParams p{};
    p.pool = pool->buf;
    p.slot_stride = pool->slot_stride;
    p.b_offset = pool->b_offset;
    p.slot_rank = pool->d_rank;
    p.slot_scale = pool->d_scale;
    p.slot_gen = pool->d_gen;
    p.n_slots = pool->n_slots;
    p.status = pool->d_status;
    p.d_in = pool->d_in;
    p.d_out = pool->d_out;
    p.n_segments = s->n_segments;
    p.n_rows = s->n_rows;
    p.n_tokens = s->n_tokens;
    p.offsets = s->segment_offsets;
    p.slots = s->adapter_slots;
    p.ranks = s->ranks;
    p.scales = s->scales;
    p.token_indices = s->token_indices;
    p.generations = s->generations;
    for (int i = 0; i < 4; ++i) p.b_map[i] = pool->b_maps_wide_ok ? pool->b_maps_wide[i] : pool->b_maps[i];
    p.b_col_div = pool->b_maps_wide_ok ? 32 : 1;
    return p;
}

// Segments with at least this many rows go to the tensor-memory (long-segment) kernels.
constexpr int kLongRows = 128;

// cuTensorMapEncodeTiled, fetched once through the runtime (no link to the driver library).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// bf16 [rows, cols] with row stride ld (elements), 128-byte swizzle, box 64 x box_rows.
bool encode_rows_map(CUtensorMap *map, const void *base, int64_t rows, int64_t cols, int64_t ld,
                     uint32_t box_rows)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (enc == nullptr || base == nullptr || rows <= 0 || cols <= 0) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t elem[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, elem,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The pool's B blocks as a 4-D tensor [slot][rank group][d_out][8] (bf16), box
// {8, cols, R/8, 1}: one chunk of `cols` columns of one slot's B for rank bucket R.
bool encode_b_map(CUtensorMap *map, const mlora_pool *pool, int R, int cols)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (enc == nullptr) return false;
    const int groups = pool->r_bucket_max / 8;
    cuuint64_t dims[4] = {8, (cuuint64_t)pool->d_out, (cuuint64_t)groups, (cuuint64_t)pool->n_slots};
    cuuint64_t strides[3] = {16, (cuuint64_t)pool->d_out * 16, (cuuint64_t)pool->slot_stride * 2};
    cuuint32_t box[4] = {8, (cuuint32_t)cols, (cuuint32_t)(R / 8), 1};
    cuuint32_t elem[4] = {1, 1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, pool->buf + pool->b_offset, dims, strides, box,
               elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The wide view of the pool's B blocks (d_out a multiple of 32), box {256, 4, R/8, 1}.
bool encode_b_map_wide(CUtensorMap *map, const mlora_pool *pool, int R)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (enc == nullptr || pool->d_out % 32 != 0) return false;
    const int groups = pool->r_bucket_max / 8;
    cuuint64_t dims[4] = {256, (cuuint64_t)pool->d_out / 32, (cuuint64_t)groups, (cuuint64_t)pool->n_slots};
    cuuint64_t strides[3] = {512, (cuuint64_t)pool->d_out * 16, (cuuint64_t)pool->slot_stride * 2};
    cuuint32_t box[4] = {256, (cuuint32_t)mlora::kExpandChunk / 32, (cuuint32_t)(R / 8), 1};
    cuuint32_t elem[4] = {1, 1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, pool->buf + pool->b_offset, dims, strides, box,
               elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Make the pool's workspace hold `bytes` (the caller holds pool->ws_mutex and keeps it
// until the kernels that use the workspace are launched, so that no other thread frees
// it in between).  Growth is stream-ordered (the old buffer is freed, and the new one
// allocated, on `stream`: no device-wide synchronisation); it is not possible while
// the stream is being captured.
mlora_status ensure_workspace(mlora_pool *pool, size_t bytes, cudaStream_t stream)
{
    if (pool->ws_bytes >= bytes) return MLORA_OK;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return MLORA_ERR_CUDA;
    if (cs != cudaStreamCaptureStatusNone) return MLORA_ERR_UNSUPPORTED;
    if (pool->ws) {
        if (cudaFreeAsync(pool->ws, stream) != cudaSuccess) return MLORA_ERR_CUDA;
        pool->ws = nullptr;
        pool->ws_bytes = 0;
    }
    // some headroom, so that a slowly growing batch does not reallocate every call
    const size_t want = std::max<size_t>(bytes + bytes / 4, (size_t)1 << 20);
    if (cudaMallocAsync(reinterpret_cast<void **>(&pool->ws), want, stream) != cudaSuccess) {
        cudaGetLastError();
        pool->ws = nullptr;
        return MLORA_ERR_OUT_OF_MEMORY;
    }
    pool->ws_bytes = want;
    return MLORA_OK;
}

// Whether the batch may hold long segments for the tensor-memory kernels: only if some
// segment may reach kLongRows (the host's hint, when given, rules them out).
bool long_path(const mlora_pool *pool, const mlora_segments *s)
{
    return s->n_tokens >= kLongRows &&
           (s->max_segment_rows <= 0 || s->max_segment_rows >= kLongRows) && pool->b_maps_ok;
}

// The single projection of a launch as entry 0 of the per-projection table.
void set_single_projection(mlora::TileParams &p)
{
    p.n_proj = 1;
    p.proj[0] = mlora::ProjView{p.pool, p.slot_stride, p.b_offset, p.slot_rank, p.slot_scale, p.slot_gen,
                                p.status, p.d_out, p.n_slice, p.Y, p.ldy};
}

mlora_status launch_long(mlora_pool *pool, const mlora_segments *s, int mode, mlora::TileParams &p,
                         cudaStream_t stream, float *ext_ws, size_t ext_ws_bytes, bool run_shrink = true);

// `ext_ws` (optional): caller-provided memory of `ext_ws_bytes` for the long-segment H
// workspace, used instead of the pool's own (which is then never grown).
mlora_status launch(mlora_pool *pool, const mlora_segments *s, int mode, mlora::TileParams &p,
                    void *stream_v, float *ext_ws = nullptr, size_t ext_ws_bytes = 0)
{
    cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
    const int c = choose_cluster(pool->d_in, pool->d_out);
    p.k_slice = (int32_t)round_up((pool->d_in + c - 1) / c, 32);
    p.n_slice = (int32_t)round_up((pool->d_out + c - 1) / c, 8);
    set_single_projection(p);
    // the decode kernel leaves the long segments alone when the long kernels run
    const bool use_long = long_path(pool, s);
    p.long_rows = use_long ? kLongRows : 0x7fffffff;
    p.early = use_long ? 0 : 1;
    mlora_status st = prepare_device(pool->device);
    if (st != MLORA_OK) return st;

    const int64_t tiles = (int64_t)s->n_segments + (int64_t)s->n_tokens / mlora::kTileRows + 1;
    cudaError_t e = mlora::launch_tile_kernel(mode, pool->r_bucket_max, p, c, tiles, stream);
    if (e != cudaSuccess) return MLORA_ERR_CUDA;
    if (!use_long) return MLORA_OK;
    return launch_long(pool, s, mode, p, stream, ext_ws, ext_ws_bytes);
}

// Upper bound on the long tiles of a batch (grid sizing of the long kernels).
int64_t long_tile_bound(const mlora_segments *s)
{
    return (int64_t)s->n_tokens / mlora::kLongTileRows + s->n_tokens / kLongRows + 1;
}

// Shrink geometry of the long-segment kernels (d_in split over a cluster of ksplit
// CTAs per tile) and the TMA views of X (tiles of consecutive rows, single rows for
// gathers).
mlora_status setup_long_shrink(const mlora_pool *pool, const mlora_segments *s, mlora::TileParams &p)
{
    p.long_rows = kLongRows;
    p.early = 0;
    const int64_t est_tiles = std::max<int64_t>(1, (s->n_tokens + mlora::kLongTileRows - 1) / mlora::kLongTileRows);
    int ksplit = mlora::long_shrink_split(pool->r_bucket_max, pool->d_in, est_tiles);
    p.k_part = (int32_t)round_up((pool->d_in + ksplit - 1) / ksplit, 64);
    ksplit = (pool->d_in + p.k_part - 1) / p.k_part;
    p.ksplit = ksplit;
    if (!encode_rows_map(&p.x_tile, p.X, s->n_rows, pool->d_in, p.ldx, mlora::kLongTileRows) ||
        !encode_rows_map(&p.x_rows, p.X, s->n_rows, pool->d_in, p.ldx, 1))
        return MLORA_ERR_CUDA;
    return MLORA_OK;
}

// The long-segment kernels (shrink, then expand) of one projection; without
// run_shrink only the expand, on the H a fused shrink already left in the workspace.
mlora_status launch_long(mlora_pool *pool, const mlora_segments *s, int mode, mlora::TileParams &p,
                         cudaStream_t stream, float *ext_ws, size_t ext_ws_bytes, bool run_shrink)
{
    mlora_status st = MLORA_OK;
    cudaError_t e = cudaSuccess;
    p.long_rows = kLongRows;
    p.early = 0;
    const int64_t long_tiles = long_tile_bound(s);
    const int rk = std::max(16, pool->r_bucket_max);
    if (mode != mlora::MODE_EXPAND && run_shrink) {
        st = setup_long_shrink(pool, s, p);
        if (st != MLORA_OK) return st;
    }
    if (mode != mlora::MODE_SHRINK &&
        (!encode_rows_map(&p.y_tile, p.Y, s->n_rows, pool->d_out, p.ldy, mlora::kLongTileRows) ||
         !encode_rows_map(&p.y_rows, p.Y, s->n_rows, pool->d_out, p.ldy, 1)))
        return MLORA_ERR_CUDA;
    if (mode == mlora::MODE_APPLY && ext_ws != nullptr) {
        if ((size_t)s->n_tokens * rk * sizeof(float) > ext_ws_bytes) return MLORA_ERR_UNSUPPORTED;
        p.ws = ext_ws;
        p.ws_ld = rk;
    }
    std::unique_lock<std::mutex> ws_lock(pool->ws_mutex, std::defer_lock);
    if (mode == mlora::MODE_APPLY && ext_ws == nullptr) {
        ws_lock.lock();   // held until the long kernels are launched
        const size_t bytes = (size_t)s->n_tokens * rk * sizeof(float);
        st = ensure_workspace(pool, bytes, stream);
        if (st != MLORA_OK) return st;
        p.ws = pool->ws;
        p.ws_ld = rk;
    } else if (mode != mlora::MODE_APPLY) {
        p.ws = p.H;
        p.ws_ld = p.ldh;
    }
    if (mode != mlora::MODE_EXPAND && run_shrink) {
        e = mlora::launch_long_shrink(pool->r_bucket_max, p, long_tiles, stream);
        if (e != cudaSuccess) return MLORA_ERR_CUDA;
    }
    if (mode != mlora::MODE_SHRINK) {
        e = mlora::launch_long_expand(pool->r_bucket_max, mode, p, long_tiles, stream);
        if (e != cudaSuccess) return MLORA_ERR_CUDA;
    }
    return MLORA_OK;
}

}  // namespace

// Fused apply whose long-segment workspace is caller-provided memory (no allocation);
// used by mlora_apply_noalloc.  Same checks as mlora_apply, plus the size limit.
mlora_status mlora_apply_with_workspace(mlora_pool *pool, const mlora_segments *segs,
                                        const void *X, int64_t ldx, void *Y, int64_t ldy,
                                        void *stream, float *ws, size_t ws_bytes)
{
    mlora_status st = check_segments(pool, segs);
    if (st != MLORA_OK) return st;
    // only batches that take the long-segment kernels use the workspace
    if (long_path(pool, segs) &&
        (size_t)segs->n_tokens * std::max(16, pool->r_bucket_max) * sizeof(float) > ws_bytes)
        return MLORA_ERR_UNSUPPORTED;
    if (segs->n_segments == 0 || segs->n_tokens == 0) return MLORA_OK;
    if (X == nullptr || Y == nullptr || !aligned16(X) || !aligned16(Y)) return MLORA_ERR_INVALID_ARG;
    if (ldx < pool->d_in || ldx % 8 != 0 || ldy < pool->d_out || ldy % 8 != 0)
        return MLORA_ERR_INVALID_ARG;
    DeviceGuard guard(pool->device);
    if (!guard.ok) return MLORA_ERR_CUDA;
    mlora::TileParams p = base_params(pool, segs);
    p.X = static_cast<const __nv_bfloat16 *>(X);
    p.ldx = ldx;
    p.Y = static_cast<__nv_bfloat16 *>(Y);
    p.ldy = ldy;
    return launch(pool, segs, mlora::MODE_APPLY, p, stream, ws, ws_bytes);
}

int mlora_pool_device(const mlora_pool *pool) { return pool ? pool->device : -1; }

extern "C" {

const char *mlora_status_string(mlora_status status)
{
    switch (status) {
    case MLORA_OK: return "ok";
    case MLORA_ERR_INVALID_ARG: return "invalid argument";
    case MLORA_ERR_UNSUPPORTED: return "unsupported shape or device";
    case MLORA_ERR_OUT_OF_MEMORY: return "out of device memory";
    case MLORA_ERR_BAD_METADATA: return "device flagged bad segment metadata";
    case MLORA_ERR_CUDA: return "CUDA runtime error";
    case MLORA_ERR_NO_SLOT: return "every slot is pinned";
    }
    return "unknown status";
}

int32_t mlora_version(void) { return 100; }

mlora_status mlora_pool_create(int32_t d_in, int32_t d_out, int32_t n_slots, int32_t r_max,
                               mlora_pool **out)
{
    if (out == nullptr) return MLORA_ERR_INVALID_ARG;
    *out = nullptr;
    if (d_in <= 0 || d_out <= 0 || n_slots <= 0 || r_max <= 0) return MLORA_ERR_INVALID_ARG;
    if (d_in % 8 != 0 || d_out % 8 != 0 || r_max > 64) return MLORA_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MLORA_ERR_CUDA;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MLORA_ERR_CUDA;
    if (prop.major != 10 || prop.minor != 0) return MLORA_ERR_UNSUPPORTED;   // built for sm_100a

    const int rb = rank_bucket(r_max);
    const int64_t stride = round_up((int64_t)rb * (d_in + d_out), 128);   // 256-byte slots
    const double bytes = (double)stride * 2.0 * n_slots;
    if (bytes > 9.0e18) return MLORA_ERR_OUT_OF_MEMORY;

    mlora_pool *pool = new (std::nothrow) mlora_pool();
    if (pool == nullptr) return MLORA_ERR_OUT_OF_MEMORY;
    pool->device = dev;
    pool->d_in = d_in;
    pool->d_out = d_out;
    pool->n_slots = n_slots;
    pool->r_max = r_max;
    pool->r_bucket_max = rb;
    pool->slot_stride = stride;
    pool->b_offset = (int64_t)rb * d_in;
    pool->buf = nullptr;
    pool->d_rank = nullptr;
    pool->d_scale = nullptr;
    pool->d_gen = nullptr;
    pool->d_status = nullptr;
    pool->ws = nullptr;
    pool->ws_bytes = 0;
    pool->h_rank.assign(n_slots, 0);
    pool->h_alpha.assign(n_slots, 0.f);
    pool->h_gen.assign(n_slots, 0u);

    mlora_status st = MLORA_OK;
    if (cudaMalloc(&pool->buf, (size_t)stride * 2 * n_slots) != cudaSuccess ||
        cudaMalloc(&pool->d_rank, sizeof(int32_t) * n_slots) != cudaSuccess ||
        cudaMalloc(&pool->d_scale, sizeof(float) * n_slots) != cudaSuccess ||
        cudaMalloc(&pool->d_gen, sizeof(uint32_t) * n_slots) != cudaSuccess ||
        cudaMalloc(&pool->d_status, sizeof(unsigned int)) != cudaSuccess) {
        st = MLORA_ERR_OUT_OF_MEMORY;
    } else if (cudaMemset(pool->d_rank, 0, sizeof(int32_t) * n_slots) != cudaSuccess ||
               cudaMemset(pool->d_scale, 0, sizeof(float) * n_slots) != cudaSuccess ||
               cudaMemset(pool->d_gen, 0, sizeof(uint32_t) * n_slots) != cudaSuccess ||
               cudaMemset(pool->d_status, 0, sizeof(unsigned int)) != cudaSuccess ||
               cudaDeviceSynchronize() != cudaSuccess) {
        st = MLORA_ERR_CUDA;
    } else {
        st = prepare_device(dev);
    }
    // the no-allocation entry point's scratch array is reserved here, with the pool's
    // device current, rather than by its first call
    if (st == MLORA_OK) st = mlora_noalloc_reserve(dev);
    if (st == MLORA_OK) {
        pool->b_maps_ok = tensor_map_encoder() != nullptr;
        for (int i = 0; i < 4 && pool->b_maps_ok; ++i)
            if ((8 << i) <= rb)
                pool->b_maps_ok = encode_b_map(&pool->b_maps[i], pool, 8 << i, mlora::kExpandChunk);
        pool->b_maps_wide_ok = pool->b_maps_ok && pool->d_out % 32 == 0;
        for (int i = 0; i < 4 && pool->b_maps_wide_ok; ++i)
            if ((8 << i) <= rb) pool->b_maps_wide_ok = encode_b_map_wide(&pool->b_maps_wide[i], pool, 8 << i);
    }
    if (st != MLORA_OK) {
        cudaGetLastError();   // clear a sticky allocation error
        mlora_pool_destroy(pool);
        return st;
    }
    *out = pool;
    return MLORA_OK;
}

mlora_status mlora_pool_destroy(mlora_pool *pool)
{
    if (pool == nullptr) return MLORA_OK;
    DeviceGuard guard(pool->device);
    cudaDeviceSynchronize();
    if (pool->buf) cudaFree(pool->buf);
    if (pool->d_rank) cudaFree(pool->d_rank);
    if (pool->d_scale) cudaFree(pool->d_scale);
    if (pool->d_gen) cudaFree(pool->d_gen);
    if (pool->d_status) cudaFree(pool->d_status);
    if (pool->ws) {   // stream-ordered allocation: freed the same way, then waited for
        cudaFreeAsync(pool->ws, nullptr);
        cudaDeviceSynchronize();
    }
    delete pool;
    return MLORA_OK;
}

mlora_status mlora_pool_shape(const mlora_pool *pool, int32_t *d_in, int32_t *d_out,
                              int32_t *n_slots, int32_t *r_max)
{
    if (pool == nullptr) return MLORA_ERR_INVALID_ARG;
    if (d_in) *d_in = pool->d_in;
    if (d_out) *d_out = pool->d_out;
    if (n_slots) *n_slots = pool->n_slots;
    if (r_max) *r_max = pool->r_max;
    return MLORA_OK;
}

mlora_status mlora_pool_load_slot(mlora_pool *pool, int32_t slot, int32_t rank, float alpha,
                                  const void *A, const void *B, int32_t src_is_device,
                                  void *stream)
{
    if (pool == nullptr || A == nullptr || B == nullptr) return MLORA_ERR_INVALID_ARG;
    if (slot < 0 || slot >= pool->n_slots) return MLORA_ERR_INVALID_ARG;
    if (rank < 1 || rank > pool->r_max) return MLORA_ERR_INVALID_ARG;
    if (!std::isfinite(alpha)) return MLORA_ERR_INVALID_ARG;
    if (src_is_device && ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(B)) & 1u))
        return MLORA_ERR_INVALID_ARG;
    DeviceGuard guard(pool->device);
    if (!guard.ok) return MLORA_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int R = rank_bucket(rank);
    const size_t a_elems = (size_t)rank * pool->d_in;
    const size_t b_elems = (size_t)pool->d_out * rank;
    const __nv_bfloat16 *a_src = static_cast<const __nv_bfloat16 *>(A);
    const __nv_bfloat16 *b_src = static_cast<const __nv_bfloat16 *>(B);
    __nv_bfloat16 *staging = nullptr;
    if (!src_is_device) {
        // Copy into stream-ordered staging first: a failed copy leaves the slot untouched.
        if (cudaMallocAsync(&staging, (a_elems + b_elems) * 2, st) != cudaSuccess) {
            cudaGetLastError();
            return MLORA_ERR_OUT_OF_MEMORY;
        }
        if (cudaMemcpyAsync(staging, A, a_elems * 2, cudaMemcpyHostToDevice, st) != cudaSuccess ||
            cudaMemcpyAsync(staging + a_elems, B, b_elems * 2, cudaMemcpyHostToDevice, st) !=
                cudaSuccess) {
            cudaGetLastError();
            cudaFreeAsync(staging, st);
            return MLORA_ERR_CUDA;
        }
        a_src = staging;
        b_src = staging + a_elems;
    }
    const float scale = alpha / (float)rank;
    const uint32_t gen = pool->h_gen[slot] + 1;
    cudaError_t e = mlora::launch_repack_slot(pool->buf + (int64_t)slot * pool->slot_stride,
                                              pool->b_offset, R, rank, pool->d_in, pool->d_out,
                                              a_src, b_src, pool->d_rank + slot,
                                              pool->d_scale + slot, scale, pool->d_gen + slot, gen, st);
    if (staging) cudaFreeAsync(staging, st);
    if (e != cudaSuccess) return MLORA_ERR_CUDA;
    pool->h_rank[slot] = rank;
    pool->h_alpha[slot] = alpha;
    pool->h_gen[slot] = gen;
    return MLORA_OK;
}

mlora_status mlora_pool_clear_slot(mlora_pool *pool, int32_t slot, void *stream)
{
    if (pool == nullptr || slot < 0 || slot >= pool->n_slots) return MLORA_ERR_INVALID_ARG;
    DeviceGuard guard(pool->device);
    if (!guard.ok) return MLORA_ERR_CUDA;
    const uint32_t gen = pool->h_gen[slot] + 1;
    if (mlora::launch_publish_slot(pool->d_rank + slot, pool->d_scale + slot, pool->d_gen + slot, 0, 0.f,
                                   gen, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return MLORA_ERR_CUDA;
    pool->h_rank[slot] = 0;
    pool->h_alpha[slot] = 0.f;
    pool->h_gen[slot] = gen;
    return MLORA_OK;
}

mlora_status mlora_pool_slot_generation(const mlora_pool *pool, int32_t slot, uint32_t *generation)
{
    if (pool == nullptr || generation == nullptr || slot < 0 || slot >= pool->n_slots)
        return MLORA_ERR_INVALID_ARG;
    *generation = pool->h_gen[slot];
    return MLORA_OK;
}

mlora_status mlora_pool_slot_info(const mlora_pool *pool, int32_t slot, int32_t *rank,
                                  float *alpha, int64_t *params)
{
    if (pool == nullptr || slot < 0 || slot >= pool->n_slots) return MLORA_ERR_INVALID_ARG;
    const int32_t r = pool->h_rank[slot];
    if (rank) *rank = r;
    if (alpha) *alpha = pool->h_alpha[slot];
    if (params) *params = (int64_t)r * ((int64_t)pool->d_in + pool->d_out);
    return MLORA_OK;
}

mlora_status mlora_pool_check(mlora_pool *pool, void *stream, uint32_t *flags)
{
    if (pool == nullptr) return MLORA_ERR_INVALID_ARG;
    DeviceGuard guard(pool->device);
    if (!guard.ok) return MLORA_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned int h = 0;
    if (cudaMemcpyAsync(&h, pool->d_status, sizeof h, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaMemsetAsync(pool->d_status, 0, sizeof(unsigned int), st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return MLORA_ERR_CUDA;
    if (flags) *flags = h;
    return h ? MLORA_ERR_BAD_METADATA : MLORA_OK;
}

mlora_status mlora_apply(mlora_pool *pool, const mlora_segments *segs, const void *X, int64_t ldx,
                         void *Y, int64_t ldy, void *stream)
{
    mlora_status st = check_segments(pool, segs);
    if (st != MLORA_OK) return st;
    if (segs->n_segments == 0 || segs->n_tokens == 0) return MLORA_OK;
    if (X == nullptr || Y == nullptr || !aligned16(X) || !aligned16(Y)) return MLORA_ERR_INVALID_ARG;
    if (ldx < pool->d_in || ldx % 8 != 0 || ldy < pool->d_out || ldy % 8 != 0)
        return MLORA_ERR_INVALID_ARG;
    DeviceGuard guard(pool->device);
    if (!guard.ok) return MLORA_ERR_CUDA;
    mlora::TileParams p = base_params(pool, segs);
    p.X = static_cast<const __nv_bfloat16 *>(X);
    p.ldx = ldx;
    p.Y = static_cast<__nv_bfloat16 *>(Y);
    p.ldy = ldy;
    return launch(pool, segs, mlora::MODE_APPLY, p, stream);
}

mlora_status mlora_apply_ex(mlora_pool *pool, const mlora_segments *segs, const void *X, int32_t x_dtype,
                            float x_scale, int64_t ldx, void *Y, int32_t y_dtype, int64_t ldy, void *stream)
{
    if (x_dtype != MLORA_DTYPE_BF16 && x_dtype != MLORA_DTYPE_FP8_E4M3) return MLORA_ERR_INVALID_ARG;
    if (y_dtype != MLORA_DTYPE_BF16 && y_dtype != MLORA_DTYPE_FP16 && y_dtype != MLORA_DTYPE_FP32)
        return MLORA_ERR_INVALID_ARG;
    if (x_dtype == MLORA_DTYPE_BF16 && y_dtype == MLORA_DTYPE_BF16)
        return mlora_apply(pool, segs, X, ldx, Y, ldy, stream);
    mlora_status st = check_segments(pool, segs);
    if (st != MLORA_OK) return st;
    const bool x8 = x_dtype == MLORA_DTYPE_FP8_E4M3;
    if (x8 && (!std::isfinite(x_scale) || pool->d_in % 16 != 0)) return MLORA_ERR_INVALID_ARG;
    if (segs->n_segments == 0 || segs->n_tokens == 0) return MLORA_OK;
    if (X == nullptr || Y == nullptr || !aligned16(X) || !aligned16(Y)) return MLORA_ERR_INVALID_ARG;
    // rows of whole 16-byte vectors
    const int64_t x_vec = x8 ? 16 : 8, y_vec = y_dtype == MLORA_DTYPE_FP32 ? 4 : 8;
    if (ldx < pool->d_in || ldx % x_vec != 0 || ldy < pool->d_out || ldy % y_vec != 0) return MLORA_ERR_INVALID_ARG;
    DeviceGuard guard(pool->device);
    if (!guard.ok) return MLORA_ERR_CUDA;
    mlora::TileParams p = base_params(pool, segs);
    p.X = static_cast<const __nv_bfloat16 *>(X);   // (element type per x_dtype)
    p.ldx = ldx;
    p.Y = static_cast<__nv_bfloat16 *>(Y);         // (element type per y_dtype)
    p.ldy = ldy;
    p.x_scale = x8 ? x_scale : 1.f;
    const int c = choose_cluster(pool->d_in, pool->d_out);
    p.k_slice = (int32_t)round_up((pool->d_in + c - 1) / c, 32);
    p.n_slice = (int32_t)round_up((pool->d_out + c - 1) / c, 8);
    set_single_projection(p);
    // every segment takes the decode-shaped kernel (the tensor-memory kernels are bf16 only)
    p.long_rows = 0x7fffffff;
    p.early = 1;
    st = prepare_device(pool->device);
    if (st != MLORA_OK) return st;
    const int dt = 3 * (x8 ? 1 : 0) + (y_dtype == MLORA_DTYPE_FP16 ? 1 : y_dtype == MLORA_DTYPE_FP32 ? 2 : 0);
    const int64_t tiles = (int64_t)segs->n_segments + (int64_t)segs->n_tokens / mlora::kTileRows + 1;
    if (mlora::launch_tile_kernel_dt(dt, pool->r_bucket_max, p, c, tiles, static_cast<cudaStream_t>(stream)) !=
        cudaSuccess)
        return MLORA_ERR_CUDA;
    return MLORA_OK;
}

mlora_status mlora_base_gemm_apply(mlora_pool *pool, const mlora_segments *segs, const void *X, int64_t ldx,
                                   const void *W, int64_t ldw, void *Y, int64_t ldy, void *stream)
{
    mlora_status st = check_segments(pool, segs);
    if (st != MLORA_OK) return st;
    if (segs->n_rows == 0) return MLORA_OK;
    if (X == nullptr || W == nullptr || Y == nullptr || !aligned16(X) || !aligned16(W) || !aligned16(Y))
        return MLORA_ERR_INVALID_ARG;
    if (ldx < pool->d_in || ldx % 8 != 0 || ldw < pool->d_in || ldw % 8 != 0 || ldy < pool->d_out ||
        ldy % 8 != 0)
        return MLORA_ERR_INVALID_ARG;
    if (!pool->b_maps_ok) return MLORA_ERR_UNSUPPORTED;
    DeviceGuard guard(pool->device);
    if (!guard.ok) return MLORA_ERR_CUDA;
    st = prepare_device(pool->device);
    if (st != MLORA_OK) return st;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    const int rk = std::max(16, pool->r_bucket_max);
    const int64_t n_mblk = (segs->n_rows + mlora::kGemmRows - 1) / mlora::kGemmRows;
    const int gn = mlora::choose_gemm_cols((int)n_mblk, pool->d_out);
    const int64_t n_nblk = (pool->d_out + gn - 1) / gn;
    // workspace: H (grouped order), the row map, the slot lists of the row blocks
    const size_t h_bytes = (size_t)round_up((int64_t)segs->n_tokens * rk * 4, 256);
    const size_t map_bytes = (size_t)round_up((int64_t)segs->n_rows * 16, 256);
    const size_t slot_bytes = (size_t)n_mblk * mlora::kBlockSlotsPitch * 4;
    std::lock_guard<std::mutex> lock(pool->ws_mutex);   // held until the kernels are launched
    st = ensure_workspace(pool, h_bytes + map_bytes + slot_bytes, cs);
    if (st != MLORA_OK) return st;
    uint8_t *ws = reinterpret_cast<uint8_t *>(pool->ws);
    float *H = reinterpret_cast<float *>(ws);
    int4 *row_info = reinterpret_cast<int4 *>(ws + h_bytes);
    int32_t *block_slots = reinterpret_cast<int32_t *>(ws + h_bytes + map_bytes);

    // 1. each row's grouped position, slot, scale and rank; each row block's slots
    mlora::TileParams p = base_params(pool, segs);
    p.X = static_cast<const __nv_bfloat16 *>(X);
    p.ldx = ldx;
    p.H = H;
    p.ldh = rk;
    if (mlora::launch_row_map(p, row_info, cs) != cudaSuccess ||
        mlora::launch_block_slots(row_info, segs->n_rows, block_slots, cs) != cudaSuccess)
        return MLORA_ERR_CUDA;
    // 2. H = X A^T for every valid segment (decode-shaped and long-segment kernels)
    const bool shrink = segs->n_segments > 0 && segs->n_tokens > 0;
    if (shrink) {
        st = launch(pool, segs, mlora::MODE_SHRINK, p, stream);
        if (st != MLORA_OK) return st;
    }
    // The GEMM reads H only in its LoRA steps, after griddepcontrol.wait, so it may
    // start while the long-segment shrink finishes (programmatic dependent launch).
    // Only then: that shrink follows a plainly launched kernel, so everything before it
    // (the row map, X) is complete when the GEMM starts.
    const bool pdl = shrink && long_path(pool, segs);
    // 3. Y = X W^T + s (H B^T) per tile
    mlora::GemmParams g{};
    // each CTA of a pair loads 128-row boxes of X and W
    if (!encode_rows_map(&g.x_map, X, segs->n_rows, pool->d_in, ldx, mlora::kGemmRows / 2) ||
        !encode_rows_map(&g.w_map, W, pool->d_out, pool->d_in, ldw, mlora::kGemmRows / 2))
        return MLORA_ERR_CUDA;
    for (int i = 0; i < 4; ++i) g.b_map[i] = pool->b_maps_wide_ok ? pool->b_maps_wide[i] : pool->b_maps[i];
    g.b_col_div = pool->b_maps_wide_ok ? 32 : 1;
    g.row_info = row_info;
    g.block_slots = block_slots;
    g.H = H;
    g.ldh = rk;
    g.Y = static_cast<__nv_bfloat16 *>(Y);
    g.ldy = ldy;
    g.status = pool->d_status;
    g.n_rows = segs->n_rows;
    g.d_in = pool->d_in;
    g.d_out = pool->d_out;
    g.n_mblk = (int32_t)n_mblk;
    g.n_nblk = (int32_t)n_nblk;
    return mlora::launch_base_gemm(gn, g, cs, pdl) == cudaSuccess ? MLORA_OK : MLORA_ERR_CUDA;
}

mlora_status mlora_apply_multi(mlora_pool *const *pools, int32_t n_proj, const mlora_segments *segs,
                               const void *X, int64_t ldx, void *const *Y, const int64_t *ldy,
                               void *stream)
{
    if (pools == nullptr || Y == nullptr || ldy == nullptr) return MLORA_ERR_INVALID_ARG;
    if (n_proj < 1 || n_proj > MLORA_MAX_FUSED) return MLORA_ERR_INVALID_ARG;
    mlora_pool *const p0 = pools[0];
    mlora_status st = check_segments(p0, segs);
    if (st != MLORA_OK) return st;
    for (int k = 0; k < n_proj; ++k) {
        const mlora_pool *q = pools[k];
        if (q == nullptr || q->device != p0->device || q->d_in != p0->d_in || q->n_slots != p0->n_slots)
            return MLORA_ERR_INVALID_ARG;
        for (int j = 0; j < k; ++j)
            if (pools[j] == q || Y[j] == Y[k]) return MLORA_ERR_INVALID_ARG;
    }
    if (segs->n_segments == 0 || segs->n_tokens == 0) return MLORA_OK;
    if (X == nullptr || !aligned16(X) || ldx < p0->d_in || ldx % 8 != 0) return MLORA_ERR_INVALID_ARG;
    for (int k = 0; k < n_proj; ++k)
        if (Y[k] == nullptr || !aligned16(Y[k]) || ldy[k] < pools[k]->d_out || ldy[k] % 8 != 0)
            return MLORA_ERR_INVALID_ARG;
    DeviceGuard guard(p0->device);
    if (!guard.ok) return MLORA_ERR_CUDA;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);

    // one cluster shape for all projections: d_in is shared, each d_out is sliced alike
    int c = 8, rmax = 8;
    bool use_long = true;
    for (int k = 0; k < n_proj; ++k) {
        c = std::min(c, choose_cluster(p0->d_in, pools[k]->d_out));
        rmax = std::max(rmax, pools[k]->r_bucket_max);
        use_long = use_long && long_path(pools[k], segs);
    }
    st = prepare_device(p0->device);
    if (st != MLORA_OK) return st;
    if (use_long) {
        // every projection's long-segment workspace first, so that a failure launches nothing
        const size_t bytes = (size_t)segs->n_tokens * std::max(16, rmax) * sizeof(float);
        for (int k = 0; k < n_proj; ++k) {
            std::lock_guard<std::mutex> lock(pools[k]->ws_mutex);
            st = ensure_workspace(pools[k], bytes, cs);
            if (st != MLORA_OK) return st;
        }
    }

    mlora::TileParams p = base_params(p0, segs);
    p.X = static_cast<const __nv_bfloat16 *>(X);
    p.ldx = ldx;
    p.Y = static_cast<__nv_bfloat16 *>(Y[0]);
    p.ldy = ldy[0];
    p.k_slice = (int32_t)round_up((p0->d_in + c - 1) / c, 32);
    p.n_slice = (int32_t)round_up((p0->d_out + c - 1) / c, 8);
    p.n_proj = n_proj;
    for (int k = 0; k < n_proj; ++k) {
        const mlora_pool *q = pools[k];
        p.proj[k] = mlora::ProjView{q->buf, q->slot_stride, q->b_offset, q->d_rank, q->d_scale, q->d_gen,
                                    q->d_status, q->d_out,
                                    (int32_t)round_up((q->d_out + c - 1) / c, 8),
                                    static_cast<__nv_bfloat16 *>(Y[k]), ldy[k]};
    }
    p.long_rows = use_long ? kLongRows : 0x7fffffff;
    p.early = use_long ? 0 : 1;
    const int64_t tiles = (int64_t)segs->n_segments + (int64_t)segs->n_tokens / mlora::kTileRows + 1;
    if (mlora::launch_tile_kernel_fused(rmax, p, c, tiles * n_proj, cs) != cudaSuccess)
        return MLORA_ERR_CUDA;
    if (!use_long) return MLORA_OK;
    // Pools of one rank bucket share one shrink launch: X's prefill rows are read once
    // for all projections, and each projection's H lands in its own workspace.
    // (The launch takes each slot's rank from pool 0 and computes projection k only where
    // pool k holds the slot at that rank, so the pools' ranks must agree slot by slot; an
    // adapter with another rank per target module takes one shrink per projection.)
    bool one_shrink = n_proj > 1;
    for (int k = 1; k < n_proj; ++k)
        one_shrink = one_shrink && pools[k]->r_bucket_max == p0->r_bucket_max && pools[k]->h_rank == p0->h_rank;
    if (one_shrink) {
        const int rk = std::max(16, p0->r_bucket_max);
        mlora::TileParams q = p;
        st = setup_long_shrink(p0, segs, q);
        if (st != MLORA_OK) return st;
        q.ws = p0->ws;
        q.ws_ld = rk;
        for (int k = 0; k < n_proj; ++k) {
            q.proj[k].ws = pools[k]->ws;
            q.proj[k].ws_ld = rk;
        }
        if (mlora::launch_long_shrink(p0->r_bucket_max, q, long_tile_bound(segs), cs, n_proj) != cudaSuccess)
            return MLORA_ERR_CUDA;
    }
    for (int k = 0; k < n_proj; ++k) {
        mlora::TileParams q = base_params(pools[k], segs);
        q.X = p.X;
        q.ldx = ldx;
        q.Y = static_cast<__nv_bfloat16 *>(Y[k]);
        q.ldy = ldy[k];
        st = launch_long(pools[k], segs, mlora::MODE_APPLY, q, cs, nullptr, 0, !one_shrink);
        if (st != MLORA_OK) return st;
    }
    return MLORA_OK;
}

mlora_status mlora_shrink(mlora_pool *pool, const mlora_segments *segs, const void *X,
                          int64_t ldx, float *H, int64_t ldh, void *stream)
{
    mlora_status st = check_segments(pool, segs);
    if (st != MLORA_OK) return st;
    if (segs->n_segments == 0 || segs->n_tokens == 0) return MLORA_OK;
    if (X == nullptr || H == nullptr || !aligned16(X) || !aligned16(H)) return MLORA_ERR_INVALID_ARG;
    if (ldx < pool->d_in || ldx % 8 != 0 || ldh < pool->r_max || ldh % 4 != 0)
        return MLORA_ERR_INVALID_ARG;
    DeviceGuard guard(pool->device);
    if (!guard.ok) return MLORA_ERR_CUDA;
    mlora::TileParams p = base_params(pool, segs);
    p.X = static_cast<const __nv_bfloat16 *>(X);
    p.ldx = ldx;
    p.H = H;
    p.ldh = ldh;
    return launch(pool, segs, mlora::MODE_SHRINK, p, stream);
}

mlora_status mlora_expand(mlora_pool *pool, const mlora_segments *segs, const float *H,
                          int64_t ldh, void *Y, int64_t ldy, void *stream)
{
    mlora_status st = check_segments(pool, segs);
    if (st != MLORA_OK) return st;
    if (segs->n_segments == 0 || segs->n_tokens == 0) return MLORA_OK;
    if (H == nullptr || Y == nullptr || !aligned16(H) || !aligned16(Y)) return MLORA_ERR_INVALID_ARG;
    if (ldh < pool->r_max || ldh % 4 != 0 || ldy < pool->d_out || ldy % 8 != 0)
        return MLORA_ERR_INVALID_ARG;
    DeviceGuard guard(pool->device);
    if (!guard.ok) return MLORA_ERR_CUDA;
    mlora::TileParams p = base_params(pool, segs);
    p.H = const_cast<float *>(H);
    p.ldh = ldh;
    p.Y = static_cast<__nv_bfloat16 *>(Y);
    p.ldy = ldy;
    return launch(pool, segs, mlora::MODE_EXPAND, p, stream);
}

mlora_status mlora_build_segments(const int32_t *row_slots, int32_t n_rows, int32_t *offsets,
                                  int32_t *slots, int32_t *token_indices, int32_t *n_segments,
                                  int32_t *max_segment_rows, const mlora_pool *pool,
                                  int32_t *ranks)
{
    if (n_rows < 0 || offsets == nullptr || n_segments == nullptr) return MLORA_ERR_INVALID_ARG;
    if (n_rows > 0 && (row_slots == nullptr || slots == nullptr || token_indices == nullptr))
        return MLORA_ERR_INVALID_ARG;
    // Pass 1: segment id of each row in order of first appearance, and counts.
    std::unordered_map<int32_t, int32_t> seg_of;
    seg_of.reserve((size_t)std::min<int32_t>(n_rows, 1 << 16) + 1);
    std::vector<int32_t> counts;
    std::vector<int32_t> row_seg((size_t)n_rows);
    for (int32_t t = 0; t < n_rows; ++t) {
        auto it = seg_of.find(row_slots[t]);
        int32_t g;
        if (it == seg_of.end()) {
            g = (int32_t)counts.size();
            seg_of.emplace(row_slots[t], g);
            slots[g] = row_slots[t];
            counts.push_back(0);
        } else {
            g = it->second;
        }
        row_seg[t] = g;
        ++counts[g];
    }
    const int32_t S = (int32_t)counts.size();
    // Pass 2: offsets; pass 3: stable scatter of rows to grouped positions.
    offsets[0] = 0;
    for (int32_t g = 0; g < S; ++g) offsets[g + 1] = offsets[g] + counts[g];
    std::vector<int32_t> cursor(offsets, offsets + S);
    for (int32_t t = 0; t < n_rows; ++t) token_indices[cursor[row_seg[t]]++] = t;
    // the longest adapter segment whose rows are consecutive (rows keep their order, so
    // first and last decide): only such segments can go to the tensor-memory kernels
    int32_t longest = 0;
    for (int32_t g = 0; g < S; ++g)
        if (slots[g] >= 0 && counts[g] > 0 &&
            token_indices[offsets[g + 1] - 1] - token_indices[offsets[g]] == counts[g] - 1)
            longest = std::max(longest, counts[g]);
    *n_segments = S;
    // at least 1: in mlora_segments a hint of 0 means "unknown", which would send a
    // batch without any run of consecutive rows to the long-segment kernels
    if (max_segment_rows) *max_segment_rows = std::max(longest, 1);
    if (pool != nullptr && ranks != nullptr) {
        for (int32_t g = 0; g < S; ++g) {
            const int32_t a = slots[g];
            ranks[g] = (a >= 0 && a < pool->n_slots) ? pool->h_rank[a] : 0;
        }
    }
    return MLORA_OK;
}

}  // extern "C"
