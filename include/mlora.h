/*
 * mlora.h -- C ABI of the heterogeneous-batch LoRA branch for B200 (sm_100a).
 *
 * The operation (page "Multi-LoRA Serving: adapter batching", charlestar.github.io,
 * sections "LoRA on one Linear layer", "The math of a mixed batch" and
 * "What metadata a segmented kernel needs"):
 *
 *   A linear layer Y = X W^T (W in R^{d_out x d_in}) gains, per adapter a, the
 *   low-rank branch  s_a (X A_a^T) B_a^T  with A_a in R^{r x d_in},
 *   B_a in R^{d_out x r} and s_a = alpha_a / r_a.  The caller computes the shared
 *   base output Y0 = X W^T for every row; this library adds each row's own
 *   adapter delta in place:
 *
 *       H[p, j]  = sum_k X[t, k] A_a[j, k]            (shrink, fp32 accumulation)
 *       Y[t, o]  = bf16( Y0[t, o] + s_g sum_j H[p, j] B_a[o, j] )   (expand, scatter)
 *
 *   where the rows are grouped into segments g (slot a = adapter_slots[g];
 *   slot -1 = base model only) and grouped position p of segment g maps to the
 *   original row t = token_indices[p].  Rows of base segments, rows in no
 *   segment and rows of rejected segments are never written (bit-identical Y0).
 *
 * Adapters live in a pre-allocated pool of fixed-stride slots indexed by slot
 * number (page "LoRA/QLoRA multi-tenant serving", ybb.press, section 1.1, unified
 * size alignment).  Ranks up to 64 are stored and computed at their own rank
 * bucket (8, 16, 32 or 64; page "Multi-LoRA Serving: adapter batching", section
 * "How LoRA ranks affect the kernel"), never padded to the pool's maximum.
 *
 * Conventions for every entry point:
 *   - bf16 tensors are IEEE bfloat16 bit patterns (2 bytes per element),
 *     row-major with an element row stride (ld*).
 *   - "device" pointers are CUDA device pointers of the device current when the
 *     pool was created; calls must be made with that device current.
 *   - stream is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Kernels are launched asynchronously on it; the caller keeps every buffer
 *     alive until the stream has passed the call.
 *   - Errors the host can see (null or misaligned pointers, bad sizes, slot or
 *     rank out of range) return at once with nothing launched.  Errors only the
 *     device can see (bad metadata contents) make the kernels skip the offending
 *     segment or row -- never trap -- and set bits in the pool's device status
 *     word, which mlora_pool_check reports.
 *   - Limits: d_in and d_out multiples of 8 (16-byte rows); rank 1..64;
 *     X, Y 16-byte aligned with ld* a multiple of 8; H 16-byte aligned with
 *     ldh a multiple of 4.
 */
#ifndef MLORA_H
#define MLORA_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MLORA_OK = 0,
    MLORA_ERR_INVALID_ARG = 1,     /* null/misaligned pointer, size or index out of range */
    MLORA_ERR_UNSUPPORTED = 2,     /* shape outside the supported limits, no sm_100 device */
    MLORA_ERR_OUT_OF_MEMORY = 3,   /* device allocation failed */
    MLORA_ERR_BAD_METADATA = 4,    /* mlora_pool_check: the device flagged bad metadata */
    MLORA_ERR_CUDA = 5,            /* a CUDA runtime call failed */
    MLORA_ERR_NO_SLOT = 6          /* mlora_slot_cache_acquire: every slot is pinned */
} mlora_status;

/* Device status bits reported by mlora_pool_check. */
#define MLORA_FLAG_BAD_OFFSETS  1u   /* offsets decreasing, negative or beyond n_tokens */
#define MLORA_FLAG_BAD_SLOT     2u   /* adapter slot < -1 or >= n_slots */
#define MLORA_FLAG_BAD_RANK     4u   /* ranks[g] differs from the rank loaded in the slot */
#define MLORA_FLAG_BAD_ROW      8u   /* token_indices entry outside [0, n_rows) */
#define MLORA_FLAG_SLOT_EMPTY  16u   /* segment refers to a slot with nothing loaded */
#define MLORA_FLAG_TIMEOUT     32u   /* an internal wait gave up (results of that tile invalid) */
#define MLORA_FLAG_STALE_SLOT  64u   /* the slot holds another generation than the batch was
                                        built for (mlora_segments.generations) */

/* Opaque adapter pool.  Owns its device slot buffer, slot table and status word. */
typedef struct mlora_pool mlora_pool;

/*
 * Segment metadata for one call (page "Multi-LoRA Serving: adapter batching",
 * section "What metadata a segmented kernel needs": segment_offsets,
 * adapter_slots, token_indices, ranks, scales).  All arrays are DEVICE memory,
 * owned by the caller, read-only to the library.
 */
typedef struct {
    int32_t n_segments;              /* S >= 0 */
    int32_t n_rows;                  /* rows of X and Y; token_indices values must be < n_rows */
    int32_t n_tokens;                /* grouped positions: length of token_indices
                                        (== segment_offsets[S] for well-formed metadata);
                                        rows of H in mlora_shrink / mlora_expand */
    int32_t max_segment_rows;        /* host hint: an upper bound on the length of any
                                        adapter segment whose rows are consecutive in X
                                        and Y (the only segments the tensor-memory
                                        kernels take), or 0 if unknown.  Only steers
                                        kernel choice; a wrong hint never changes results. */
    const int32_t *segment_offsets;  /* [S+1], non-decreasing, offsets[0] >= 0 */
    const int32_t *adapter_slots;    /* [S], -1 = base model only, else 0..n_slots-1 */
    const int32_t *ranks;            /* [S] or NULL; if given, must equal the slot's rank
                                        (entries of base segments are ignored) */
    const float *scales;             /* [S] or NULL (then each slot's alpha / rank) */
    const int32_t *token_indices;    /* [n_tokens] grouped position -> original row, no
                                        duplicates; NULL = identity (p -> row p) */
    const uint32_t *generations;     /* [S] or NULL: the generation of each adapter
                                        segment's slot the batch was built for (see
                                        mlora_pool_slot_generation); a segment whose slot
                                        has since been reloaded or cleared is skipped and
                                        flagged MLORA_FLAG_STALE_SLOT.  Base entries are
                                        ignored. */
} mlora_segments;

/*
 * Create a pool of n_slots adapter slots for one projection (d_in -> d_out) with
 * ranks up to r_max (1..64): one pre-allocated buffer of fixed-size slots, so a
 * slot's address is base + slot * stride (page "LoRA/QLoRA multi-tenant serving",
 * ybb.press, section 1.1 on the adapter pool and unified size alignment; page
 * "Multi-LoRA Serving: adapter batching", section "Why the adapter cache needs
 * tiers", on keeping hot adapters resident in GPU memory).  Allocates
 * n_slots * bucket(r_max) * (d_in + d_out) bf16 elements of device memory on the
 * current device; all slots start empty.  It also reserves, once per device, the
 * scratch array of mlora_apply_noalloc.  Returns MLORA_ERR_OUT_OF_MEMORY if an
 * allocation fails, MLORA_ERR_UNSUPPORTED without an sm_100 device or for r_max > 64
 * or d_in, d_out not multiples of 8.
 */
mlora_status mlora_pool_create(int32_t d_in, int32_t d_out, int32_t n_slots, int32_t r_max,
                               mlora_pool **out);

/* Free the pool (synchronises the device first).  NULL is accepted. */
mlora_status mlora_pool_destroy(mlora_pool *pool);

/*
 * Load an adapter into a slot: A is bf16 [rank, d_in] row-major, B is bf16
 * [d_out, rank] row-major (the PEFT layout of lora_A / lora_B), both in host
 * memory (src_is_device = 0) or device memory (1).  The slot is repacked into
 * the pool's internal layout and zero-filled up to its rank bucket, and its
 * generation advances by one.  The load is stream-ordered on `stream`: pageable host
 * sources may be reused when the call returns; page-locked host sources are copied
 * asynchronously and must stay unchanged until the stream has passed the load (so a
 * load on one stream can overlap applies on another that use other slots).
 * On any error the slot keeps its previous contents, rank and generation.
 */
mlora_status mlora_pool_load_slot(mlora_pool *pool, int32_t slot, int32_t rank, float alpha,
                                  const void *A, const void *B, int32_t src_is_device,
                                  void *stream);

/* Mark a slot empty (stream-ordered).  Segments that use it are then rejected. */
mlora_status mlora_pool_clear_slot(mlora_pool *pool, int32_t slot, void *stream);

/*
 * Generation of a slot: 0 for a slot never loaded, then one more with every
 * mlora_pool_load_slot and mlora_pool_clear_slot (host-side counter; the device copy
 * the kernels compare with mlora_segments.generations is updated in stream order by
 * the load or clear).  A serving loop records the generation when it builds a batch,
 * so a batch that runs after its adapter was replaced is rejected rather than
 * applied with the wrong weights (page "Multi-LoRA Serving: adapter batching",
 * section "Eviction cannot look only at LRU": a replaced slot must not serve
 * requests bound to the old adapter).  Loads that run concurrently with applies
 * reading the same slot are the caller's to prevent (pin it, see mlora_slot_cache).
 */
mlora_status mlora_pool_slot_generation(const mlora_pool *pool, int32_t slot, uint32_t *generation);

/* Host-side view of a slot: rank (0 if empty), alpha, and the parameter count
 * r (d_in + d_out) (page "Multi-LoRA Serving: adapter batching", section "LoRA on
 * one Linear layer").  Any output pointer may be NULL. */
mlora_status mlora_pool_slot_info(const mlora_pool *pool, int32_t slot, int32_t *rank,
                                  float *alpha, int64_t *params);

/* Pool geometry.  Any output pointer may be NULL. */
mlora_status mlora_pool_shape(const mlora_pool *pool, int32_t *d_in, int32_t *d_out,
                              int32_t *n_slots, int32_t *r_max);

/*
 * Synchronise `stream`, read and clear the pool's device status word.  Returns
 * MLORA_ERR_BAD_METADATA if any MLORA_FLAG_* bit was set since the last check
 * (the bits are stored to *flags if flags is not NULL), else MLORA_OK.
 */
mlora_status mlora_pool_check(mlora_pool *pool, void *stream, uint32_t *flags);

/*
 * Shrink alone (page "Multi-LoRA Serving: adapter batching", section "What metadata
 * a segmented kernel needs", the shrink step; page "S-LoRA deep dive", section 3 on
 * the segmented gather + GEMM):
 * H[p, 0:r] = X[t_p, :] A_a^T for every grouped position p of every
 * adapter segment, fp32, grouped order (row stride ldh >= r).  X is device bf16
 * [n_rows, d_in] (row stride ldx); H is device fp32 [n_tokens, ldh].  Entries of
 * base or rejected segments and columns >= r are not written.
 */
mlora_status mlora_shrink(mlora_pool *pool, const mlora_segments *segs, const void *X,
                          int64_t ldx, float *H, int64_t ldh, void *stream);

/*
 * Expand alone (page "Multi-LoRA Serving: adapter batching", section "What metadata
 * a segmented kernel needs", the expand and scatter-add steps, with s = alpha / r
 * from section "LoRA on one Linear layer"):
 * Y[t_p, :] = bf16(Y[t_p, :] + s_g H[p, 0:r] B_a^T) for every grouped
 * position p of every adapter segment.  H is device fp32 [n_tokens, ldh] in
 * grouped order; Y is device bf16 [n_rows, d_out] (row stride ldy), updated in
 * place.
 */
mlora_status mlora_expand(mlora_pool *pool, const mlora_segments *segs, const float *H,
                          int64_t ldh, void *Y, int64_t ldy, void *stream);

/*
 * Fused shrink + expand: Y[t, :] = bf16(Y0[t, :] + s_g (X[t, :] A_a^T) B_a^T) in
 * place on the caller's base output Y (= Y0 = X W^T on entry).  For short segments
 * the rank-r intermediate stays on chip; for segments of 128 or more consecutive
 * rows it passes through an fp32 workspace the pool owns (grown, stream-ordered on
 * `stream` with no device-wide synchronisation, when a batch needs more; growth is
 * not possible during stream capture: MLORA_ERR_UNSUPPORTED, so run the largest
 * batch once before capturing).  Calls on one pool whose kernels overlap on the GPU
 * (several streams) share that workspace and race on it: serialise them, give each
 * stream its own pool, or use mlora_shrink / mlora_expand with caller-owned H.
 * X: device bf16 [n_rows, d_in]; Y: device bf16 [n_rows, d_out].
 */
mlora_status mlora_apply(mlora_pool *pool, const mlora_segments *segs, const void *X,
                         int64_t ldx, void *Y, int64_t ldy, void *stream);

/* Element types at the dtype boundary of a quantized base model (mlora_apply_ex). */
#define MLORA_DTYPE_BF16      0
#define MLORA_DTYPE_FP16      1
#define MLORA_DTYPE_FP32      2
#define MLORA_DTYPE_FP8_E4M3  3

/*
 * mlora_apply at the dtype boundary of a quantized base model (page "Multi-LoRA
 * Serving: adapter batching", section "The dtype boundary between a quantized base
 * model and LoRA": the base GEMM's accumulation and output dtype, whether the LoRA
 * branch reuses the activation from before quantization, the dtype and scale of A and
 * B, and where the two paths add).  The answers this entry point gives:
 *   - A and B stay bf16 in the pool, s = alpha / r is applied inside the kernel;
 *   - the LoRA input X is either the bf16 activation from before quantization
 *     (x_dtype MLORA_DTYPE_BF16; x_scale ignored) or the FP8 e4m3 codes the base GEMM
 *     reads (MLORA_DTYPE_FP8_E4M3), whose value is code * x_scale (one per-tensor
 *     scale); the codes are widened exactly, the shrink sums in fp32 and H is scaled by
 *     x_scale before the expand;
 *   - the two paths add once, on the base GEMM's output in its own dtype
 *     (y_dtype MLORA_DTYPE_BF16, _FP16 or _FP32): Y[t, :] = round(Y0[t, :] + s H B^T)
 *     with the sum in fp32 and one rounding to y_dtype (none for fp32).
 * X: device [n_rows, d_in] of x_dtype, row stride ldx elements (a multiple of 16 for
 * FP8 codes, of 8 for bf16; FP8 also needs d_in a multiple of 16); Y: device
 * [n_rows, d_out] of y_dtype, row stride ldy (a multiple of 8, of 4 for fp32); both
 * 16-byte aligned.  The all-bf16 pair is mlora_apply itself.  Other pairs run every
 * segment on the decode-shaped kernel (the tensor-memory kernels for segments of 128+
 * consecutive rows are bf16 only), so they allocate nothing.  Errors as mlora_apply,
 * plus MLORA_ERR_INVALID_ARG for another dtype or a non-finite x_scale.
 */
mlora_status mlora_apply_ex(mlora_pool *pool, const mlora_segments *segs, const void *X, int32_t x_dtype,
                            float x_scale, int64_t ldx, void *Y, int32_t y_dtype, int64_t ldy, void *stream);

/*
 * The base projection and the LoRA delta in one pass (page "Multi-LoRA serving",
 * ybb.press ai-applications, section 3.3 on fusing W0 x + B(A x) into one kernel, and
 * its paragraph on cuBLASLt epilogue fusion after section 5.3):
 *
 *   Y[t, :] = bf16(X[t, :] W^T + s_g (X[t, :] A_a^T) B_a^T)   rows t of adapter segments
 *   Y[t, :] = bf16(X[t, :] W^T)                                every other row
 *
 * with the whole sum in fp32 and one rounding.  Unlike mlora_apply, Y is an output
 * only: it is never read, and every row of it is written.  The shrink runs first (as
 * in mlora_shrink, into the pool's workspace); then a tensor-core GEMM adds each
 * 128-row tile's low-rank products (one per distinct adapter among its rows, on the
 * same fp32 H as the other entry points) into the accumulator of X W^T before the
 * single store.
 * X: device bf16 [n_rows, d_in] (row stride ldx); W: the base weight, device bf16
 * [d_out, d_in] (row stride ldw, the nn.Linear layout); Y: device bf16
 * [n_rows, d_out] (row stride ldy).  Strides are multiples of 8 elements, pointers
 * 16-byte aligned (else MLORA_ERR_INVALID_ARG).  The workspace (H, a 16-byte row map
 * per row and per 128 rows a list of slots) is the pool's, grown as for mlora_apply
 * (not during stream capture: MLORA_ERR_UNSUPPORTED) and shared with it.  Segments
 * that mlora_apply rejects set the same status bits here and their rows get X W^T
 * only; a row claimed by two segments keeps one claim and sets MLORA_FLAG_BAD_ROW.
 */
mlora_status mlora_base_gemm_apply(mlora_pool *pool, const mlora_segments *segs, const void *X, int64_t ldx,
                                   const void *W, int64_t ldw, void *Y, int64_t ldy, void *stream);

/* Projections one mlora_apply_multi call may cover. */
#define MLORA_MAX_FUSED 4

/*
 * mlora_apply over several projections of one layer that read the same input rows
 * -- q_proj, k_proj and v_proj, or gate_proj and up_proj -- in one pass over X.
 * An adapter covers several target modules of a layer, each with its own A and B
 * (page "Multi-LoRA Serving: adapter batching", section "An adapter is not one
 * contiguous weight"); with one pool per module, slot a of every pool holds the
 * same adapter's weights for that module, so one batch's segments serve them all.
 *
 *   For k = 0 .. n_proj-1:  Y_k[t, :] = bf16(Y_k[t, :] + s (X[t, :] A_{a,k}^T) B_{a,k}^T)
 *
 * with the same results as n_proj mlora_apply calls on (pools[k], Y[k]).
 * pools[n_proj]: distinct pools with equal d_in and n_slots (d_out, r_max may
 * differ); the rank and scale come from each pool's slot (segs->ranks, when given,
 * must match every pool; segs->scales, when given, applies to all;
 * segs->generations, when given, must match the slot's generation in every pool,
 * which holds when an adapter is always loaded into all the pools together).  X: device bf16
 * [n_rows, d_in], shared; Y[k]: device bf16 [n_rows, d_out of pools[k]] with row
 * stride ldy[k], distinct, non-overlapping buffers.  1 <= n_proj <= MLORA_MAX_FUSED.
 * Short segments run in one launch whose work items are (tile, projection) with a
 * tile's projections side by side, so its X rows are read from HBM once.  Long
 * segments: when all pools have the same rank bucket and hold every slot at the same
 * rank, one shrink launch computes H for every projection (X's rows read once), each
 * into its pool's workspace; otherwise each projection runs its own shrink; then each
 * projection's expand (workspaces grown as in mlora_apply, all before anything is
 * launched).
 * Errors: host-side as mlora_apply (plus a repeated pool or output, different
 * d_in / n_slots / device: MLORA_ERR_INVALID_ARG).  Device-side: metadata problems
 * found while scanning the segments (bad offsets or slots) go to pools[0]'s status
 * word; problems of one projection's tile (bad row, empty slot, rank or generation
 * mismatch) to that projection's pool.
 */
mlora_status mlora_apply_multi(mlora_pool *const *pools, int32_t n_proj,
                               const mlora_segments *segs, const void *X, int64_t ldx,
                               void *const *Y, const int64_t *ldy, void *stream);

/*
 * mlora_apply for callers that cannot allocate device memory.  The paper has no
 * counterpart: this entry point is an interface choice of this library.
 *
 * Same operation, arguments and errors as mlora_apply.  mlora_apply keeps the fp32
 * H values of long segments (128 rows or more) in a workspace that the pool grows
 * with cudaMalloc the first time a batch needs more.  Some callers cannot allow
 * that: a serving engine that reserves nearly all of HBM for weights and KV cache
 * up front and hands out memory only from its own allocator (a library cudaMalloc
 * would fail or eat into that reservation), or a latency-critical loop that must not
 * hit the device-wide synchronisation a cudaMalloc / cudaFree can cause.  This
 * variant takes the workspace from a fixed scratch array in the library's own device
 * memory instead, and calls no cudaMalloc, cudaFree or other allocating routine.
 *   - The scratch array is 4 MiB.  It is reserved on a device when the first pool
 *     is created there (mlora_pool_create looks up its address, which under CUDA's
 *     lazy module loading is what brings it onto the device), so the first
 *     mlora_apply_noalloc call finds it in place; every GPU that has held a pool keeps
 *     it until the process exits.
 *   - Only batches that take the long-segment kernels use it: n_tokens >= 128 and
 *     segs->max_segment_rows either 0 (unknown) or >= 128.  Such
 *     a batch needs n_tokens * max(16, bucket(r_max)) * 4 bytes (up to 16384 grouped
 *     rows for a rank-64 pool, 65536 for r_max <= 16); a larger one returns
 *     MLORA_ERR_UNSUPPORTED with nothing launched.  Other batches have no size limit.
 *   - Every call shares the one array, which keeps the last call's contents (no
 *     part of it needs to start at zero: each call writes the H values it reads).
 *     Calls whose kernels overlap on the GPU -- on different streams, from several
 *     threads, or for several pools -- race on it: serialise them.
 */
mlora_status mlora_apply_noalloc(mlora_pool *pool, const mlora_segments *segs, const void *X,
                                 int64_t ldx, void *Y, int64_t ldy, void *stream);

/*
 * Host helper: group rows by slot (row_slots[t] = slot of row t, -1 = base).
 * Segments come in the order their slot first appears; rows keep their original
 * order inside a segment.  Outputs are HOST arrays the caller sizes:
 * offsets[n_rows + 1], slots[n_rows], token_indices[n_rows].  *n_segments gets S,
 * *max_segment_rows (may be NULL) the longest adapter segment whose rows are
 * consecutive (the mlora_segments hint), at least 1 (0 would read as "unknown").  If pool and
 * ranks are both non-NULL, ranks[n_rows] gets each segment's slot rank (0 for
 * base).  Slots are not range-checked here (the device checks them).
 */
mlora_status mlora_build_segments(const int32_t *row_slots, int32_t n_rows,
                                  int32_t *offsets, int32_t *slots, int32_t *token_indices,
                                  int32_t *n_segments, int32_t *max_segment_rows,
                                  const mlora_pool *pool, int32_t *ranks);

/*
 * Host-side adapter cache over the slots of a pool: which adapter (a caller-chosen
 * 64-bit id) each slot holds, how many in-flight batches pin it, and least-recently
 * used order among the unpinned ones (page "LoRA/QLoRA multi-tenant serving",
 * section 2 on the adapter memory manager, and page "Multi-LoRA Serving: adapter
 * batching", sections "Why the adapter cache needs tiers" and "Eviction cannot look
 * only at LRU": pinned slots are never evicted).  No device memory, no CUDA calls;
 * all functions are thread-safe.
 */
typedef struct mlora_slot_cache mlora_slot_cache;

/* A cache of n_slots empty slots. */
mlora_status mlora_slot_cache_create(int32_t n_slots, mlora_slot_cache **out);

/* NULL is accepted. */
mlora_status mlora_slot_cache_destroy(mlora_slot_cache *cache);

/*
 * Find or place adapter `adapter_id` and pin its slot (one more pin).  On a hit
 * *needs_load = 0.  On a miss the slot is taken from the never-used slots first,
 * then from the least recently released unpinned slot, whose adapter is forgotten
 * (*evicted_id gets it, or UINT64_MAX if the slot was empty; evicted_id may be
 * NULL); *needs_load = 1 and the caller loads the adapter (mlora_pool_load_slot)
 * before using the slot.  MLORA_ERR_NO_SLOT if every slot is pinned.
 */
mlora_status mlora_slot_cache_acquire(mlora_slot_cache *cache, uint64_t adapter_id, int32_t *slot,
                                      int32_t *needs_load, uint64_t *evicted_id);

/* Drop one pin of a slot; with no pins left it becomes the most recently used
 * candidate for eviction.  MLORA_ERR_INVALID_ARG if the slot is not pinned. */
mlora_status mlora_slot_cache_release(mlora_slot_cache *cache, int32_t slot);

/* Forget the adapter a slot holds (e.g. after its load failed); pins are kept. */
mlora_status mlora_slot_cache_invalidate(mlora_slot_cache *cache, int32_t slot);

/* Slot holding `adapter_id` (-1 if none), without pinning or touching the order. */
mlora_status mlora_slot_cache_lookup(const mlora_slot_cache *cache, uint64_t adapter_id, int32_t *slot);

/* Counters since creation: hits, misses, evictions of a held adapter.  NULL accepted. */
mlora_status mlora_slot_cache_stats(const mlora_slot_cache *cache, int64_t *hits, int64_t *misses,
                                    int64_t *evictions);

/* Static description of a status code. */
const char *mlora_status_string(mlora_status status);

/* Library version: major * 10000 + minor * 100 + patch. */
int32_t mlora_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MLORA_H */
