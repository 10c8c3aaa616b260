/*
 * oracle.c -- plain fp64 CPU oracle for the heterogeneous-batch LoRA branch.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke entry point and the
 * benchmark's CPU-baseline leg may load this file's library.  It shares no code,
 * header, table or helper with the CUDA path and includes no CUDA header.
 *
 * What it computes (page "Multi-LoRA Serving: adapter batching", charlestar.github.io,
 * sections "LoRA on one Linear layer" and "What metadata a segmented kernel needs"):
 *
 *   For a linear layer W in R^{d_out x d_in}, LoRA adds  s (X A^T) B^T  with
 *   A in R^{r x d_in}, B in R^{d_out x r} and s = alpha / r.  In a mixed batch the
 *   rows are grouped into segments; segment g uses slot a = adapter_slots[g]
 *   (slot -1 = base model only, no delta), and for each grouped position p of
 *   the segment, t = token_indices[p] is the original row:
 *       H[p, j]  = sum_k X[t, k] * A_a[j, k]          (shrink,  j < r)
 *       Y[t, o] += s_g * sum_j H[p, j] * B_a[o, j]     (expand + scatter-add)
 *
 * All arithmetic is fp64 on the exact values of the bf16 inputs.  No blocking, no
 * reordering: each row is one straight loop over k and then over o.  The
 * per-row ("gather") formulation of the same sum, as the Punica gather-scatter
 * section of the S-LoRA page describes it (tbr8.org, section 3.2), is a second
 * entry point that never looks at the segments.
 *
 * Invalid metadata (the library's contract): a segment whose offsets are out of
 * order or out of range, whose slot is out of range or not loaded, or whose rank
 * differs from the slot's rank is skipped; a row index outside [0, n_rows) is
 * skipped.  Each skip sets a reason bit in the returned flags.
 */
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_BAD_OFFSETS   1
#define ORC_BAD_SLOT      2
#define ORC_BAD_RANK      4
#define ORC_BAD_ROW       8
#define ORC_SLOT_EMPTY   16

#define ORC_MAX_RANK    256   /* bound of the per-row h[] buffer */

/* bf16 -> double: the bf16 bit pattern is the high half of an IEEE binary32. */
static double bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Rank of slot a or -1 if the segment may not use it (sets *flags). */
static int check_segment(int g, int n_tokens, const int32_t *offsets, const int32_t *slots,
                         const int32_t *ranks, int n_slots, const int32_t *slot_rank,
                         int *flags)
{
    int a = slots[g];
    int p0 = offsets[g], p1 = offsets[g + 1];
    if (a == -1) return -1;
    if (p0 < 0 || p1 < p0 || p1 > n_tokens) { *flags |= ORC_BAD_OFFSETS; return -1; }
    if (a < -1 || a >= n_slots) { *flags |= ORC_BAD_SLOT; return -1; }
    if (slot_rank[a] <= 0) { *flags |= ORC_SLOT_EMPTY; return -1; }
    if (slot_rank[a] > ORC_MAX_RANK) { *flags |= ORC_BAD_RANK; return -1; }
    if (ranks != NULL && ranks[g] != slot_rank[a]) { *flags |= ORC_BAD_RANK; return -1; }
    return slot_rank[a];
}

/* One row: h = x A^T (length r), then y += s * h B^T.  The fixed loop order is the
 * whole of the oracle's arithmetic; both formulations call it. */
static void lora_row(int d_in, int d_out, int r, const uint16_t *x, double *y, double s,
                     const uint16_t *A, const uint16_t *B, double *h)
{
    for (int j = 0; j < r; ++j) {
        double acc = 0.0;
        const uint16_t *a_row = A + (size_t)j * d_in;
        for (int k = 0; k < d_in; ++k) acc += bf16_value(x[k]) * bf16_value(a_row[k]);
        h[j] = acc;
    }
    for (int o = 0; o < d_out; ++o) {
        double acc = 0.0;
        const uint16_t *b_row = B + (size_t)o * r;
        for (int j = 0; j < r; ++j) acc += h[j] * bf16_value(b_row[j]);
        y[o] += s * acc;
    }
}

/* The same row with the activation given as fp64 values rather than bf16 bits -- an
 * activation whose exact value is known by other means, such as an FP8 code times its
 * scale at the dtype boundary of a quantized base model (page "Multi-LoRA Serving:
 * adapter batching", section "The dtype boundary between a quantized base model and
 * LoRA").  Same loop order. */
static void lora_row_xf64(int d_in, int d_out, int r, const double *x, double *y, double s,
                          const uint16_t *A, const uint16_t *B, double *h)
{
    for (int j = 0; j < r; ++j) {
        double dot = 0.0;
        const uint16_t *arow_j = A + (size_t)d_in * j;
        for (int k = 0; k < d_in; ++k) dot += x[k] * bf16_value(arow_j[k]);
        h[j] = dot;
    }
    for (int o = 0; o < d_out; ++o) {
        double dot = 0.0;
        const uint16_t *brow_o = B + (size_t)r * o;
        for (int j = 0; j < r; ++j) dot += h[j] * bf16_value(brow_o[j]);
        y[o] = y[o] + s * dot;
    }
}

static void set_threads(int n_threads)
{
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
}

/*
 * Segmented formulation.  Y (fp64, row stride ldy) holds Y0 on entry and
 * Y0 + delta on return.  scales may be NULL (then s = alpha/r of the slot);
 * token_indices may be NULL (then grouped position p is row p).
 * A[a] is the slot's [r, d_in] row-major bf16 matrix, B[a] its [d_out, r].
 * Returns the OR of the skip reasons.
 */
int orc_apply_segments(int n_rows, int d_in, int d_out,
                       const uint16_t *X, int64_t ldx, double *Y, int64_t ldy,
                       int n_segments, const int32_t *offsets, const int32_t *slots,
                       const int32_t *ranks, const double *scales,
                       int n_tokens, const int32_t *token_indices,
                       int n_slots, const int32_t *slot_rank, const double *slot_alpha,
                       const uint16_t *const *A, const uint16_t *const *B, int n_threads)
{
    int flags = 0;
    set_threads(n_threads);
    /* grouped position -> segment, or -1 for positions nobody computes */
    int32_t *seg_of = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n_tokens > 0 ? n_tokens : 1));
    for (int p = 0; p < n_tokens; ++p) seg_of[p] = -1;
    for (int g = 0; g < n_segments; ++g) {
        if (check_segment(g, n_tokens, offsets, slots, ranks, n_slots, slot_rank, &flags) < 0)
            continue;
        for (int p = offsets[g]; p < offsets[g + 1]; ++p) seg_of[p] = g;
    }
    int row_flags = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : row_flags)
    for (int p = 0; p < n_tokens; ++p) {
        int g = seg_of[p];
        if (g < 0) continue;
        int a = slots[g];
        int r = slot_rank[a];
        int t = token_indices ? token_indices[p] : p;
        if (t < 0 || t >= n_rows) { row_flags |= ORC_BAD_ROW; continue; }
        double s = scales ? scales[g] : slot_alpha[a] / (double)r;
        double h[ORC_MAX_RANK];
        lora_row(d_in, d_out, r, X + (size_t)t * ldx, Y + (size_t)t * ldy, s, A[a], B[a], h);
    }
    free(seg_of);
    return flags | row_flags;
}

/*
 * Per-row (gather) formulation: rows in original order, row_slot[t] = -1 for
 * base-only rows; row_scale may be NULL (then alpha/r of the slot).
 */
int orc_apply_rows(int n_rows, int d_in, int d_out,
                   const uint16_t *X, int64_t ldx, double *Y, int64_t ldy,
                   const int32_t *row_slot, const double *row_scale,
                   int n_slots, const int32_t *slot_rank, const double *slot_alpha,
                   const uint16_t *const *A, const uint16_t *const *B, int n_threads)
{
    int flags = 0;
    set_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : flags)
    for (int t = 0; t < n_rows; ++t) {
        int a = row_slot[t];
        if (a == -1) continue;
        if (a < -1 || a >= n_slots) { flags |= ORC_BAD_SLOT; continue; }
        int r = slot_rank[a];
        if (r <= 0) { flags |= ORC_SLOT_EMPTY; continue; }
        if (r > ORC_MAX_RANK) { flags |= ORC_BAD_RANK; continue; }
        double s = row_scale ? row_scale[t] : slot_alpha[a] / (double)r;
        double h[ORC_MAX_RANK];
        lora_row(d_in, d_out, r, X + (size_t)t * ldx, Y + (size_t)t * ldy, s, A[a], B[a], h);
    }
    return flags;
}

/*
 * Per-row formulation with the activation as fp64 values (X fp64 [n_rows, ldx]); the
 * rest as orc_apply_rows.
 */
int orc_apply_rows_xf64(int n_rows, int d_in, int d_out,
                        const double *X, int64_t ldx, double *Y, int64_t ldy,
                        const int32_t *row_slot, const double *row_scale,
                        int n_slots, const int32_t *slot_rank, const double *slot_alpha,
                        const uint16_t *const *A, const uint16_t *const *B, int n_threads)
{
    int flags = 0;
    set_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : flags)
    for (int t = 0; t < n_rows; ++t) {
        int a = row_slot[t];
        if (a == -1) continue;
        if (a < -1 || a >= n_slots) { flags |= ORC_BAD_SLOT; continue; }
        int r = slot_rank[a];
        if (r <= 0) { flags |= ORC_SLOT_EMPTY; continue; }
        if (r > ORC_MAX_RANK) { flags |= ORC_BAD_RANK; continue; }
        double s = row_scale ? row_scale[t] : slot_alpha[a] / (double)r;
        double h[ORC_MAX_RANK];
        lora_row_xf64(d_in, d_out, r, X + (size_t)t * ldx, Y + (size_t)t * ldy, s, A[a], B[a], h);
    }
    return flags;
}

/*
 * Shrink alone: H[p, j] = sum_k X[t_p, k] A_a[j, k] for j < r, grouped order,
 * H row stride ldh.  Entries of skipped positions and j >= r are not written.
 */
int orc_shrink(int n_rows, int d_in, const uint16_t *X, int64_t ldx,
               int n_segments, const int32_t *offsets, const int32_t *slots,
               const int32_t *ranks, int n_tokens, const int32_t *token_indices,
               int n_slots, const int32_t *slot_rank, const uint16_t *const *A,
               double *H, int64_t ldh, int n_threads)
{
    int flags = 0;
    set_threads(n_threads);
    for (int g = 0; g < n_segments; ++g) {
        int r = check_segment(g, n_tokens, offsets, slots, ranks, n_slots, slot_rank, &flags);
        if (r < 0) continue;
        const uint16_t *Aa = A[slots[g]];
        int row_flags = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : row_flags)
        for (int p = offsets[g]; p < offsets[g + 1]; ++p) {
            int t = token_indices ? token_indices[p] : p;
            if (t < 0 || t >= n_rows) { row_flags |= ORC_BAD_ROW; continue; }
            const uint16_t *x = X + (size_t)t * ldx;
            for (int j = 0; j < r; ++j) {
                double acc = 0.0;
                for (int k = 0; k < d_in; ++k)
                    acc += bf16_value(x[k]) * bf16_value(Aa[(size_t)j * d_in + k]);
                H[(size_t)p * ldh + j] = acc;
            }
        }
        flags |= row_flags;
    }
    return flags;
}

/*
 * Expand alone: Y[t_p, o] += s_g * sum_j H[p, j] B_a[o, j]  (fp64 H given).
 */
int orc_expand(int n_rows, int d_out, const double *H, int64_t ldh,
               double *Y, int64_t ldy,
               int n_segments, const int32_t *offsets, const int32_t *slots,
               const int32_t *ranks, const double *scales,
               int n_tokens, const int32_t *token_indices,
               int n_slots, const int32_t *slot_rank, const double *slot_alpha,
               const uint16_t *const *B, int n_threads)
{
    int flags = 0;
    set_threads(n_threads);
    for (int g = 0; g < n_segments; ++g) {
        int r = check_segment(g, n_tokens, offsets, slots, ranks, n_slots, slot_rank, &flags);
        if (r < 0) continue;
        int a = slots[g];
        double s = scales ? scales[g] : slot_alpha[a] / (double)r;
        const uint16_t *Ba = B[a];
        int row_flags = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : row_flags)
        for (int p = offsets[g]; p < offsets[g + 1]; ++p) {
            int t = token_indices ? token_indices[p] : p;
            if (t < 0 || t >= n_rows) { row_flags |= ORC_BAD_ROW; continue; }
            const double *h = H + (size_t)p * ldh;
            double *y = Y + (size_t)t * ldy;
            for (int o = 0; o < d_out; ++o) {
                double acc = 0.0;
                for (int j = 0; j < r; ++j) acc += h[j] * bf16_value(Ba[(size_t)o * r + j]);
                y[o] += s * acc;
            }
        }
        flags |= row_flags;
    }
    return flags;
}

/*
 * Number of distinct adapter parameters one row's delta reads, found by walking
 * the same index ranges lora_row walks and counting each (matrix, i, j) once.
 * The page's parameter count is r (d_in + d_out).
 */
int64_t orc_adapter_params_read(int d_in, int d_out, int r)
{
    int64_t n = 0;
    for (int j = 0; j < r; ++j)
        for (int k = 0; k < d_in; ++k) ++n;       /* A[j, k] */
    for (int o = 0; o < d_out; ++o)
        for (int j = 0; j < r; ++j) ++n;          /* B[o, j] */
    return n;
}

int orc_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
