/*
 * oracle.h -- FP64 CPU reference for attention over a KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA library under
 * attention_split_attn_b200/, and neither includes the other.
 *
 * What it computes is the plain definition of softmax attention, written out
 * with no online softmax, no tiling and no splits (every split/online form on
 * the GPU is an exact re-association of it):
 *
 *   For query row r and query head h (KV head g = floor(h / (Hq/Hkv))), over
 *   the visible cell set V_r:
 *     x_c   = scale * sum_d q[r,h,d] * k[c,g,d]
 *     x_c   = softcap * tanh(x_c / softcap)              if softcap > 0
 *     x_c  += slope_h * (-|row_pos_r - cell_pos_c|)      if ALiBi slopes given
 *     x_c  += (double) mask[r,c]                         if a mask is given
 *     sigma = sinks ? sinks[h] : -inf
 *     any NaN among {x_c} u {sigma}           -> output NaN in every d
 *     M = max({x_c} u {sigma})
 *     M == -inf, or V_r empty with finite sigma -> output +0.0 in every d
 *     otherwise w_c = exp(x_c - M),
 *               L   = sum_c w_c + exp(sigma - M),
 *               out[d] = (sum_c w_c * v[c,g,d]) / L
 *
 * Sources:
 *  - softcap before ALiBi, fully excluded rows give zero, NaN survives the
 *    split combine, F32 mask bias is not narrowed, sink edge cases:
 *    HartsyInference PR #910 "PR 02: attention semantic correctness",
 *    PR description and the review of flash_attn_f32.cu / FlashAttentionKernels.cs
 *    / attention_softmax.cu, and the author's M03 comment.
 *  - visibility by a per-query selection list (sorted, invalid and duplicate
 *    entries skipped, no mask): strix-llama.cpp PR #115 "qwen4exp: use maskless
 *    block selection only where the selected-key kernels run", commit message
 *    of flash_attn_sel.comp (#119).
 *  - visibility in a unified multi-sequence cache (one conversation's output
 *    must not depend on another's cells): same page, "Isolation" measurements.
 *  - the FP64 reference compared by NMSE: same page, #119 commit message.
 *
 * Readings taken where the pages are silent:
 *  - GQA mapping g = floor(h / G); ALiBi bias = -slope_h * |row_pos - cell_pos|;
 *  - a mask value of exactly -inf excludes the cell (it is never read); any
 *    other value (finite, +inf, NaN) is added;
 *  - the sink is one extra logit with no value vector, applied raw;
 *  - selection entries < 0 or >= n_cells are invalid; duplicates count once;
 *  - with no explicit positions, cell c sits at c - row_begin and the row at
 *    row_end - row_begin - 1, from the range as given (a range reaching outside
 *    [0, n_cells) is clipped for visibility only).
 */
#ifndef ATTN_ORACLE_H
#define ATTN_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* One attention problem.  Q/K/V are already widened (exactly) to double by
 * the caller.  Strides are in elements.  All pointers are host memory.      */
typedef struct {
    int32_t n_rows, n_head_q, n_head_kv, head_dim, n_cells;

    const double *q;   int64_t q_stride_row, q_stride_head;
    const double *k;   const double *v;
    int64_t kv_stride_cell, kv_stride_head;

    const int32_t *row_begin, *row_end;   /* NULL: every row spans [0, n_cells)   */
    const int32_t *cell_seq,  *row_seq;   /* both non-NULL: sequence filter        */
    const int32_t *cell_pos,  *row_pos;   /* NULL: cell pos = c - begin_r,
                                             row pos = end_r - begin_r - 1         */
    int32_t causal;                       /* 1: visible only if cell_pos <= row_pos */
    const float *mask; int64_t mask_stride_row;   /* F32 additive bias or NULL     */

    double scale, softcap;                /* softcap <= 0: off                      */
    const float *alibi_slopes;            /* [n_head_q] or NULL                     */
    const float *sinks;                   /* [n_head_q] or NULL (= -inf)            */

    /* Selected-key visibility.  When sel != NULL the visible set of row r is
     * the distinct entries e of sel[r*sel_stride_row + 0 .. n_sel-1] with
     * 0 <= e < n_cells, and row_begin/row_end/cell_seq/causal/mask are not
     * consulted (the op carries no mask).                                     */
    const int32_t *sel; int64_t sel_stride_row; int32_t n_sel;
} oracle_problem;

/* out: [n_rows][n_head_q][head_dim], row-major doubles.  n_threads <= 0
 * means one thread per online host core.  Returns 0, or -1 on bad input.   */
int oracle_attn(const oracle_problem *p, double *out, int n_threads);

/* The same result computed the split way, in FP64: each row's cell range is
 * cut into n_slices pieces at multiples of 32 cells from begin_r (as evenly as
 * the 32-cell granularity allows); each piece yields (m_s, l_s, o_s) and the
 * pieces are folded with the sink in slice order.  Not valid for selected
 * visibility (sel must be NULL).                                             */
int oracle_attn_split(const oracle_problem *p, int n_slices, double *out, int n_threads);

/* Selection list compaction: for each row, the valid entries (0 <= e < n_cells)
 * sorted ascending with duplicates removed.  sorted_out: [n_rows][n_sel],
 * entries past count are set to -1; count_out: [n_rows].                     */
int oracle_select_compact(const int32_t *sel, int64_t sel_stride_row, int32_t n_rows,
                          int32_t n_sel, int32_t n_cells,
                          int32_t *sorted_out, int32_t *count_out);

/* Planted mistakes, for the tests that show the pins catch them.  0 = none.
 * Never set outside those tests.                                             */
void oracle_set_mutation(int m);
int  oracle_get_mutation(void);

#ifdef __cplusplus
}
#endif
#endif
