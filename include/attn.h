/*
 * attn.h -- C ABI of libattn_b200: attention over a KV cache on B200 (sm_100a).
 *
 * Three operations share one argument block and one set of semantics:
 *
 *   attn_decode    split-K decode.  Work is cut into (row, KV head, slice)
 *                  units on a (rows, heads, slices) grid; each unit runs an
 *                  online softmax over its slice for every query head of the
 *                  KV head (GQA sharing), and a split_k_reduce pass folds the
 *                  slice partials.  Defined by TensorFold PR #2595 ("attn_decode
 *                  grid becomes (rows, heads, slices)"; attn_decode + attn_merge
 *                  registered as one operator: Q rows, K/V cache -> attention
 *                  rows; 32-key slices).  Supported: K/V in F32, F16, BF16,
 *                  or e4m3 / int8 codes with scales (see "Quantized caches"
 *                  below); Q in F32, F16 or BF16; head_dim 64, 128 or 256;
 *                  1 to 16 query heads per KV head; any out dtype.
 *   attn_selected  maskless selected-key attention: a query row sees exactly
 *                  the cells named in its selection list; the list is sorted,
 *                  invalid and duplicate entries are skipped, and K/V are
 *                  gathered in blocks of 32 cells; rows are split into parts
 *                  combined by split_k_reduce when the grid would under-fill
 *                  the GPU.  Defined by strix-llama.cpp PR #115 / #119
 *                  (FLASH_ATTN_EXT with a selection list src[5];
 *                  flash_attn_sel.comp; flash_attn_split_k_reduce).
 *   attn_prefill   causal prefill: many query rows over the cache with the
 *                  semantics below (softcap before ALiBi, F32 mask bias,
 *                  sinks, +0 for excluded rows, NaN propagation; HartsyInference
 *                  PR #910).  QK^T and PV run on the tensor cores in tiles of
 *                  128 rows x 128 cells; P is rounded to the K/V dtype before
 *                  PV.  Supported: K/V and Q in F16 or BF16 (same dtype),
 *                  head_dim 64, 128 or 256, Q 16-byte aligned with strides
 *                  that are multiples of 16 bytes; any out dtype.  n_slices,
 *                  max_row_len and grid_order are ignored.  With fewer than
 *                  128 rows and G >= 2 query heads per KV head (draft-tree
 *                  rows, short prefills) a tile's 128 rows hold 128 / G
 *                  query rows x the G heads of one KV group, so each K/V
 *                  tile is read once for the whole group; few work units
 *                  are split into up to 32 parts over their cell tiles.
 *                  Workspace: one byte per (row tile, 128-cell tile) and per
 *                  (cell tile, KV head), the visibility bits of every tile
 *                  when a mask is given, and the split parts' partial
 *                  results (attn_workspace_size gives the total).
 *
 * Unified caches.  When cell_seq/row_seq are given (several sequences'
 * cells interleaved in one cache, strix-llama.cpp PR #115 "Isolation"), the
 * cells a row may see are scattered, so attn_decode and attn_prefill first
 * list each row's visible cells (ascending) and then gather them in blocks
 * of 32 cells as attn_selected does, adding the F32 mask bias per cell; rows
 * are split into parts folded by split_k_reduce.  This route needs F16/BF16
 * K/V with Q in that dtype (and cell_pos/row_pos when ALiBi slopes are
 * given); its workspace holds one int32 list of n_cells entries per row.
 *
 * Semantics (all three; HartsyInference PR #910 "attention semantic
 * correctness"):  for row r and query head h (KV head g = h / (Hq/Hkv)),
 *   x_c = scale * q.k_c;  x_c = softcap*tanh(x_c/softcap) if softcap > 0;
 *   then x_c += slope_h * -|row_pos - cell_pos| (ALiBi, after the softcap);
 *   then x_c += mask[r,c] in F32, never narrowed;
 *   sigma = sinks[h] (an extra logit with no value vector) or -inf;
 *   out = sum_c exp(x_c - M) v_c / (sum_c exp(x_c - M) + exp(sigma - M)),
 *   M = max(x, sigma); a row with no visible cell (and sigma = -inf or
 *   finite) is +0.0; NaN anywhere among the logits or the sink gives NaN in
 *   every element; NaN in a visible V gives NaN in that element, also across
 *   the split combine; +inf logit or sink gives NaN.
 *
 * Visibility of cell c for row r (decode and prefill):
 *   row_begin[r] <= c < row_end[r]            (NULL: [0, n_cells))
 *   and cell_seq[c] == row_seq[r]             (if both are non-NULL)
 *   and cell_pos[c] <= row_pos[r]             (if causal)
 *   and mask[r, c] != -inf                    (if mask; a -inf cell is never read)
 * Positions: cell_pos NULL -> c - row_begin[r]; row_pos NULL ->
 * row_end[r] - row_begin[r] - 1, both from row_begin/row_end as given: a
 * range reaching below 0 or past n_cells is clipped to [0, n_cells) for
 * visibility only, never for positions.  Selected: the distinct entries e of
 * row r's list with 0 <= e < n_cells; no range, sequence, causal or mask
 * filter.
 *
 * Memory and ownership.  Every pointer in the argument blocks is DEVICE
 * memory owned by the caller.  The caller also owns the workspace (sized by
 * attn_workspace_size) and the stream.  The library allocates nothing per
 * call, never synchronizes in attn_decode/attn_selected/attn_prefill, and is
 * asynchronous on `stream` (a cudaStream_t passed as void*; NULL = legacy
 * default stream).  Arguments are read during the call; the argument block
 * may be reused as soon as the call returns.
 *
 * Errors.  Every call returns an attn_status.  A shape, dtype, stride or
 * workspace the kernels do not cover is refused with ATTN_ERR_UNSUPPORTED or
 * ATTN_ERR_INVALID_ARG before anything is launched (never a wrong result);
 * attn_last_error() gives a one-line reason (thread-local).  The library
 * never aborts or traps.  Kernels that wait on a barrier give up after a
 * bounded number of polls and record ATTN_ERR_DEVICE_TIMEOUT in a device
 * status word, read by attn_check_device_status().
 *
 * Layouts (strides in ELEMENTS; the head dimension is contiguous):
 *   q   [n_rows][n_head_q][head_dim]      q_stride_row, q_stride_head
 *   k,v [n_cells][n_head_kv][head_dim]    kv_stride_cell, kv_stride_head (shared by k and v)
 *   out [n_rows][n_head_q][head_dim]      o_stride_row, o_stride_head
 *   mask [n_rows][n_cells] F32            mask_stride_row
 * K and V base addresses and their cell/head strides must be 16-byte
 * aligned (tile loads by the Tensor Memory Accelerator).
 *
 * Quantized caches (attn_decode and attn_prefill; TensorFold PR #911: e4m3 rows with one
 * fp32 scale per (position, key head) = amax / 448, half the bytes of bf16;
 * TensorFold PR #2595: an int8 cache with a K scale and a V scale per key).
 * With kv_type ATTN_FP8_E4M3 or ATTN_I8 the stored codes are one byte each and
 *   k_c[d] = k_scale[c * scale_stride_cell + g] * code(K[c][g][d]),
 *   v_c[d] = v_scale[c * scale_stride_cell + g] * code(V[c][g][d]),
 * with code() the OCP FP8 E4M3 value (bias 7, no infinities, S.1111.111 is
 * NaN) or the two's-complement int8 value; everything else is as above on the
 * dequantized K/V.  Strides stay in elements (= bytes).  k_scale, v_scale:
 * F32 device arrays, non-NULL for a quantized cache with n_cells > 0 and NULL
 * otherwise; scale_stride_cell >= n_head_kv.  Q and out are never quantized.
 * With n_slices == 0, Q in BF16 or F16 (16-byte aligned, strides multiples of
 * 8 elements), head_dim 128 or 256 and at most 8 query heads per KV head, the
 * codes run on the tensor cores (widened to f16 in registers, which is exact);
 * other shapes and forced slice counts run on the CUDA cores.
 * attn_prefill takes them with Q in F16 or BF16: one
 * kernel writes code x scale, rounded once to F16, into a contiguous
 * [n_cells][n_head_kv][head_dim] copy of K and of V at the start of the
 * workspace (as TensorFold PR #911's prefill stages e4m3 rows widened to
 * bf16; F16 keeps the one rounding well inside the tolerances), a BF16 Q is
 * copied to F16 after them (the tensor cores take both operands in one type),
 * and the F16 tensor-core prefill runs on the copies.  Values beyond F16's
 * range (|x| > 65504) become infinite.  K, V and their strides must be
 * 16-byte aligned.  attn_selected refuses quantized caches
 * (ATTN_ERR_UNSUPPORTED).
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ATTN_ABI_VERSION 2

typedef enum { ATTN_F32 = 0, ATTN_F16 = 1, ATTN_BF16 = 2, ATTN_FP8_E4M3 = 3, ATTN_I8 = 4 } attn_dtype;

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_INVALID_ARG = -1,     /* null/negative/inconsistent argument           */
    ATTN_ERR_UNSUPPORTED = -2,     /* valid, but not a shape/dtype the kernels take  */
    ATTN_ERR_WORKSPACE = -3,       /* workspace missing or smaller than required     */
    ATTN_ERR_CUDA = -4,            /* a CUDA runtime call failed (launch, attribute) */
    ATTN_ERR_DEVICE_TIMEOUT = -5   /* a kernel gave up waiting on a barrier          */
} attn_status;

enum { ATTN_OP_DECODE = 0, ATTN_OP_SELECTED = 1, ATTN_OP_PREFILL = 2, ATTN_OP_SELECTED_MASKED = 3 };

/* Shared argument block (see the file comment for meaning and layout). */
typedef struct {
    int32_t n_rows, n_head_q, n_head_kv, head_dim, n_cells;

    const void *q;   int32_t q_type;   int64_t q_stride_row, q_stride_head;
    const void *k;   const void *v;    int32_t kv_type;
    int64_t kv_stride_cell, kv_stride_head;
    void *out;       int32_t out_type; int64_t o_stride_row, o_stride_head;

    const int32_t *row_begin, *row_end;   /* [n_rows] or NULL                       */
    const int32_t *cell_seq, *row_seq;    /* [n_cells], [n_rows] or NULL            */
    const int32_t *cell_pos, *row_pos;    /* [n_cells], [n_rows] or NULL            */
    int32_t causal;                       /* 0/1                                     */
    const float *mask; int64_t mask_stride_row;   /* F32 [n_rows][n_cells] or NULL  */

    float scale;                          /* applied to q.k before everything else  */
    float softcap;                        /* <= 0: off                               */
    const float *alibi_slopes;            /* [n_head_q] or NULL                      */
    const float *sinks;                   /* [n_head_q] or NULL (= -inf)             */

    int32_t n_slices;     /* decode: 0 = from occupancy; else 1..64 slices per row  */
    int32_t max_row_len;  /* decode: host-side upper bound on row_end - row_begin
                             (sizes the slices); 0 = unknown, n_cells is used.  A
                             longer row is still correct: its last slice takes the
                             excess.                                                 */
    int32_t grid_order;   /* 0: rows vary fastest over the (rows, heads, slices)
                             grid; 1: slices fastest.  Results are bit-identical;
                             exposed for tests and tuning.                           */
    int32_t reserved[5];  /* must be zero, except reserved[0] in attn_prefill: a
                             test of the kernels' bounded waits.  A value t in
                             1..1000000 makes every CTA of the dense tensor-core
                             prefill first wait, for at most t microseconds, on
                             a barrier nothing arrives at; the wait gives up,
                             the CTA winds down (no copy left in flight, tensor
                             memory freed) without writing its output, and
                             attn_check_device_status() then reports
                             ATTN_ERR_DEVICE_TIMEOUT.  For tests only.      */

    const float *k_scale, *v_scale;   /* quantized caches: per (cell, KV head) scales, else NULL */
    int64_t scale_stride_cell;        /* elements between cells' scale rows (>= n_head_kv)   */
} attn_args;

/* Selected-key arguments.  base.row_begin/row_end/cell_seq/row_seq/mask must be
 * NULL and base.causal 0 (the op is maskless; visibility is the list alone).
 * cell_pos/row_pos are still used for ALiBi distances.                       */
typedef struct {
    attn_args base;
    const int32_t *sel;       /* [n_rows][sel_stride_row], first n_sel used      */
    int64_t sel_stride_row;
    int32_t n_sel;            /* 1..4096 entries per row                          */
    int32_t *sel_sorted_out;  /* optional [n_rows][n_sel]: valid distinct entries
                                 ascending, then -1 padding                        */
    int32_t *sel_count_out;   /* optional [n_rows]: number of distinct valid entries */
} attn_selected_args;

/* Workspace bytes the op needs for these arguments (0 is possible).  n_sel is
 * used by ATTN_OP_SELECTED and ATTN_OP_SELECTED_MASKED only.  Returns 0 also for invalid arguments; call
 * attn_supports() to tell the two apart.                                     */
size_t attn_workspace_size(const attn_args *args, int32_t op, int32_t n_sel);

/* ATTN_OK if the op takes these arguments, else the status the op would
 * return (nothing is launched).                                              */
int32_t attn_supports(const attn_args *args, int32_t op);

/* The three operations.  ws/ws_bytes: device workspace of at least
 * attn_workspace_size() bytes, 256-byte aligned (may be NULL when 0 bytes are
 * needed).  Contents on entry are irrelevant; on return they are scratch.
 * Two calls that share a workspace must be ordered on the GPU.             */
int32_t attn_decode(const attn_args *args, void *ws, size_t ws_bytes, void *stream);
int32_t attn_selected(const attn_selected_args *args, void *ws, size_t ws_bytes, void *stream);
int32_t attn_prefill(const attn_args *args, void *ws, size_t ws_bytes, void *stream);

/* Timing hooks: the same operations, and additionally cudaEventRecord of
 * events[0] before the first kernel, events[1] right after the main kernel
 * (decode: the slice kernel; selected: the gather kernel; prefill: the
 * tensor-core kernel) and events[2] after the last kernel, all on `stream`.
 * Each entry is a cudaEvent_t passed as void*, or NULL to skip it.          */
int32_t attn_decode_timed(const attn_args *args, void *ws, size_t ws_bytes, void *stream,
                          void *const events[3]);
int32_t attn_selected_timed(const attn_selected_args *args, void *ws, size_t ws_bytes, void *stream,
                            void *const events[3]);
int32_t attn_prefill_timed(const attn_args *args, void *ws, size_t ws_bytes, void *stream,
                           void *const events[3]);

/* attn_decode with the step's K/V cache append fused into the same launch
 * (TensorFold PR #985, change list: for a single row the attention launch
 * also does the cache append).  Row r's new K and V rows (k_new, v_new: DEVICE,
 * the cache dtype, [n_rows][n_head_kv][head_dim] with the given element
 * strides, 16-byte aligned) are written into cell row_end[r] - 1 of the cache
 * (args->k / args->v, written here) and the attention of the call already
 * sees them: the result and the cache are those of an append followed by
 * attn_decode, bit for bit.  Runs on the balanced tensor-core kernel: a
 * 16-bit cache with Q in its dtype, n_slices 0, no per-cell sequence ids;
 * row_end must be given when n_rows > 1 (NULL with one row: cell n_cells - 1),
 * and row_end[r] - 1 must lie in [row_begin[r], n_cells).  No row's range may
 * include another row's append cell (rows of separate sequences).  Workspace
 * as attn_decode.                                                           */
int32_t attn_decode_append(const attn_args *args, const void *k_new, const void *v_new, int64_t new_stride_row,
                           int64_t new_stride_head, void *ws, size_t ws_bytes, void *stream);

/* attn_decode for few, long rows without a workspace: one thread-block
 * cluster of 16 CTAs per (row, KV head) (TensorFold PR #985, change list: a
 * cluster of CTAs shares a head over distributed shared memory).  Each of the
 * cluster's 128 warps folds an equal run of the row's 16-cell tiles on the
 * tensor cores; CTA rank 0 then reads the 128 partials over distributed shared
 * memory and folds them in order with the sink -- one launch, no workspace,
 * no split_k_reduce pass.  Same arguments and result as attn_decode (bit-
 * identical across runs); takes a 16-bit cache with Q in its dtype, head_dim
 * 64 or 128, up to 16 q heads per KV head, n_slices 0, no per-cell sequence
 * ids.  Intended for few rows (n_rows x n_head_kv clusters of 16 CTAs).    */
int32_t attn_decode_cluster(const attn_args *args, void *stream);

/* The masked per-cell route of selected-key attention (strix-llama.cpp PR
 * #115, "Measurements": the route a backend without the selected-key kernels
 * takes, a dense per-cell mask over the cache).  Same arguments and result as
 * attn_selected: it writes each row's F32 mask [n_cells] into the workspace
 * (-inf, 0 at every valid listed cell) and runs the attn_prefill tensor-core
 * kernel on it, whose tile classifier skips the tiles no row of a row tile
 * selected.  Takes what that kernel takes (Q in the K/V dtype, F16/BF16,
 * head_dim 64, 128 or 256); cell_pos/row_pos serve ALiBi as in attn_selected
 * (NULL: cell c at c, every row at n_cells - 1).  sel_sorted_out /
 * sel_count_out are not written.  Workspace: attn_workspace_size(base,
 * ATTN_OP_SELECTED_MASKED, n_sel) -- the mask (n_rows x n_cells floats, rows
 * padded to 4) first, then the dense pass's workspace; it grows with the
 * cache, which is the point of the selected-key kernel.  The timed form
 * records events[0] before the mask kernel and events[1], events[2] as
 * attn_prefill_timed does.                                                  */
int32_t attn_selected_masked(const attn_selected_args *args, void *ws, size_t ws_bytes, void *stream);
int32_t attn_selected_masked_timed(const attn_selected_args *args, void *ws, size_t ws_bytes, void *stream,
                                   void *const events[3]);

/* attn_decode for callers that cannot allocate device memory (a real-time
 * loop that must not block in an allocator, a plugin with no memory pool of
 * its own, code that only receives pointers to its inputs and outputs).  The
 * pages have no counterpart: this is a convenience of this library.
 * Arguments and results are those of attn_decode; the split partials live in
 * one built-in 16 MiB device array per GPU (held until the process exits)
 * instead of a caller workspace, and nothing is allocated per call.
 *  - A problem needing more scratch than that returns ATTN_ERR_WORKSPACE
 *    (attn_last_error() gives the size); nothing is launched.
 *  - All calls share the array: calls that may overlap on the GPU race and
 *    corrupt each other; issue them in order on one stream.  Nothing in the
 *    array needs to start at zero.
 *  - The first call on each device looks up the array's address
 *    (cudaGetSymbolAddress, no allocation); make it before any stream capture. */
int32_t attn_decode_noalloc(const attn_args *args, void *stream);

/* Draft-tree rows (TensorFold PR #2595: attn_decode over "Q rows, K/V cache,
 * tree table" with heap-order parents, tree widths 1..16).  Writes the F32
 * additive mask [n_rows][n_cells] (row stride mask_stride_row, DEVICE memory)
 * under which attn_decode computes the tree rows: row r is tree node r, whose
 * token is in cell prefix_cells + r; parent[r] (DEVICE, int32) is its parent
 * node, smaller than r, or -1 for a root.  Row r sees cells [0, prefix_cells)
 * and the cells of its ancestors and itself (mask 0); every other cell is
 * -inf.  n_rows <= 4096; prefix_cells + n_rows <= n_cells.  A parent that is
 * not smaller than its child records ATTN_ERR_INVALID_ARG in the device status
 * word (attn_check_device_status) and hides the ancestors above it.
 * Asynchronous on `stream`; allocates nothing.                              */
int32_t attn_tree_mask(const int32_t *parent, int32_t n_rows, int32_t prefix_cells, int32_t n_cells,
                       float *mask, int64_t mask_stride_row, void *stream);

/* Synchronizes `stream`, then reads and clears the device status word on the
 * current device: ATTN_OK, or ATTN_ERR_DEVICE_TIMEOUT if a kernel gave up on
 * a bounded wait since the last check.                                      */
int32_t attn_check_device_status(void *stream);

/* Human-readable name of a status; reason of the last refusal on this thread. */
const char *attn_strerror(int32_t status);
const char *attn_last_error(void);

/* ATTN_ABI_VERSION of the loaded library. */
int32_t attn_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* ATTN_B200_H */
