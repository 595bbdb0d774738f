// internal.h -- host-side plans handed from the C-ABI layer (api.cu) to the
// kernel launchers.  Not installed.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "attn.h"

namespace attn {

// Visibility ingredients of a row (dense ops).  Field meaning as in attn.h.
struct RowFilter {
  const int32_t *row_begin, *row_end, *cell_seq, *row_seq, *cell_pos, *row_pos;
  int32_t causal;
  const float* mask;
  int64_t mask_sr;
};

// Logit transforms and the sink.
struct Logits {
  float scale, softcap;
  const float* slopes;
  const float* sinks;
};

struct OutSpec {
  void* out;
  int32_t type;
  int64_t sr, sh;
};

struct QSpec {
  const void* q;
  int32_t type;
  int64_t sr, sh;
};

// Split partials: one record per (slot, q head of the KV group): the running
// max m and sum l (natural-log domain) and the unnormalised output o[D].
// Records are laid out [slot][G][D] (o) and [slot][G][2] (ml).
struct Partials {
  float* o;
  float* ml;
  int32_t S;   // slice scheme: slices per (row, KV head); slot = (r*Hkv + g)*S + s
};

// ---- decode ----------------------------------------------------------------
struct DecodePlan {
  int32_t R, Hq, Hkv, G, D, N;
  QSpec q;
  OutSpec out;
  RowFilter f;
  Logits lg;
  int32_t S;          // slice scheme: slices per row (grid extent)
  int32_t C;          // slice scheme: cells per slice (multiple of 32); the last slice takes the rest
  int32_t grid_order; // 0: natural order; 1: reversed / slices fastest (results identical)
  Partials part;      // used when S > 1 or in the balanced scheme
  int* status;
  int32_t kv_type;
  int32_t hpw, hg;    // CUDA-core kernel: q heads per warp (padded) and head groups
  int32_t mma;        // 1: tensor-core kernels (16-bit cache, Q in the cache dtype)
  // balanced persistent scheme (n_slices == 0 with the tensor-core kernels):
  int32_t W;          // warps of the persistent grid
  int64_t* row_tiles; // [R+1] exclusive prefix of 16-cell tiles per row (planner output)
  int32_t plan_inline; // 1: few rows; the stream kernel computes the prefix (no planner)
  // e4m3 / int8 caches: per (cell, KV head) scales at c * scale_sc + g
  const float *k_scale, *v_scale;
  int64_t scale_sc;
  // fused append (attn_decode_append; balanced 16-bit kernel): row r's new K/V
  // rows [Hkv][D] at k_new + r * new_sr + g * new_sh go to cell row_end[r] - 1
  // of the cache (k_out / v_out: the cache, written)
  const void *k_new, *v_new;
  int64_t new_sr, new_sh;
  void *k_out, *v_out;
  int64_t kv_sc, kv_sh;
};

bool decode_uses_mma(int kv_type, int q_type, const void* q, int64_t q_sr, int64_t q_sh);
bool decode_shape_supported(int kv_type, int D, int G);

// (rows, heads, slices) grid: one CTA per unit; split_k combine when S > 1.
cudaError_t launch_decode_slices(const DecodePlan& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                                 cudaStream_t stream);

// Balanced persistent scheme: planner kernel, then W single-warp CTAs that
// each take an equal run of the flattened (row, KV head, 16-cell tile) space.
int decode_stream_warps(int kv_type, int D, int G, int sms);
// Cluster decode (attn_decode_cluster): one 16-CTA cluster per (row, KV head),
// partials folded over distributed shared memory; 16-bit caches, head dim
// 64 or 128.
cudaError_t launch_decode_cluster(const DecodePlan& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                                  cudaStream_t stream);
// One-byte caches (e4m3 / int8) that the balanced tensor-core kernel takes.
bool decode_stream8_supported(int kv_type, int q_type, const void* q, int64_t q_sr, int64_t q_sh, int D, int G);
cudaError_t launch_decode_stream(const DecodePlan& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                                 cudaStream_t stream, cudaEvent_t after_main);

// ---- selected-key attention ---------------------------------------------------
struct SelectedPlan {
  int32_t R, Hq, Hkv, G, D, N;
  const void* q;
  int64_t q_sr, q_sh;
  const void *k, *v;
  int64_t kv_sc, kv_sh;
  int32_t kv_type;
  OutSpec out;
  Logits lg;
  const int32_t *cell_pos, *row_pos;   // ALiBi distances only
  const float* mask;                   // optional F32 bias [R][mask_sr] added per listed cell
  int64_t mask_sr;                     //   (unified-cache route; NULL for the selected op)
  const int32_t* sel;                  // [R][sel_stride], first n_sel used
  int64_t sel_stride;
  int32_t n_sel, n_pow2;               // n_pow2: n_sel rounded up to a power of 2
  int32_t* compact;                    // workspace [R][n_sel]: valid distinct cells, ascending
  int32_t* count;                      // workspace [R]: their number
  int32_t *sorted_out, *count_out;     // caller's optional copies (or NULL)
  int32_t S, C;                        // parts per row and cells per part (multiple of 32)
  Partials part;                       // when S > 1
  int* status;
};

int selected_pow2(int n_sel);
cudaError_t launch_select_compact(const SelectedPlan& p, cudaStream_t stream);
cudaError_t launch_selected(const SelectedPlan& p, cudaStream_t stream);

// Unified-cache route of decode and prefill (per-cell sequence ids): one CTA
// per row scans the row's cell range and writes the visible cells (same
// sequence, causal, mask != -inf) in ascending order into compact[r][0..),
// their number into count[r]; the selected-key gather kernel then runs on
// those lists with the mask bias added per cell.
cudaError_t launch_visible_lists(const SelectedPlan& p, const RowFilter& f, cudaStream_t stream);

// ---- causal prefill -----------------------------------------------------------
// Tiles of 128 query rows x 128 cells.  A classifier kernel tags every (row
// tile, cell tile) as skipped (no row sees any cell), full (every row sees
// every cell and the mask adds exactly 0 there), bits (with a mask: the mask
// adds exactly 0 on every visible cell, so the visibility bits the classifier
// stores say everything) or mixed (visible cells with a nonzero mask value),
// plus a flag for a visible cell after its row's position; and every (cell
// tile, KV head) whose V holds a non-finite value.  The tensor-core kernel then
// runs one CTA per (row tile, pair of q heads of one KV group).
enum : uint8_t {
  kTileSkip = 0, kTileFull = 1, kTileMixed = 2, kTileBits = 3,   // stored class (low 2 bits)
  kTileLate = 8,                                                  // stored flag
  kTileMixedBadV = 4                                              // kernel-side code only
};

struct PrefillPlan {
  int32_t R, Hq, Hkv, G, D, N;
  int32_t kv_type;
  const void* k;            // K cache (tile norms for the softcap range bound)
  const void* v;            // V cache (scanned for non-finite values)
  int64_t kv_sc, kv_sh;     // its cell and head strides (elements)
  OutSpec out;
  RowFilter f;
  Logits lg;
  int32_t n_rt, n_kt;       // row tiles, cell tiles (128 each)
  int32_t n_pairs;          // CTAs per (row tile, KV head): ceil(G / 2) up to head dim 128, G at 256 (1 packed)
  // Packed rows (pack > 1, fewer rows than a tile): the 128 lanes of a tile
  // hold rpt = 128 / pack rows x the pack = G q heads of one KV group (lane
  // t: row t / pack, head t % pack), so every K and V tile serves all of the
  // group's heads at once; one CTA per (row tile, KV head).  Else pack = 1,
  // rpt = 128.
  int32_t pack, rpt;
  uint8_t* cls;             // workspace [n_rt][n_kt]
  uint32_t* bits;           // workspace [n_rt][n_kt][128 rows][4 words] (with a mask) or NULL
  uint8_t* vbad;            // workspace [n_kt][Hkv]
  float cap_lim;            // |scale * q.k| at or below which the softcap polynomial is used
  float k3, k5, k7;         // softcap polynomial coefficients t_n / softcap^(n-1)
  // Packed path: the odd Taylor series of c tanh(u / c) through u^9 in the raw
  // dot product s (u = scale s): x = s (scale + w (a3 + w (a5 + w (a7 + w a9)))),
  // w = s^2, a_n = t_n scale^n / c^(n-1); truncation below 3.7e-7 c for
  // |u| <= 0.4 c, i.e. |s| <= s_lim.  cap_raw = 0 when these coefficients are
  // not normal floats (then the scalar path's polynomial in u is used).
  float a3, a5, a7, a9, s_lim;
  int32_t cap_raw;
  // A tile needs no per-cell range check when |s| <= |q| |k| is within s_lim
  // for every row: |q_r|^2 max_c |k_c|^2 <= bound2 (= 0.998 s_lim^2).
  float bound2;
  float* kn2;               // workspace [n_kt][Hkv]: max |k_c|^2 over the tile (NaN/inf kept)
  // Bound path (bf16 K/V): the softcap constants times log2(e) (b_n = a_n log2 e,
  // bsc = scale log2 e) and the |q|^2 max|k|^2 limits under which it runs:
  // degree-7 series (bound7: |u| <= c / 3), degree 9 (bound9: |u| <= 0.4 c),
  // no softcap (nc_lim2); each also keeps |scale| |q| max|k| <= 30.
  float b3, b5, b7, b9, bsc, bound7, bound9, nc_lim2;
  int32_t out_vec;          // output rows may be written with 16-byte stores
  int32_t mask_vec;         // mask rows may be read with 16-byte loads
  int* status;
  // Split units: CTAs [0, n_full) are whole units; the next n_split units
  // run as k_split parts each (CTA n_full + u * k_split + part) whose
  // (m, l, O) go to part_o / part_ml and are folded by the last part to finish
  // (split_cnt: one counter per split unit, zeroed by the classifier).
  int64_t n_full, n_split;
  int32_t k_split;
  int* split_cnt;
  float *part_o, *part_ml;
  uint64_t wait_ns;         // bound of every barrier wait (a timeout records ATTN_ERR_DEVICE_TIMEOUT)
  int32_t test_stall;       // 1: the softmax warps first wait on a barrier nothing arrives at
};

// ---- widening of e4m3 / int8 caches for prefill ------------------------------
struct DequantPlan {
  int32_t N, Hkv, D;
  int32_t code_type;        // ATTN_FP8_E4M3 or ATTN_I8 (widened to F16)
  const void *k, *v;        // codes [N][Hkv][D] with strides sc, sh (bytes = elements)
  int64_t sc, sh;
  const float *k_scale, *v_scale;   // [N][ss], column = KV head
  int64_t ss;
  void *k_out, *v_out;      // [N][Hkv][D] contiguous, F16
  // a BF16 Q copied to F16 ([R][Hq][D] contiguous), or q_out NULL
  int32_t R, Hq;
  const void* q;
  int64_t q_sr, q_sh;
  void* q_out;
};
cudaError_t launch_dequant(const DequantPlan& p, int sms, cudaStream_t stream);

cudaError_t launch_prefill(const PrefillPlan& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                           const CUtensorMap& tmV, cudaStream_t stream, cudaEvent_t after_classify);

// ---- combine (split_k_reduce) -------------------------------------------------
// Folds the partial records of each (row, q head) in slot order with the sink.
struct CombinePlan {
  int32_t R, Hq, Hkv, G, D;
  OutSpec out;
  const float* sinks;
  Partials part;
  int32_t mode;                          // 0: slice scheme, 1: balanced scheme
  const int32_t *row_begin, *row_end;    // slice scheme: n_used(r) from ranges ...
  int32_t N, C;
  const int32_t* n_used;                 // ... or from per-row counts (selected op)
  const int32_t* row_len;                // ... or from per-row lengths with C (selected op)
  const int64_t* row_tiles;              // balanced scheme
  int32_t W;
  int use_pdl;
};
cudaError_t launch_combine(const CombinePlan& p, cudaStream_t stream);

// ---- masked route of selected-key attention ------------------------------------------
// Row r of the F32 mask [n_rows][mask_sr]: -inf, 0 at the valid entries of
// row r's selection list (mask 16-byte aligned, mask_sr a multiple of 4).
cudaError_t launch_sel_mask(const int32_t* sel, int64_t sel_sr, int32_t n_sel, int32_t n_rows, int32_t n_cells,
                            float* mask, int64_t mask_sr, cudaStream_t stream);

// ---- draft-tree rows ------------------------------------------------------------
cudaError_t launch_tree_mask(const int32_t* parent, int32_t n_rows, int32_t prefix_cells, int32_t n_cells,
                             float* mask, int64_t mask_sr, int* status, cudaStream_t stream);
int max_tree_rows();

// Set the message attn_last_error() returns on this thread.
void set_last_error(const char* msg);

// ATTN_OK when the current device is one the kernels run on (sm_100), else
// the status the operations return for it (with attn_last_error() set).
int32_t check_device();

}  // namespace attn
