// internal.h -- host-side plans handed from the C-ABI layer (api.cu) to the
// kernel launchers (decode.cu, selected.cu, prefill.cu).  Not installed.
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

// Output of a row: where and in which dtype.
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

// Split-K partial store: per (row, q head, slice) the slice's running max m
// and sum l (natural-log domain) and its unnormalised output o[D].
struct Partials {
  float* o;    // [R][Hq][S][D]
  float* ml;   // [R][Hq][S][2]
  int32_t S;
};

// ---- decode ----------------------------------------------------------------
struct DecodePlan {
  int32_t R, Hq, Hkv, G, D, N;
  QSpec q;
  OutSpec out;
  RowFilter f;
  Logits lg;
  int32_t S;          // slices per row (grid extent)
  int32_t C;          // cells per slice (multiple of 32); the last slice takes the rest
  int32_t grid_order; // 0 rows fastest, 1 slices fastest
  Partials part;      // used when S > 1
  int* status;
  int32_t kv_type;
  int32_t hpw, hg;    // q heads per warp (padded) and head groups
};

bool decode_shape_supported(int kv_type, int D, int G);
cudaError_t launch_decode(const DecodePlan& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                          cudaStream_t stream);

// split_k_reduce over decode partials (also used by the selected op).  Reads
// n_used(r) slices for row r: n_used = 0 if empty else min(S, ceil(len/C)),
// with len from `f` (decode) or from `counts` (selected: per-row list length).
struct ReducePlan {
  int32_t R, Hq, D;
  OutSpec out;
  const float* sinks;
  Partials part;
  // slice count per row: either from ranges (row_begin/row_end, C) or a
  // device array of counts (n_used per row)
  const int32_t *row_begin, *row_end;
  int32_t N, C;
  const int32_t* n_used;  // if non-NULL, overrides the range rule
  int use_pdl;
};
cudaError_t launch_split_k_reduce(const ReducePlan& p, cudaStream_t stream);

}  // namespace attn
