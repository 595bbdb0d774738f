// selmask.cu -- the masked per-cell route of selected-key attention.
//
// strix-llama.cpp PR #115 ("Measurements") sets the selected-key kernel
// against the route a backend without it takes: the selection becomes a dense
// per-cell mask over the whole cache, [n_kv, strip], and the ordinary masked
// attention runs on it.  Here that route is attn_selected_masked: this kernel
// writes row r's F32 mask [n_cells] (-inf everywhere, 0 at every valid entry
// of r's selection list; duplicates and invalid entries need no special case)
// and the tensor-core prefill kernel then runs on it, its tile classifier
// skipping the tiles no row of a row tile selected.  The result is the
// selected-key result (the same visible set); the mask and the dense pass
// grow with the cache, which is the pages' point.
#include "common.cuh"
#include "internal.h"

namespace attn {

namespace {

constexpr int kSelMaskThreads = 256;

// One CTA per row: fill the row with -inf (16-byte stores; mask_sr is a
// multiple of 4 and the mask 16-byte aligned), then clear the listed cells.
__global__ void __launch_bounds__(kSelMaskThreads) sel_mask_kernel(const int32_t* sel, int64_t sel_sr, int32_t n_sel,
                                                                  int32_t n_cells, float* mask, int64_t mask_sr) {
  const int r = blockIdx.x;
  float* row = mask + (int64_t)r * mask_sr;
  const float4 ninf = make_float4(neg_inf(), neg_inf(), neg_inf(), neg_inf());
  for (int64_t c = 4 * (int64_t)threadIdx.x; c < n_cells; c += 4 * kSelMaskThreads) {
    if (c + 4 <= n_cells) {
      *reinterpret_cast<float4*>(row + c) = ninf;
    } else {
      for (int64_t e = c; e < n_cells; ++e) row[e] = neg_inf();
    }
  }
  __syncthreads();
  const int32_t* list = sel + (int64_t)r * sel_sr;
  for (int i = threadIdx.x; i < n_sel; i += kSelMaskThreads) {
    const int32_t e = __ldg(list + i);
    if (e >= 0 && e < n_cells) row[e] = 0.f;
  }
}

}  // namespace

cudaError_t launch_sel_mask(const int32_t* sel, int64_t sel_sr, int32_t n_sel, int32_t n_rows, int32_t n_cells,
                            float* mask, int64_t mask_sr, cudaStream_t stream) {
  if (n_rows <= 0) return cudaSuccess;
  sel_mask_kernel<<<dim3((unsigned)n_rows), kSelMaskThreads, 0, stream>>>(sel, sel_sr, n_sel, n_cells, mask, mask_sr);
  return cudaGetLastError();
}

}  // namespace attn
