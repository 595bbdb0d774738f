// tree.cu -- draft-tree decode rows (attn_tree_mask).
//
// TensorFold PR #2595 decodes the nodes of a draft tree as rows of one
// attn_decode call: the operator maps "bf16 Q rows, bf16 K/V cache, tree table
// -> bf16 attention rows", with heap-order parents (a node's parent has a
// smaller index) at tree widths 1, 2, 4, 8, 12 and 16.  Row r of the call is
// node r; its token sits in cell prefix_cells + r; it sees every prefix cell
// and the cells of its ancestors and itself, nothing else.  This kernel writes
// that visibility as the F32 additive mask attn_decode takes (0 visible, -inf
// hidden), so the tree rows run through the ordinary split-K path and share
// the prefix's K/V tiles in L2.
//
// One CTA per row: the row walks its parent chain into a shared-memory bitmap
// of tree nodes (at most n_rows steps: a parent index that is not smaller than
// its child, or out of range, ends the walk and records ATTN_ERR_INVALID_ARG in
// the device status word; the nodes walked up to that link, the row itself
// included, stay visible and the ancestors above it are hidden), then writes
// the mask row with coalesced stores.
#include "common.cuh"
#include "internal.h"

namespace attn {

namespace {

constexpr int kTreeThreads = 256;
constexpr int kMaxTreeRows = 4096;   // bitmap of 4096 nodes: 512 bytes

__global__ void __launch_bounds__(kTreeThreads) tree_mask_kernel(const int32_t* parent, int32_t n_rows,
                                                                  int32_t prefix_cells, int32_t n_cells, float* mask,
                                                                  int64_t mask_sr, int* status) {
  __shared__ uint32_t anc[kMaxTreeRows / 32];
  const int r = blockIdx.x, tid = threadIdx.x;
  for (int i = tid; i < kMaxTreeRows / 32; i += kTreeThreads) anc[i] = 0u;
  __syncthreads();
  if (tid == 0) {
    int node = r;
    for (int steps = 0; node >= 0 && steps <= n_rows; ++steps) {
      anc[node >> 5] |= 1u << (node & 31);
      const int up = __ldg(parent + node);
      if (up >= node || up < -1) {   // not heap order: hide the ancestors above
        record_status(status, ATTN_ERR_INVALID_ARG);
        break;
      }
      node = up;
    }
  }
  __syncthreads();
  float* row = mask + (int64_t)r * mask_sr;
  for (int64_t c = tid; c < n_cells; c += kTreeThreads) {
    bool vis = c < prefix_cells;
    const int64_t node = c - prefix_cells;
    if (!vis && node < n_rows) vis = (anc[node >> 5] >> (node & 31)) & 1u;
    row[c] = vis ? 0.f : neg_inf();
  }
}

}  // namespace

cudaError_t launch_tree_mask(const int32_t* parent, int32_t n_rows, int32_t prefix_cells, int32_t n_cells,
                             float* mask, int64_t mask_sr, int* status, cudaStream_t stream) {
  tree_mask_kernel<<<dim3((unsigned)n_rows), kTreeThreads, 0, stream>>>(parent, n_rows, prefix_cells, n_cells,
                                                                       mask, mask_sr, status);
  return cudaGetLastError();
}

int max_tree_rows() { return kMaxTreeRows; }

}  // namespace attn
