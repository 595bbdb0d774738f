// noalloc.cu -- attn_decode_noalloc: split-K decode for callers that cannot
// allocate device memory.
//
// Who needs it: code that runs where a cudaMalloc is not allowed or not
// wanted -- inside a real-time or latency-critical loop that must never block
// in the allocator, in a plugin or callback that does not own a memory pool,
// or in a caller that only ever receives pointers to its inputs and outputs
// and has no place to keep a workspace.  attn_decode needs a caller-owned
// workspace for the split partials; this entry point keeps them instead in
// one fixed, file-scope device array that the CUDA runtime creates when the
// library is loaded on a GPU, so a call allocates nothing.
//
// Costs and limits:
//  * the array is kNoAllocScratchBytes (16 MiB) on every GPU the process uses
//    the library on, held until the process exits;
//  * a problem whose partials need more than that is refused with
//    ATTN_ERR_WORKSPACE (use attn_decode with a workspace instead);
//  * every call uses the same array: two calls that may overlap on the GPU
//    (different streams, or different host threads, on one device) race and
//    corrupt each other's results; order them on one stream;
//  * nothing in the array has to start at zero: each call writes every
//    partial record it later reads, so a previous call's leftovers are
//    harmless;
//  * the first call on each device resolves the array's device address with
//    cudaGetSymbolAddress (no allocation); make that first call before any
//    stream capture on that device.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "attn.h"
#include "internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 16u << 20;   // 16 MiB

// The scratch.  In host code this name is only a handle for the runtime's
// symbol lookup, never a device address; kernels get the address resolved
// below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

extern "C" int32_t attn_decode_noalloc(const attn_args* args, void* stream) {
  // Arguments and device first, so this call refuses exactly what attn_decode
  // refuses (an unsupported device included) before touching the array.
  const int32_t ok = attn_supports(args, ATTN_OP_DECODE);
  if (ok != ATTN_OK) return ok;
  const int32_t dev_ok = attn::check_device();
  if (dev_ok != ATTN_OK) return dev_ok;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();   // leave no error behind for the next call to report
    attn::set_last_error("attn_decode_noalloc: no usable current device");
    return ATTN_ERR_CUDA;
  }
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess || p == nullptr) {
        cudaGetLastError();
        attn::set_last_error("attn_decode_noalloc: cudaGetSymbolAddress of the scratch array failed");
        return ATTN_ERR_CUDA;
      }
      g_scratch_ptr[dev] = p;
    }
    scratch = g_scratch_ptr[dev];
  }
  const size_t need = attn_workspace_size(args, ATTN_OP_DECODE, 0);
  if (need > kNoAllocScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "attn_decode_noalloc: this problem needs %zu bytes of scratch; the built-in array holds %zu "
             "(call attn_decode with a workspace instead)",
             need, kNoAllocScratchBytes);
    attn::set_last_error(msg);
    return ATTN_ERR_WORKSPACE;
  }
  return attn_decode(args, scratch, kNoAllocScratchBytes, stream);
}
