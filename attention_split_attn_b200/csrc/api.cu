// api.cu -- the C ABI of libattn_b200 (declared in include/attn.h):
// argument validation, the slice planner, workspace sizing, TMA descriptors,
// the device status word, and dispatch to the kernel launchers.
//
// Refusal instead of a wrong result: every shape, dtype, stride or workspace
// the kernels do not cover is rejected here before any launch (the
// supports_op refusal of strix-llama.cpp PR #115: a backend declines an op it
// cannot compute rather than computing it wrongly; TensorFold PR #2595's
// launch guard: a grid is launched only where it stays inside the buffers).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "attn.h"
#include "common.cuh"
#include "internal.h"

namespace attn {
namespace {

thread_local std::string g_last_error;

int32_t fail(int32_t status, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return status;
}

int dtype_size(int32_t t) {
  switch (t) {
    case ATTN_F32: return 4;
    case ATTN_F16: return 2;
    case ATTN_BF16: return 2;
    case ATTN_FP8_E4M3: return 1;
    case ATTN_I8: return 1;
    default: return 0;
  }
}

// ---- device facts ------------------------------------------------------------
constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool init = false;
  int sms = 0;
  int* status = nullptr;   // device address of g_status_word on this device
};
std::mutex g_dev_mutex;
DeviceInfo g_dev[kMaxDevices];

}  // namespace
}  // namespace attn

// One status word per device, written by kernels that gave up on a bounded wait.
__device__ int g_status_word = 0;

namespace attn {
namespace {

// A failed runtime query is cleared (cudaGetLastError) before returning, so
// that a later launch check does not report it again.
int32_t device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return fail(ATTN_ERR_CUDA, "cudaGetDevice failed");
  }
  std::lock_guard<std::mutex> lk(g_dev_mutex);
  DeviceInfo& d = g_dev[dev];
  if (!d.init) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return fail(ATTN_ERR_CUDA, "cannot query device %d", dev);
    }
    if (major != 10 || minor != 0)
      return fail(ATTN_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", dev,
                  major, minor);
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_status_word) != cudaSuccess) {
      cudaGetLastError();
      return fail(ATTN_ERR_CUDA, "cannot resolve the device status word");
    }
    d.status = static_cast<int*>(addr);
    d.init = true;
  }
  *out = &d;
  return ATTN_OK;
}

// ---- TMA descriptors ---------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

CUtensorMapDataType tma_dtype(int32_t t) {
  switch (t) {
    case ATTN_F32: return CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    case ATTN_F16: return CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    case ATTN_FP8_E4M3:
    case ATTN_I8: return CU_TENSOR_MAP_DATA_TYPE_UINT8;   // raw codes; the kernel decodes them
    default: return CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  }
}

// 3-D map over a [cells][heads][D] cache: box = (box_d, box_heads, box_cells);
// with swizzle the box rows are 128 bytes and stored with the 128-byte
// swizzle (box row index = cell * box_heads + head).
int32_t make_kv_map(CUtensorMap* map, const void* base, int32_t type, int D, int Hkv, int N,
                    int64_t stride_cell, int64_t stride_head, int box_cells, int box_d = 0,
                    bool swizzle128 = false, int box_heads = 1) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const int es = dtype_size(type);
  // A stride of an extent-1 dimension is never used; give the encoder a legal one.
  const int64_t sh = Hkv > 1 ? stride_head : D;
  const int64_t sc = N > 1 ? stride_cell : D;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)N};
  cuuint64_t strides[2] = {(cuuint64_t)(sh * es), (cuuint64_t)(sc * es)};
  cuuint32_t box[3] = {(cuuint32_t)(box_d > 0 ? box_d : D), (cuuint32_t)box_heads, (cuuint32_t)box_cells};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(map, tma_dtype(type), 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE,
                   swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return ATTN_OK;
}

// ---- validation ----------------------------------------------------------------
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_quantized(int32_t t) { return t == ATTN_FP8_E4M3 || t == ATTN_I8; }

int32_t validate_common(const attn_args* a, int32_t op) {
  if (!a) return fail(ATTN_ERR_INVALID_ARG, "args is NULL");
  for (int i = op == ATTN_OP_PREFILL ? 1 : 0; i < 5; ++i)
    if (a->reserved[i] != 0) return fail(ATTN_ERR_INVALID_ARG, "reserved fields must be zero");
  if (a->n_rows < 0 || a->n_cells < 0) return fail(ATTN_ERR_INVALID_ARG, "negative n_rows or n_cells");
  if (a->n_head_q <= 0 || a->n_head_kv <= 0)
    return fail(ATTN_ERR_INVALID_ARG, "n_head_q and n_head_kv must be positive");
  if (a->n_head_q % a->n_head_kv != 0)
    return fail(ATTN_ERR_INVALID_ARG, "n_head_q (%d) is not a multiple of n_head_kv (%d)", a->n_head_q,
                a->n_head_kv);
  if (!dtype_size(a->q_type) || !dtype_size(a->kv_type) || !dtype_size(a->out_type))
    return fail(ATTN_ERR_INVALID_ARG, "unknown dtype");
  if (is_quantized(a->q_type) || is_quantized(a->out_type))
    return fail(ATTN_ERR_UNSUPPORTED, "Q and out cannot be e4m3 or int8 (only the K/V cache can)");
  if (is_quantized(a->kv_type)) {
    if (op != ATTN_OP_DECODE && op != ATTN_OP_PREFILL)
      return fail(ATTN_ERR_UNSUPPORTED, "e4m3/int8 K/V caches are supported by attn_decode and attn_prefill only");
    if (a->n_cells > 0 && (!a->k_scale || !a->v_scale))
      return fail(ATTN_ERR_INVALID_ARG, "an e4m3/int8 cache needs k_scale and v_scale");
    if (a->n_cells > 1 && a->scale_stride_cell < a->n_head_kv)
      return fail(ATTN_ERR_INVALID_ARG, "scale_stride_cell is smaller than n_head_kv");
  } else if (a->k_scale || a->v_scale) {
    return fail(ATTN_ERR_INVALID_ARG, "k_scale/v_scale are only for e4m3/int8 caches");
  }
  if (a->head_dim != 64 && a->head_dim != 128 && a->head_dim != 256)
    return fail(ATTN_ERR_UNSUPPORTED, "head_dim %d not in {64, 128, 256}", a->head_dim);
  const int G = a->n_head_q / a->n_head_kv;
  if (G > 16) return fail(ATTN_ERR_UNSUPPORTED, "GQA group %d > 16", G);
  if ((a->row_begin == nullptr) != (a->row_end == nullptr))
    return fail(ATTN_ERR_INVALID_ARG, "row_begin and row_end must both be given or both be NULL");
  if ((a->cell_seq == nullptr) != (a->row_seq == nullptr))
    return fail(ATTN_ERR_INVALID_ARG, "cell_seq and row_seq must both be given or both be NULL");
  if (a->causal != 0 && a->causal != 1) return fail(ATTN_ERR_INVALID_ARG, "causal must be 0 or 1");
  if (a->mask && a->mask_stride_row < 0) return fail(ATTN_ERR_INVALID_ARG, "negative mask stride");
  if (a->n_slices < 0 || a->n_slices > 64) return fail(ATTN_ERR_INVALID_ARG, "n_slices must be 0..64");
  if (a->max_row_len < 0) return fail(ATTN_ERR_INVALID_ARG, "negative max_row_len");
  if (a->grid_order != 0 && a->grid_order != 1) return fail(ATTN_ERR_INVALID_ARG, "grid_order must be 0 or 1");
  if (!(a->scale == a->scale)) return fail(ATTN_ERR_INVALID_ARG, "scale is NaN");
  if (a->n_rows == 0) return ATTN_OK;
  if (!a->q || !a->out) return fail(ATTN_ERR_INVALID_ARG, "q or out is NULL");
  if (a->n_cells > 0 && (!a->k || !a->v)) return fail(ATTN_ERR_INVALID_ARG, "k or v is NULL");
  if (a->q_stride_row < 0 || a->q_stride_head < 0 || a->o_stride_row < 0 || a->o_stride_head < 0 ||
      a->kv_stride_cell < 0 || a->kv_stride_head < 0)
    return fail(ATTN_ERR_INVALID_ARG, "negative stride");
  const int es = dtype_size(a->kv_type);
  if (a->n_cells > 0) {
    if (!aligned16(a->k) || !aligned16(a->v))
      return fail(ATTN_ERR_UNSUPPORTED, "k and v must be 16-byte aligned");
    if ((a->kv_stride_cell * es) % 16 || (a->kv_stride_head * es) % 16)
      return fail(ATTN_ERR_UNSUPPORTED, "kv strides must be multiples of 16 bytes");
    if ((a->n_cells > 1 && a->kv_stride_cell == 0) || (a->n_head_kv > 1 && a->kv_stride_head == 0))
      return fail(ATTN_ERR_UNSUPPORTED, "zero kv stride (broadcast caches are not supported)");
  }
  return ATTN_OK;
}

// ---- decode planning -------------------------------------------------------------
constexpr int kSliceGrain = 32;     // slices are cut at multiples of 32 cells

struct DecodeShape {
  bool mma;       // tensor-core kernels (16-bit cache, Q in the cache dtype)
  bool stream;    // balanced persistent scheme (mma and no forced slice count)
  int32_t S, C, hpw, hg;
  int32_t W;      // balanced scheme: warps of the persistent grid
};

int pick_hpw(int G) { return G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : 8; }

// Two schemes.  With the tensor-core kernels and no forced slice count, every
// resident warp takes an equal run of the flattened (row, KV head, 16-cell
// tile) space (decode_stream.cu).  Otherwise the (rows, heads, slices) grid:
// S slices per row (forced, or about 256 cells each -- 2048 for an e4m3 or
// int8 cache --, at most 16 CTAs per SM in all and at most 64 slices), each C cells long on the 32-cell grid, the
// last slice taking whatever remains of a longer row.
DecodeShape plan_decode(const attn_args* a, int sms) {
  DecodeShape d;
  const int G = a->n_head_q / a->n_head_kv;
  d.mma = decode_uses_mma(a->kv_type, a->q_type, a->q, a->q_stride_row, a->q_stride_head);
  // one-byte caches take the balanced tensor-core kernel too (codes widened
  // to f16 in registers); forced slice counts keep the CUDA-core grid kernel
  const bool mma8 = a->n_slices == 0 && decode_stream8_supported(a->kv_type, a->q_type, a->q, a->q_stride_row,
                                                                 a->q_stride_head, a->head_dim, G);
  d.stream = (d.mma && a->n_slices == 0) || mma8;
  d.hg = G > 8 ? 2 : 1;
  d.hpw = G > 8 ? 8 : pick_hpw(G);
  d.W = d.stream ? decode_stream_warps(a->kv_type, a->head_dim, G, sms) : 0;
  int64_t max_len = a->max_row_len > 0 ? std::min(a->max_row_len, a->n_cells) : a->n_cells;
  max_len = std::max<int64_t>(max_len, 1);
  int64_t S = a->n_slices;
  if (S == 0) {
    const int64_t units = (int64_t)a->n_rows * a->n_head_kv;
    // e4m3 / int8 caches run on the CUDA cores, where longer slices pay
    // (measured on the quantized GQA decode batch: 2048-cell slices 11%
    // faster than 256-cell ones)
    const int64_t grain = is_quantized(a->kv_type) ? 2048 : 256;
    S = (max_len + grain - 1) / grain;
    const int64_t cap = std::max<int64_t>(1, (16LL * std::max(sms, 1)) / std::max<int64_t>(units, 1));
    S = std::min(S, cap);
    S = std::min<int64_t>(std::max<int64_t>(S, 1), 64);
  }
  int64_t C = (max_len + S - 1) / S;
  C = (C + kSliceGrain - 1) / kSliceGrain * kSliceGrain;
  d.S = d.stream ? 0 : (int32_t)S;
  d.C = (int32_t)std::max<int64_t>(C, kSliceGrain);
  return d;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Workspace layout: [row_tiles (balanced scheme)] [partial o records] [partial (m, l)].
struct DecodeWs {
  size_t tiles_off, o_off, ml_off, total;
};

DecodeWs decode_ws_layout(const attn_args* a, const DecodeShape& d) {
  DecodeWs w{0, 0, 0, 0};
  const int G = a->n_head_q / a->n_head_kv;
  size_t records;
  if (d.stream) {
    w.tiles_off = 0;
    w.o_off = align256(((size_t)a->n_rows + 1) * sizeof(int64_t));
    records = ((size_t)d.W + (size_t)a->n_rows * a->n_head_kv) * G;
  } else {
    if (d.S <= 1) return w;
    records = (size_t)a->n_rows * a->n_head_q * d.S;
  }
  w.ml_off = w.o_off + align256(records * a->head_dim * sizeof(float));
  w.total = w.ml_off + align256(records * 2 * sizeof(float));
  return w;
}

size_t decode_ws_bytes(const attn_args* a, const DecodeShape& d) { return decode_ws_layout(a, d).total; }

int32_t check_decode(const attn_args* a) {
  int32_t st = validate_common(a, ATTN_OP_DECODE);
  if (st != ATTN_OK) return st;
  const int G = a->n_head_q / a->n_head_kv;
  if (!decode_shape_supported(a->kv_type, a->head_dim, G))
    return fail(ATTN_ERR_UNSUPPORTED, "decode: unsupported kv dtype/head_dim/group");
  return ATTN_OK;
}

// ---- selected-key planning ---------------------------------------------------------
constexpr int kMaxSel = 4096;

int32_t check_selected_base(const attn_args* a) {
  int32_t st = validate_common(a, ATTN_OP_SELECTED);
  if (st != ATTN_OK) return st;
  if (a->row_begin || a->row_end || a->cell_seq || a->row_seq || a->mask || a->causal)
    return fail(ATTN_ERR_INVALID_ARG,
                "selected: the op is maskless; row ranges, sequence ids, causal and mask must be unset");
  if (a->kv_type != ATTN_F16 && a->kv_type != ATTN_BF16)
    return fail(ATTN_ERR_UNSUPPORTED, "selected: K/V must be F16 or BF16");
  if (a->q_type != a->kv_type) return fail(ATTN_ERR_UNSUPPORTED, "selected: Q must be in the K/V dtype");
  if (a->n_rows > 0 && ((reinterpret_cast<uintptr_t>(a->q) & 3u) || (a->q_stride_row % 2) || (a->q_stride_head % 2)))
    return fail(ATTN_ERR_UNSUPPORTED, "selected: Q must be 4-byte aligned with even strides");
  return ATTN_OK;
}

struct SelShape {
  int32_t S, C;
};

// Parts per row: one when the (row, KV head) units fill the GPU about twice
// over, else enough parts to (the pages' rule: split rows when the grid would
// under-fill the device), at most 64 and at most one per 32-cell block.
SelShape plan_selected(const attn_args* a, int n_sel, int sms) {
  SelShape s;
  int64_t S = a->n_slices;
  if (S == 0) {
    const int64_t units = std::max<int64_t>(1, (int64_t)a->n_rows * a->n_head_kv);
    const int64_t target = 4LL * std::max(sms, 1);
    S = units >= target ? 1 : (target + units - 1) / units;
  }
  S = std::min<int64_t>(S, std::max<int64_t>(1, (n_sel + 31) / 32));
  S = std::min<int64_t>(std::max<int64_t>(S, 1), 64);
  int64_t C = (n_sel + S - 1) / S;
  C = (C + 31) / 32 * 32;
  s.S = (int32_t)S;
  s.C = (int32_t)std::max<int64_t>(C, 32);
  return s;
}

struct SelWs {
  size_t count_off, o_off, ml_off, total;
};

SelWs selected_ws_layout(const attn_args* a, int n_sel, const SelShape& sh) {
  SelWs w;
  w.count_off = align256((size_t)a->n_rows * n_sel * sizeof(int32_t));
  w.o_off = w.count_off + align256((size_t)a->n_rows * sizeof(int32_t));
  w.ml_off = w.o_off;
  w.total = w.o_off;
  if (sh.S > 1) {
    const size_t records = (size_t)a->n_rows * a->n_head_q * sh.S;
    w.ml_off = w.o_off + align256(records * a->head_dim * sizeof(float));
    w.total = w.ml_off + align256(records * 2 * sizeof(float));
  }
  return w;
}

// ---- prefill planning ---------------------------------------------------------------
constexpr int kPfTile = 128;   // rows and cells per prefill tile

bool unified_route(const attn_args* a);

int32_t check_prefill(const attn_args* a) {
  int32_t st = validate_common(a, ATTN_OP_PREFILL);
  if (st != ATTN_OK) return st;
  if (is_quantized(a->kv_type)) {
    // codes widened to the Q dtype in the workspace, then the 16-bit path
    if (a->q_type != ATTN_F16 && a->q_type != ATTN_BF16)
      return fail(ATTN_ERR_UNSUPPORTED, "prefill over an e4m3/int8 cache: Q must be F16 or BF16");
    if (a->n_cells > 0 && (!aligned16(a->k) || !aligned16(a->v) ||
                           (a->n_cells > 1 && a->kv_stride_cell % 16) || (a->n_head_kv > 1 && a->kv_stride_head % 16)))
      return fail(ATTN_ERR_UNSUPPORTED, "prefill over an e4m3/int8 cache: K/V and their strides 16-byte aligned");
  } else {
    if (a->kv_type != ATTN_F16 && a->kv_type != ATTN_BF16)
      return fail(ATTN_ERR_UNSUPPORTED, "prefill: K/V must be F16 or BF16");
    if (a->q_type != a->kv_type) return fail(ATTN_ERR_UNSUPPORTED, "prefill: Q must be in the K/V dtype");
  }
  if (a->head_dim != 64 && a->head_dim != 128 && a->head_dim != 256)
    return fail(ATTN_ERR_UNSUPPORTED, "prefill: head_dim %d not in {64, 128, 256}", a->head_dim);
  if (a->reserved[0] < 0 || a->reserved[0] > 1000000)
    return fail(ATTN_ERR_INVALID_ARG, "prefill: reserved[0] (the bounded-wait test) must be 0..1000000 us");
  if (a->reserved[0] != 0 && unified_route(a))
    return fail(ATTN_ERR_INVALID_ARG, "prefill: the bounded-wait test runs on the dense tensor-core kernel only");
  if (a->n_rows > 0) {
    if (!aligned16(a->q)) return fail(ATTN_ERR_UNSUPPORTED, "prefill: q must be 16-byte aligned");
    if ((a->n_rows > 1 && (a->q_stride_row % 8)) || (a->n_head_q > 1 && (a->q_stride_head % 8)) ||
        (a->n_rows > 1 && a->q_stride_row == 0) || (a->n_head_q > 1 && a->q_stride_head == 0))
      return fail(ATTN_ERR_UNSUPPORTED, "prefill: q strides must be nonzero multiples of 16 bytes");
  }
  const int64_t n_rt = ((int64_t)a->n_rows + kPfTile - 1) / kPfTile;
  const int G = a->n_head_q / a->n_head_kv;
  const int64_t ctas = 4 * n_rt * a->n_head_kv * (a->head_dim <= 128 ? (G + 1) / 2 : G);   // split parts included
  const int64_t n_kt = ((int64_t)a->n_cells + kPfTile - 1) / kPfTile;
  if (ctas > 0x7fffffffLL || n_rt * n_kt + n_kt * a->n_head_kv > 0x7fffffffLL)
    return fail(ATTN_ERR_UNSUPPORTED, "prefill: grid too large");
  return ATTN_OK;
}

// Work units of the tensor-core kernel: (row tile, KV head, q heads per CTA),
// heaviest row tiles first.  The units of a last, partial wave over the SMs
// (or every unit, when there are fewer units than SMs) are split into k
// parts over their cell tiles, k = SMs / (those units) clamped to 2..32, so
// the last wave holds shorter pieces; the parts' (m, l, O) are folded by the
// last part to finish.
struct PrefillSplit {
  int64_t units, n_full, n_split;   // n_split units of k parts each
  int32_t k;
  int64_t ctas() const { return n_full + n_split * k; }
};

// Packed rows: with fewer rows than a tile and several q heads per KV head,
// a tile's 128 lanes hold 128 / G rows x the G heads of one KV group, so each
// K and V tile is read once for all of them (draft-tree rows, short prefills).
int32_t prefill_pack(const attn_args* a) {
  const int G = a->n_head_q / a->n_head_kv;
  return (G >= 2 && G <= kPfTile && a->n_rows < kPfTile) ? G : 1;
}
int32_t prefill_rows_per_tile(const attn_args* a) { return kPfTile / prefill_pack(a); }

PrefillSplit plan_prefill_split(const attn_args* a, int sms) {
  PrefillSplit s{};
  const int rpt = prefill_rows_per_tile(a);
  const int64_t n_rt = ((int64_t)a->n_rows + rpt - 1) / rpt;
  const int G = a->n_head_q / a->n_head_kv;
  s.units = n_rt * a->n_head_kv * (prefill_pack(a) > 1 ? 1 : a->head_dim <= 128 ? (G + 1) / 2 : G);
  const int64_t r = s.units > sms ? s.units % sms : s.units;
  const int64_t k = r > 0 ? std::min<int64_t>(32, sms / r) : 1;
  s.k = (int32_t)k;
  s.n_split = k >= 2 ? r : 0;
  s.n_full = s.units - s.n_split;
  if (k < 2) s.k = 1;
  return s;
}

struct PrefillWs {
  size_t vbad_off, kn2_off, bits_off, cnt_off, po_off, pml_off, total;
};

PrefillWs prefill_ws_layout(const attn_args* a, const PrefillSplit& sp) {
  const size_t rpt = (size_t)prefill_rows_per_tile(a);
  const size_t n_rt = ((size_t)a->n_rows + rpt - 1) / rpt;
  const size_t n_kt = ((size_t)a->n_cells + kPfTile - 1) / kPfTile;
  PrefillWs w;
  w.vbad_off = align256(n_rt * n_kt);
  w.kn2_off = w.vbad_off + align256(n_kt * a->n_head_kv);
  w.bits_off = w.kn2_off + align256(n_kt * a->n_head_kv * sizeof(float));
  // visibility bits of every tile when a mask is given (1/32 of the mask's size)
  const size_t bits = a->mask ? n_rt * n_kt * (size_t)kPfTile * 16 : 0;
  w.cnt_off = w.bits_off + align256(bits);
  // split units: a counter each, and per part and q head slot the 128 rows'
  // unnormalised O [D] and (m, l)
  const size_t hpc = a->head_dim <= 128 ? 2 : 1;
  const size_t recs = (size_t)sp.n_split * (size_t)sp.k * hpc * kPfTile;
  w.po_off = w.cnt_off + align256((size_t)sp.n_split * 2 * kPfTile * sizeof(int));   // per (unit, slot, row)
  w.pml_off = w.po_off + align256(recs * a->head_dim * sizeof(float));
  w.total = w.pml_off + align256(recs * 2 * sizeof(float));
  return w;
}

void record_event(void* const* events, int i, cudaStream_t s) {
  if (events && events[i]) cudaEventRecord(static_cast<cudaEvent_t>(events[i]), s);
}

// ---- unified-cache route (decode and prefill) -----------------------------------
// With per-cell sequence ids the cells of a row's sequence are scattered over
// the cache, so the dense kernels would stream every cell for every row.
// Instead each row's visible cells are listed (same sequence, causal, mask
// != -inf) and the selected-key gather kernel runs on the lists, adding the
// mask bias per cell; rows are split into parts (folded by split_k_reduce)
// as for the selected op.  Taken for 16-bit K/V with Q in their dtype, and
// with ALiBi only when cell and row positions are given (the gather kernel's
// distances use them as they are).
bool unified_route(const attn_args* a) {
  return a->cell_seq && a->row_seq && a->n_cells > 0 && (a->kv_type == ATTN_F16 || a->kv_type == ATTN_BF16) &&
         a->q_type == a->kv_type && (reinterpret_cast<uintptr_t>(a->q) & 3u) == 0 && a->q_stride_row % 2 == 0 &&
         a->q_stride_head % 2 == 0 && (!a->alibi_slopes || (a->cell_pos && a->row_pos));
}

// Parts per row: forced by n_slices, else enough that a part holds at most
// about 4096 cells of the longest possible list (rows' lists differ wildly in
// length; a part past the end of its row's list exits at once).
SelShape plan_unified(const attn_args* a, int sms) {
  if (a->n_slices > 0) return plan_selected(a, a->n_cells, sms);
  const int64_t max_len = a->max_row_len > 0 ? std::min(a->max_row_len, a->n_cells) : a->n_cells;
  const int64_t S = std::min<int64_t>(64, std::max<int64_t>(1, (max_len + 4095) / 4096));
  SelShape sh;
  sh.S = (int32_t)S;
  int64_t C = (a->n_cells + S - 1) / S;
  C = (C + 31) / 32 * 32;
  sh.C = (int32_t)std::max<int64_t>(C, 32);
  return sh;
}

size_t unified_ws_bytes(const attn_args* a, int sms) {
  return selected_ws_layout(a, a->n_cells, plan_unified(a, sms)).total;
}

int32_t run_unified(const attn_args* a, void* ws, size_t ws_bytes, cudaStream_t s, void* const events[3],
                    const DeviceInfo* di) {
  const SelShape sh = plan_unified(a, di->sms);
  const SelWs wl = selected_ws_layout(a, a->n_cells, sh);
  if (ws == nullptr || ws_bytes < wl.total)
    return fail(ATTN_ERR_WORKSPACE, "unified-cache attention needs %zu workspace bytes, got %zu", wl.total, ws_bytes);
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(ATTN_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  const int64_t blocks = (int64_t)a->n_rows * a->n_head_kv * sh.S;
  if (blocks > 0x7fffffffLL) return fail(ATTN_ERR_UNSUPPORTED, "grid of %lld CTAs is too large", (long long)blocks);
  char* wsb = static_cast<char*>(ws);
  SelectedPlan p{};
  p.R = a->n_rows; p.Hq = a->n_head_q; p.Hkv = a->n_head_kv; p.G = a->n_head_q / a->n_head_kv;
  p.D = a->head_dim; p.N = a->n_cells;
  p.q = a->q; p.q_sr = a->q_stride_row; p.q_sh = a->q_stride_head;
  p.k = a->k; p.v = a->v; p.kv_sc = a->kv_stride_cell; p.kv_sh = a->kv_stride_head; p.kv_type = a->kv_type;
  p.out = OutSpec{a->out, a->out_type, a->o_stride_row, a->o_stride_head};
  p.lg = Logits{a->scale, a->softcap, a->alibi_slopes, a->sinks};
  p.cell_pos = a->cell_pos; p.row_pos = a->row_pos;
  p.mask = a->mask; p.mask_sr = a->mask_stride_row;
  p.n_sel = a->n_cells;   // row stride of the lists
  p.compact = reinterpret_cast<int32_t*>(wsb);
  p.count = reinterpret_cast<int32_t*>(wsb + wl.count_off);
  p.S = sh.S; p.C = sh.C;
  if (sh.S > 1) {
    p.part.o = reinterpret_cast<float*>(wsb + wl.o_off);
    p.part.ml = reinterpret_cast<float*>(wsb + wl.ml_off);
    p.part.S = sh.S;
  }
  p.status = di->status;
  const RowFilter f{a->row_begin, a->row_end, a->cell_seq, a->row_seq, a->cell_pos, a->row_pos,
                    a->causal, a->mask, a->mask_stride_row};
  record_event(events, 0, s);
  cudaError_t e = launch_visible_lists(p, f, s);
  if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "visible-list launch: %s", cudaGetErrorString(e));
  e = launch_selected(p, s);
  if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "gather launch: %s", cudaGetErrorString(e));
  record_event(events, 1, s);
  if (sh.S > 1) {
    CombinePlan cp{};
    cp.R = a->n_rows; cp.Hq = a->n_head_q; cp.Hkv = a->n_head_kv; cp.G = p.G; cp.D = a->head_dim;
    cp.out = p.out; cp.sinks = a->sinks; cp.part = p.part;
    cp.mode = 0;
    cp.row_len = p.count; cp.C = sh.C; cp.N = a->n_cells;
    cp.use_pdl = (events && events[1]) ? 0 : 1;
    e = launch_combine(cp, s);
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "combine launch: %s", cudaGetErrorString(e));
  }
  record_event(events, 2, s);
  return ATTN_OK;
}

}  // namespace
}  // namespace attn

namespace attn {
void set_last_error(const char* msg) { g_last_error = msg; }
int32_t check_device() {
  DeviceInfo* di = nullptr;
  return device_info(&di);
}
}  // namespace attn

using namespace attn;

extern "C" {

int32_t attn_abi_version(void) { return ATTN_ABI_VERSION; }

const char* attn_strerror(int32_t s) {
  switch (s) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
    case ATTN_ERR_WORKSPACE: return "ATTN_ERR_WORKSPACE";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
    case ATTN_ERR_DEVICE_TIMEOUT: return "ATTN_ERR_DEVICE_TIMEOUT";
    default: return "unknown attn_status";
  }
}

const char* attn_last_error(void) { return g_last_error.c_str(); }

// ---- masked route of selected-key attention ----------------------------------------
// The dense prefill arguments under which the masked route computes the
// selected op: the selected arguments plus the per-cell mask (row stride a
// multiple of 4 floats), no ranges, sequences or causal flag; positions as given.
int64_t sel_mask_ld(const attn_args* b) { return ((int64_t)b->n_cells + 3) / 4 * 4; }
attn_args sel_mask_args(const attn_args* b, float* mask) {
  attn_args pa = *b;
  pa.mask = mask;
  pa.mask_stride_row = sel_mask_ld(b);
  return pa;
}
size_t sel_mask_bytes(const attn_args* b) { return align256((size_t)b->n_rows * sel_mask_ld(b) * sizeof(float)); }

int32_t check_selected_masked(const attn_args* b) {
  int32_t st = check_selected_base(b);
  if (st != ATTN_OK) return st;
  // the dense route's own limits (the mask pointer only needs to be non-NULL and aligned here)
  const attn_args pa = sel_mask_args(b, reinterpret_cast<float*>(static_cast<uintptr_t>(256)));
  return check_prefill(&pa);
}

// Prefill over an e4m3 / int8 cache: K and V widened to F16 (code x scale,
// rounded once) into two contiguous [n_cells][n_head_kv][head_dim] arrays at
// the start of the workspace, and a BF16 Q copied to F16 after them (the
// tensor cores take both operands in one type); the prefill then runs on
// these copies.
size_t widened_kv_bytes(const attn_args* a) {
  return align256((size_t)a->n_cells * a->n_head_kv * a->head_dim * 2);
}
size_t widened_q_bytes(const attn_args* a) {
  return a->q_type == ATTN_BF16 ? align256((size_t)a->n_rows * a->n_head_q * a->head_dim * 2) : 0;
}
size_t widened_bytes(const attn_args* a) { return 2 * widened_kv_bytes(a) + widened_q_bytes(a); }
attn_args widened_args(const attn_args* a, void* ws) {
  attn_args b = *a;
  char* base = static_cast<char*>(ws);
  b.k = base;
  b.v = base ? base + widened_kv_bytes(a) : nullptr;
  b.kv_type = ATTN_F16;
  b.kv_stride_cell = (int64_t)a->n_head_kv * a->head_dim;
  b.kv_stride_head = a->head_dim;
  b.k_scale = b.v_scale = nullptr;
  b.scale_stride_cell = 0;
  if (a->q_type == ATTN_BF16) {
    b.q = base ? base + 2 * widened_kv_bytes(a) : reinterpret_cast<void*>(static_cast<uintptr_t>(256));
    b.q_type = ATTN_F16;
    b.q_stride_row = (int64_t)a->n_head_q * a->head_dim;
    b.q_stride_head = a->head_dim;
  }
  return b;
}

int32_t attn_supports(const attn_args* a, int32_t op) {
  switch (op) {
    case ATTN_OP_DECODE: return check_decode(a);
    case ATTN_OP_SELECTED: return check_selected_base(a);
    case ATTN_OP_PREFILL: return check_prefill(a);
    case ATTN_OP_SELECTED_MASKED: return check_selected_masked(a);
    default: return fail(ATTN_ERR_INVALID_ARG, "unknown op %d", op);
  }
}

size_t attn_workspace_size(const attn_args* a, int32_t op, int32_t n_sel) {
  if (attn_supports(a, op) != ATTN_OK) return 0;
  int sms = 148;
  DeviceInfo* di = nullptr;
  if (device_info(&di) == ATTN_OK) sms = di->sms;
  switch (op) {
    case ATTN_OP_DECODE: return unified_route(a) ? unified_ws_bytes(a, sms) : decode_ws_bytes(a, plan_decode(a, sms));
    case ATTN_OP_SELECTED:
      if (n_sel < 1 || n_sel > kMaxSel) return 0;
      return selected_ws_layout(a, n_sel, plan_selected(a, n_sel, sms)).total;
    case ATTN_OP_PREFILL: {
      if (unified_route(a)) return unified_ws_bytes(a, sms);
      if (!is_quantized(a->kv_type)) return prefill_ws_layout(a, plan_prefill_split(a, sms)).total;
      const attn_args b = widened_args(a, nullptr);
      return widened_bytes(a) + prefill_ws_layout(&b, plan_prefill_split(&b, sms)).total;
    }
    case ATTN_OP_SELECTED_MASKED: {
      if (n_sel < 1 || n_sel > kMaxSel) return 0;
      const attn_args pa = sel_mask_args(a, reinterpret_cast<float*>(static_cast<uintptr_t>(256)));
      return sel_mask_bytes(a) + prefill_ws_layout(&pa, plan_prefill_split(&pa, sms)).total;
    }
    default: return 0;
  }
}


int32_t attn_decode(const attn_args* a, void* ws, size_t ws_bytes, void* stream) {
  return attn_decode_timed(a, ws, ws_bytes, stream, nullptr);
}

// New K/V rows of attn_decode_append.
struct AppendSpec {
  const void *k_new, *v_new;
  int64_t sr, sh;
};

int32_t decode_run(const attn_args* a, void* ws, size_t ws_bytes, void* stream, void* const events[3],
                   const AppendSpec* app);

int32_t attn_decode_timed(const attn_args* a, void* ws, size_t ws_bytes, void* stream,
                          void* const events[3]) {
  return decode_run(a, ws, ws_bytes, stream, events, nullptr);
}

int32_t attn_decode_append(const attn_args* a, const void* k_new, const void* v_new, int64_t new_stride_row,
                           int64_t new_stride_head, void* ws, size_t ws_bytes, void* stream) {
  int32_t st = check_decode(a);
  if (st != ATTN_OK) return st;
  if (a->n_rows == 0) return ATTN_OK;
  if (!k_new || !v_new) return fail(ATTN_ERR_INVALID_ARG, "append: k_new or v_new is NULL");
  if (!aligned16(k_new) || !aligned16(v_new) || (a->n_rows > 1 && new_stride_row % 8) ||
      (a->n_head_kv > 1 && new_stride_head % 8))
    return fail(ATTN_ERR_UNSUPPORTED, "append: new rows must be 16-byte aligned with strides that are multiples of 8");
  if (new_stride_head < a->head_dim || (a->n_rows > 1 && new_stride_row < (int64_t)a->n_head_kv * new_stride_head))
    return fail(ATTN_ERR_INVALID_ARG, "append: new row strides overlap");
  if (!a->row_end && a->n_rows > 1)
    return fail(ATTN_ERR_INVALID_ARG, "append: with several rows, row_end must say where each row's token goes");
  if (unified_route(a) || a->n_slices != 0 || !decode_uses_mma(a->kv_type, a->q_type, a->q, a->q_stride_row,
                                                                 a->q_stride_head))
    return fail(ATTN_ERR_UNSUPPORTED,
                "append: runs on the balanced tensor-core kernel (16-bit cache, Q in its dtype, n_slices 0, "
                "no per-cell sequence ids)");
  const AppendSpec app{k_new, v_new, new_stride_row, new_stride_head};
  return decode_run(a, ws, ws_bytes, stream, nullptr, &app);
}

int32_t attn_decode_cluster(const attn_args* a, void* stream) {
  int32_t st = check_decode(a);
  if (st != ATTN_OK) return st;
  const int G = a->n_head_q / a->n_head_kv;
  if (unified_route(a) || a->n_slices != 0 || (a->head_dim != 64 && a->head_dim != 128) ||
      !decode_uses_mma(a->kv_type, a->q_type, a->q, a->q_stride_row, a->q_stride_head))
    return fail(ATTN_ERR_UNSUPPORTED,
                "cluster decode: a 16-bit cache with Q in its dtype, head_dim 64 or 128, n_slices 0, no per-cell "
                "sequence ids");
  if (a->n_rows == 0) return ATTN_OK;
  if ((int64_t)a->n_rows * a->n_head_kv * 16 > 0x7fffffffLL) return fail(ATTN_ERR_UNSUPPORTED, "grid too large");
  DeviceInfo* di = nullptr;
  if ((st = device_info(&di)) != ATTN_OK) return st;
  CUtensorMap tmK, tmV;
  memset(&tmK, 0, sizeof(tmK));
  memset(&tmV, 0, sizeof(tmV));
  if (a->n_cells > 0) {
    if ((st = make_kv_map(&tmK, a->k, a->kv_type, a->head_dim, a->n_head_kv, a->n_cells, a->kv_stride_cell,
                          a->kv_stride_head, 16, 64, true)) != ATTN_OK)
      return st;
    if ((st = make_kv_map(&tmV, a->v, a->kv_type, a->head_dim, a->n_head_kv, a->n_cells, a->kv_stride_cell,
                          a->kv_stride_head, 16, 64, true)) != ATTN_OK)
      return st;
  }
  DecodePlan p{};
  p.R = a->n_rows; p.Hq = a->n_head_q; p.Hkv = a->n_head_kv; p.G = G;
  p.D = a->head_dim; p.N = a->n_cells;
  p.q = QSpec{a->q, a->q_type, a->q_stride_row, a->q_stride_head};
  p.out = OutSpec{a->out, a->out_type, a->o_stride_row, a->o_stride_head};
  p.f = RowFilter{a->row_begin, a->row_end, a->cell_seq, a->row_seq, a->cell_pos, a->row_pos,
                  a->causal, a->mask, a->mask_stride_row};
  p.lg = Logits{a->scale, a->softcap, a->alibi_slopes, a->sinks};
  p.kv_type = a->kv_type;
  p.mma = 1;
  p.status = di->status;
  const cudaError_t e = launch_decode_cluster(p, tmK, tmV, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "cluster decode launch: %s", cudaGetErrorString(e));
  return ATTN_OK;
}

int32_t decode_run(const attn_args* a, void* ws, size_t ws_bytes, void* stream, void* const events[3],
                   const AppendSpec* app) {
  int32_t st = check_decode(a);
  if (st != ATTN_OK) return st;
  if (a->n_rows == 0) return ATTN_OK;
  DeviceInfo* di = nullptr;
  if ((st = device_info(&di)) != ATTN_OK) return st;
  if (unified_route(a)) return run_unified(a, ws, ws_bytes, static_cast<cudaStream_t>(stream), events, di);
  const DecodeShape sh = plan_decode(a, di->sms);
  const size_t need = decode_ws_bytes(a, sh);
  if (need > 0 && (ws == nullptr || ws_bytes < need))
    return fail(ATTN_ERR_WORKSPACE, "decode needs %zu workspace bytes, got %zu", need, ws_bytes);
  if (need > 0 && (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(ATTN_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  const int64_t blocks = sh.stream ? sh.W : (int64_t)a->n_rows * a->n_head_kv * sh.S;
  if (blocks > 0x7fffffffLL) return fail(ATTN_ERR_UNSUPPORTED, "grid of %lld CTAs is too large", (long long)blocks);

  const bool mma = sh.mma;
  // tile maps: tensor-core kernels take 16-cell tiles in 128-byte swizzled
  // boxes (64 16-bit values or 128 one-byte codes per cell); the CUDA-core
  // grid kernel takes 32-cell tiles of whole rows
  const bool tc = sh.stream || mma;
  CUtensorMap tmK, tmV;
  memset(&tmK, 0, sizeof(tmK));
  memset(&tmV, 0, sizeof(tmV));
  if (a->n_cells > 0) {
    const int box_d = !tc ? 0 : dtype_size(a->kv_type) == 1 ? 128 : 64;
    if ((st = make_kv_map(&tmK, a->k, a->kv_type, a->head_dim, a->n_head_kv, a->n_cells, a->kv_stride_cell,
                          a->kv_stride_head, tc ? 16 : 32, box_d, tc)) != ATTN_OK)
      return st;
    if ((st = make_kv_map(&tmV, a->v, a->kv_type, a->head_dim, a->n_head_kv, a->n_cells, a->kv_stride_cell,
                          a->kv_stride_head, tc ? 16 : 32, box_d, tc)) != ATTN_OK)
      return st;
  }

  DecodePlan p{};
  p.R = a->n_rows; p.Hq = a->n_head_q; p.Hkv = a->n_head_kv; p.G = a->n_head_q / a->n_head_kv;
  p.D = a->head_dim; p.N = a->n_cells;
  p.q = QSpec{a->q, a->q_type, a->q_stride_row, a->q_stride_head};
  p.out = OutSpec{a->out, a->out_type, a->o_stride_row, a->o_stride_head};
  p.f = RowFilter{a->row_begin, a->row_end, a->cell_seq, a->row_seq, a->cell_pos, a->row_pos,
                  a->causal, a->mask, a->mask_stride_row};
  p.lg = Logits{a->scale, a->softcap, a->alibi_slopes, a->sinks};
  p.S = sh.S; p.C = sh.C; p.grid_order = a->grid_order;
  p.hpw = sh.hpw; p.hg = sh.hg; p.kv_type = a->kv_type; p.mma = mma ? 1 : 0;
  p.k_scale = a->k_scale; p.v_scale = a->v_scale; p.scale_sc = a->scale_stride_cell;
  if (app) {
    p.k_new = app->k_new; p.v_new = app->v_new; p.new_sr = app->sr; p.new_sh = app->sh;
    p.k_out = const_cast<void*>(a->k); p.v_out = const_cast<void*>(a->v);
    p.kv_sc = a->kv_stride_cell; p.kv_sh = a->kv_stride_head;
  }
  p.status = di->status;
  const DecodeWs wl = decode_ws_layout(a, sh);
  char* wsb = static_cast<char*>(ws);
  if (wl.total > 0) {
    p.part.o = reinterpret_cast<float*>(wsb + wl.o_off);
    p.part.ml = reinterpret_cast<float*>(wsb + wl.ml_off);
    p.part.S = sh.S;
  }
  if (sh.stream) {
    p.W = sh.W;
    p.row_tiles = reinterpret_cast<int64_t*>(wsb + wl.tiles_off);
    p.plan_inline = a->n_rows <= 64 ? 1 : 0;   // kInlineRows of the stream kernel
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  record_event(events, 0, s);
  cudaError_t e;
  if (sh.stream) {
    e = launch_decode_stream(p, tmK, tmV, s, events ? static_cast<cudaEvent_t>(events[1]) : nullptr);
  } else {
    e = launch_decode_slices(p, tmK, tmV, s);
    record_event(events, 1, s);
  }
  if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
  if (sh.stream || sh.S > 1) {
    CombinePlan cp{};
    cp.R = a->n_rows; cp.Hq = a->n_head_q; cp.Hkv = a->n_head_kv; cp.G = p.G; cp.D = a->head_dim;
    cp.out = p.out; cp.sinks = a->sinks; cp.part = p.part;
    cp.mode = sh.stream ? 1 : 0;
    cp.row_begin = a->row_begin; cp.row_end = a->row_end; cp.N = a->n_cells; cp.C = sh.C;
    cp.n_used = nullptr;
    cp.row_tiles = p.row_tiles; cp.W = p.W;
    // PDL overlap is off when the caller asked for an event between the two
    // kernels: the event must see the main kernel complete.
    cp.use_pdl = (events && events[1]) ? 0 : 1;
    e = launch_combine(cp, s);
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "combine launch: %s", cudaGetErrorString(e));
  }
  record_event(events, 2, s);
  return ATTN_OK;
}

int32_t attn_selected(const attn_selected_args* a, void* ws, size_t ws_bytes, void* stream) {
  return attn_selected_timed(a, ws, ws_bytes, stream, nullptr);
}

int32_t attn_selected_masked(const attn_selected_args* a, void* ws, size_t ws_bytes, void* stream) {
  return attn_selected_masked_timed(a, ws, ws_bytes, stream, nullptr);
}

int32_t attn_selected_masked_timed(const attn_selected_args* a, void* ws, size_t ws_bytes, void* stream,
                                   void* const events[3]) {
  if (!a) return fail(ATTN_ERR_INVALID_ARG, "args is NULL");
  const attn_args* b = &a->base;
  int32_t st = check_selected_masked(b);
  if (st != ATTN_OK) return st;
  if (a->n_sel < 1 || a->n_sel > kMaxSel) return fail(ATTN_ERR_UNSUPPORTED, "n_sel must be 1..%d", kMaxSel);
  if (b->n_rows == 0) return ATTN_OK;
  if (!a->sel) return fail(ATTN_ERR_INVALID_ARG, "sel is NULL");
  if (a->sel_stride_row < a->n_sel) return fail(ATTN_ERR_INVALID_ARG, "sel_stride_row is smaller than n_sel");
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(ATTN_ERR_WORKSPACE, "the masked route needs a 256-byte aligned workspace");
  const size_t mb = sel_mask_bytes(b);
  if (ws_bytes < mb) return fail(ATTN_ERR_WORKSPACE, "the masked route needs %zu bytes for its mask", mb);
  float* mask = static_cast<float*>(ws);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  record_event(events, 0, s);
  if (b->n_cells > 0) {
    const cudaError_t e = launch_sel_mask(a->sel, a->sel_stride_row, a->n_sel, b->n_rows, b->n_cells, mask,
                                          sel_mask_ld(b), s);
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "selection mask launch: %s", cudaGetErrorString(e));
  }
  const attn_args pa = sel_mask_args(b, mask);
  // the dense pass (its own workspace after the mask); the first event stays
  // in front of the mask kernel
  void* const ev2[3] = {nullptr, events ? events[1] : nullptr, events ? events[2] : nullptr};
  return attn_prefill_timed(&pa, static_cast<char*>(ws) + mb, ws_bytes - mb, stream, events ? ev2 : nullptr);
}

int32_t attn_selected_timed(const attn_selected_args* a, void* ws, size_t ws_bytes, void* stream,
                            void* const events[3]) {
  if (!a) return fail(ATTN_ERR_INVALID_ARG, "args is NULL");
  const attn_args* b = &a->base;
  int32_t st = check_selected_base(b);
  if (st != ATTN_OK) return st;
  if (a->n_sel < 1 || a->n_sel > kMaxSel) return fail(ATTN_ERR_UNSUPPORTED, "n_sel must be 1..%d", kMaxSel);
  if (b->n_rows == 0) return ATTN_OK;
  if (!a->sel) return fail(ATTN_ERR_INVALID_ARG, "sel is NULL");
  if (a->sel_stride_row < a->n_sel) return fail(ATTN_ERR_INVALID_ARG, "sel_stride_row is smaller than n_sel");
  DeviceInfo* di = nullptr;
  if ((st = device_info(&di)) != ATTN_OK) return st;
  const SelShape sh = plan_selected(b, a->n_sel, di->sms);
  const SelWs wl = selected_ws_layout(b, a->n_sel, sh);
  if (ws == nullptr || ws_bytes < wl.total)
    return fail(ATTN_ERR_WORKSPACE, "selected needs %zu workspace bytes, got %zu", wl.total, ws_bytes);
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(ATTN_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  const int64_t blocks = (int64_t)b->n_rows * b->n_head_kv * sh.S;
  if (blocks > 0x7fffffffLL || b->n_rows > 0x7fffffff)
    return fail(ATTN_ERR_UNSUPPORTED, "grid of %lld CTAs is too large", (long long)blocks);

  char* wsb = static_cast<char*>(ws);
  SelectedPlan p{};
  p.R = b->n_rows; p.Hq = b->n_head_q; p.Hkv = b->n_head_kv; p.G = b->n_head_q / b->n_head_kv;
  p.D = b->head_dim; p.N = b->n_cells;
  p.q = b->q; p.q_sr = b->q_stride_row; p.q_sh = b->q_stride_head;
  p.k = b->k; p.v = b->v; p.kv_sc = b->kv_stride_cell; p.kv_sh = b->kv_stride_head; p.kv_type = b->kv_type;
  p.out = OutSpec{b->out, b->out_type, b->o_stride_row, b->o_stride_head};
  p.lg = Logits{b->scale, b->softcap, b->alibi_slopes, b->sinks};
  p.cell_pos = b->cell_pos; p.row_pos = b->row_pos;
  p.sel = a->sel; p.sel_stride = a->sel_stride_row; p.n_sel = a->n_sel; p.n_pow2 = selected_pow2(a->n_sel);
  p.compact = reinterpret_cast<int32_t*>(wsb);
  p.count = reinterpret_cast<int32_t*>(wsb + wl.count_off);
  p.sorted_out = a->sel_sorted_out; p.count_out = a->sel_count_out;
  p.S = sh.S; p.C = sh.C;
  if (sh.S > 1) {
    p.part.o = reinterpret_cast<float*>(wsb + wl.o_off);
    p.part.ml = reinterpret_cast<float*>(wsb + wl.ml_off);
    p.part.S = sh.S;
  }
  p.status = di->status;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  record_event(events, 0, s);
  cudaError_t e = launch_select_compact(p, s);
  if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "select_compact launch: %s", cudaGetErrorString(e));
  e = launch_selected(p, s);
  if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "selected launch: %s", cudaGetErrorString(e));
  record_event(events, 1, s);
  if (sh.S > 1) {
    CombinePlan cp{};
    cp.R = b->n_rows; cp.Hq = b->n_head_q; cp.Hkv = b->n_head_kv; cp.G = p.G; cp.D = b->head_dim;
    cp.out = p.out; cp.sinks = b->sinks; cp.part = p.part;
    cp.mode = 0;
    cp.row_len = p.count; cp.C = sh.C; cp.N = b->n_cells;
    cp.use_pdl = (events && events[1]) ? 0 : 1;
    e = launch_combine(cp, s);
    if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "combine launch: %s", cudaGetErrorString(e));
  }
  record_event(events, 2, s);
  return ATTN_OK;
}

int32_t attn_prefill(const attn_args* a, void* ws, size_t ws_bytes, void* stream) {
  return attn_prefill_timed(a, ws, ws_bytes, stream, nullptr);
}

int32_t prefill_dense(const attn_args* a, void* ws, size_t ws_bytes, void* stream, void* const events[3],
                      DeviceInfo* di, bool started);

int32_t attn_prefill_timed(const attn_args* a, void* ws, size_t ws_bytes, void* stream, void* const events[3]) {
  int32_t st = check_prefill(a);
  if (st != ATTN_OK) return st;
  if (a->n_rows == 0) return ATTN_OK;
  DeviceInfo* di = nullptr;
  if ((st = device_info(&di)) != ATTN_OK) return st;
  if (unified_route(a)) return run_unified(a, ws, ws_bytes, static_cast<cudaStream_t>(stream), events, di);
  if (!is_quantized(a->kv_type)) return prefill_dense(a, ws, ws_bytes, stream, events, di, false);
  // e4m3 / int8 cache: widen K and V into the workspace, then the dense path
  // (sequence ids included: its classifier applies them)
  const size_t wb = widened_bytes(a);
  if (ws == nullptr || ws_bytes < wb)
    return fail(ATTN_ERR_WORKSPACE, "prefill over an e4m3/int8 cache needs %zu workspace bytes for the widened "
                "K/V, got %zu", wb, ws_bytes);
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(ATTN_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  const attn_args b = widened_args(a, ws);
  {   // the rest of the workspace must hold the dense path's part before anything is launched
    const PrefillWs wl = prefill_ws_layout(&b, plan_prefill_split(&b, di->sms));
    if (ws_bytes - wb < wl.total)
      return fail(ATTN_ERR_WORKSPACE, "prefill needs %zu workspace bytes, got %zu", wb + wl.total, ws_bytes);
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  record_event(events, 0, s);
  DequantPlan dp{};
  dp.N = a->n_cells; dp.Hkv = a->n_head_kv; dp.D = a->head_dim;
  dp.code_type = a->kv_type;
  dp.k = a->k; dp.v = a->v; dp.sc = a->kv_stride_cell; dp.sh = a->kv_stride_head;
  dp.k_scale = a->k_scale; dp.v_scale = a->v_scale; dp.ss = a->scale_stride_cell;
  dp.k_out = const_cast<void*>(b.k); dp.v_out = const_cast<void*>(b.v);
  dp.R = a->n_rows; dp.Hq = a->n_head_q;
  dp.q = a->q; dp.q_sr = a->q_stride_row; dp.q_sh = a->q_stride_head;
  dp.q_out = a->q_type == ATTN_BF16 ? const_cast<void*>(b.q) : nullptr;
  cudaError_t e = launch_dequant(dp, di->sms, s);
  if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "widening launch: %s", cudaGetErrorString(e));
  return prefill_dense(&b, static_cast<char*>(ws) + wb, ws_bytes - wb, stream, events, di, true);
}

// The tensor-core path over a 16-bit cache (started: event 0 was recorded by
// the caller, ahead of its own kernels).
int32_t prefill_dense(const attn_args* a, void* ws, size_t ws_bytes, void* stream, void* const events[3],
                      DeviceInfo* di, bool started) {
  int32_t st = ATTN_OK;
  const PrefillSplit sp = plan_prefill_split(a, di->sms);
  const PrefillWs wl = prefill_ws_layout(a, sp);
  if (wl.total > 0 && (ws == nullptr || ws_bytes < wl.total))
    return fail(ATTN_ERR_WORKSPACE, "prefill needs %zu workspace bytes, got %zu", wl.total, ws_bytes);
  if (wl.total > 0 && (reinterpret_cast<uintptr_t>(ws) & 255u))
    return fail(ATTN_ERR_WORKSPACE, "workspace must be 256-byte aligned");

  CUtensorMap tmQ, tmK, tmV;
  memset(&tmQ, 0, sizeof(tmQ));
  memset(&tmK, 0, sizeof(tmK));
  memset(&tmV, 0, sizeof(tmV));
  // Q as a [rows][heads][D] array with boxes of 128 rows of one head (packed:
  // 128 / G rows of the G heads of a KV group); K and V with 128-cell boxes.
  const int32_t pack = prefill_pack(a), rpt = prefill_rows_per_tile(a);
  if ((st = make_kv_map(&tmQ, a->q, a->q_type, a->head_dim, a->n_head_q, a->n_rows, a->q_stride_row,
                        a->q_stride_head, rpt, 64, true, pack)) != ATTN_OK)
    return st;
  if (a->n_cells > 0) {
    if ((st = make_kv_map(&tmK, a->k, a->kv_type, a->head_dim, a->n_head_kv, a->n_cells, a->kv_stride_cell,
                          a->kv_stride_head, kPfTile, 64, true)) != ATTN_OK)
      return st;
    if ((st = make_kv_map(&tmV, a->v, a->kv_type, a->head_dim, a->n_head_kv, a->n_cells, a->kv_stride_cell,
                          a->kv_stride_head, kPfTile, 64, true)) != ATTN_OK)
      return st;
  }

  PrefillPlan p{};
  p.R = a->n_rows; p.Hq = a->n_head_q; p.Hkv = a->n_head_kv; p.G = a->n_head_q / a->n_head_kv;
  p.D = a->head_dim; p.N = a->n_cells; p.kv_type = a->kv_type;
  p.k = a->k; p.v = a->v; p.kv_sc = a->kv_stride_cell; p.kv_sh = a->kv_stride_head;
  p.out = OutSpec{a->out, a->out_type, a->o_stride_row, a->o_stride_head};
  p.f = RowFilter{a->row_begin, a->row_end, a->cell_seq, a->row_seq, a->cell_pos, a->row_pos,
                  a->causal, a->mask, a->mask_stride_row};
  p.lg = Logits{a->scale, a->softcap, a->alibi_slopes, a->sinks};
  p.pack = pack;
  p.rpt = rpt;
  p.n_rt = (a->n_rows + rpt - 1) / rpt;
  p.n_kt = (a->n_cells + kPfTile - 1) / kPfTile;
  // q heads per CTA: 2 up to head dim 128, 1 at 256; packed: all G in one slot
  p.n_pairs = pack > 1 ? 1 : a->head_dim <= 128 ? (p.G + 1) / 2 : p.G;
  char* wsb = static_cast<char*>(ws);
  p.cls = reinterpret_cast<uint8_t*>(wsb);
  p.vbad = reinterpret_cast<uint8_t*>(wsb + wl.vbad_off);
  p.kn2 = reinterpret_cast<float*>(wsb + wl.kn2_off);
  p.bits = a->mask ? reinterpret_cast<uint32_t*>(wsb + wl.bits_off) : nullptr;
  p.n_full = sp.n_full;
  p.n_split = sp.n_split;
  p.k_split = sp.k;
  p.split_cnt = reinterpret_cast<int*>(wsb + wl.cnt_off);
  p.part_o = reinterpret_cast<float*>(wsb + wl.po_off);
  p.part_ml = reinterpret_cast<float*>(wsb + wl.pml_off);
  // Softcap polynomial: x = u + u w (k3 + w (k5 + w k7)), w = u^2, the odd
  // Taylor series of c tanh(u / c) through u^7, used for |u| <= c / 5.
  if (a->softcap > 0.f) {
    const double c = a->softcap, c2 = c * c;
    p.cap_lim = (float)(0.2 * c);
    p.k3 = (float)(-1.0 / (3.0 * c2));
    p.k5 = (float)(2.0 / (15.0 * c2 * c2));
    p.k7 = (float)(-17.0 / (315.0 * c2 * c2 * c2));
    // tanh y = y - y^3/3 + 2 y^5/15 - 17 y^7/315 + 62 y^9/2835 - ...
    const double sc = a->scale, s2 = sc * sc;
    const double a3 = -1.0 / 3.0 / c2 * sc * s2;
    const double a5 = 2.0 / 15.0 / (c2 * c2) * sc * s2 * s2;
    const double a7 = -17.0 / 315.0 / (c2 * c2 * c2) * sc * s2 * s2 * s2;
    const double a9 = 62.0 / 2835.0 / (c2 * c2 * c2 * c2) * sc * s2 * s2 * s2 * s2;
    const double s_lim = 0.4 * c / std::fabs(sc);
    auto normal = [](double v) { return std::fabs(v) >= 1.1754943508222875e-38 && std::fabs(v) <= 3.0e38; };
    if (sc != 0.0 && std::isfinite(sc) && normal(a3) && normal(a5) && normal(a7) && normal(a9) &&
        normal(s_lim) && normal(s_lim * s_lim)) {
      p.a3 = (float)a3;
      p.a5 = (float)a5;
      p.a7 = (float)a7;
      p.a9 = (float)a9;
      p.s_lim = (float)s_lim;
      p.bound2 = (float)(0.998 * s_lim * s_lim);
      p.cap_raw = 1;
      // bound path: the same series with log2(e) folded in; degree 7 for
      // |u| <= c / 3 (the next term, 62/2835 (1/3)^9 c, is below 1e-6 c)
      const double L = 1.4426950408889634, s7 = c / (3.0 * std::fabs(sc));
      p.b3 = (float)(a3 * L);
      p.b5 = (float)(a5 * L);
      p.b7 = (float)(a7 * L);
      p.b9 = (float)(a9 * L);
      p.bound7 = normal(s7 * s7) ? (float)(0.998 * s7 * s7) : -1.f;
    }
  }
  // Bound path of bf16 prefill: logits bounded through |q| max|k| (needs a
  // finite scale); the packed softcap also uses the tile norms.
  const bool scale_ok = std::isfinite(a->scale);
  p.bsc = (float)((double)a->scale * 1.4426950408889634);
  // |scale| |q| max|k| <= 30: the bound then sits within 60 of the tile's
  // true max, so no visible weight underflows
  const double s2 = (double)a->scale * a->scale;
  const double lim2 = s2 > 0.0 ? 900.0 / s2 : 1e30;
  p.nc_lim2 = scale_ok ? (float)std::min(lim2, 1e30) : -1.f;
  p.bound7 = scale_ok ? std::min(p.bound7, p.nc_lim2) : -1.f;
  p.bound9 = scale_ok && p.cap_raw ? std::min(p.bound2, p.nc_lim2) : -1.f;
  if (!p.cap_raw && a->kv_type != ATTN_BF16) p.kn2 = nullptr;
  const int oes = dtype_size(a->out_type);
  const int64_t ovec = 16 / oes;
  p.out_vec = aligned16(a->out) && (a->n_rows <= 1 || a->o_stride_row % ovec == 0) &&
              (a->n_head_q <= 1 || a->o_stride_head % ovec == 0);
  p.mask_vec = a->mask && aligned16(a->mask) && (a->n_rows <= 1 || a->mask_stride_row % 4 == 0);
  p.status = di->status;
  p.wait_ns = a->reserved[0] > 0 ? (uint64_t)a->reserved[0] * 1000ull : kWaitLimitNs;
  p.test_stall = a->reserved[0] > 0 ? 1 : 0;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!started) record_event(events, 0, s);
  cudaError_t e = launch_prefill(p, tmQ, tmK, tmV, s, nullptr);
  if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "prefill launch: %s", cudaGetErrorString(e));
  record_event(events, 1, s);
  record_event(events, 2, s);
  return ATTN_OK;
}

int32_t attn_tree_mask(const int32_t* parent, int32_t n_rows, int32_t prefix_cells, int32_t n_cells, float* mask,
                       int64_t mask_stride_row, void* stream) {
  if (n_rows < 0 || prefix_cells < 0 || n_cells < 0) return fail(ATTN_ERR_INVALID_ARG, "negative size");
  if (n_rows == 0) return ATTN_OK;
  if (!parent || !mask) return fail(ATTN_ERR_INVALID_ARG, "parent or mask is NULL");
  if (n_rows > max_tree_rows()) return fail(ATTN_ERR_UNSUPPORTED, "tree of %d rows > %d", n_rows, max_tree_rows());
  if (mask_stride_row < n_cells) return fail(ATTN_ERR_INVALID_ARG, "mask_stride_row is smaller than n_cells");
  if ((int64_t)prefix_cells + n_rows > n_cells)
    return fail(ATTN_ERR_INVALID_ARG, "the tree cells [prefix_cells, prefix_cells + n_rows) pass n_cells");
  DeviceInfo* di = nullptr;
  int32_t st = device_info(&di);
  if (st != ATTN_OK) return st;
  const cudaError_t e = launch_tree_mask(parent, n_rows, prefix_cells, n_cells, mask, mask_stride_row, di->status,
                                         static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(ATTN_ERR_CUDA, "tree mask launch: %s", cudaGetErrorString(e));
  return ATTN_OK;
}

int32_t attn_check_device_status(void* stream) {
  DeviceInfo* di = nullptr;
  int32_t st = device_info(&di);
  if (st != ATTN_OK) return st;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return fail(ATTN_ERR_CUDA, "stream synchronize failed");
  int word = 0;
  if (cudaMemcpy(&word, di->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return fail(ATTN_ERR_CUDA, "cannot read the device status word");
  if (word != 0) {
    const int zero = 0;
    cudaMemcpy(di->status, &zero, sizeof(int), cudaMemcpyHostToDevice);
    return fail(word, "a kernel reported %s", attn_strerror(word));
  }
  return ATTN_OK;
}

}  // extern "C"
