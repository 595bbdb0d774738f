// quant.cuh -- the one-byte codes of quantized K/V caches (attn_decode with
// kv_type ATTN_FP8_E4M3 or ATTN_I8): element types for the kernel templates
// and their decoding to floats.  A cache value is the code times the scale
// of its (cell, KV head) (TensorFold PR #911: e4m3 rows with one fp32 scale
// per position and key head; TensorFold PR #2595: an int8 cache with K and V
// scales); the kernels apply the scales, these helpers only decode codes.
#pragma once

#include "common.cuh"

namespace attn {

struct e4m3_code { uint8_t bits; };
struct i8_code { int8_t bits; };
template <> struct Storage<e4m3_code> { static constexpr int kDtype = ATTN_FP8_E4M3; };
template <> struct Storage<i8_code> { static constexpr int kDtype = ATTN_I8; };

template <typename T>
constexpr bool is_code_type() {
  return Storage<T>::kDtype == ATTN_FP8_E4M3 || Storage<T>::kDtype == ATTN_I8;
}

// Two e4m3 codes (low byte first) to floats, by the hardware conversion to
// f16x2 (exact: every e4m3 value is an f16 value; S.1111.111 gives NaN).
__device__ __forceinline__ void unpack_e4m3x2(uint32_t two, float& lo, float& hi) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((unsigned short)(two & 0xffffu)));
  const float2 f = __half22float2(*reinterpret_cast<__half2*>(&h2));
  lo = f.x;
  hi = f.y;
}

// One 16-byte vector of cache elements to floats: 16 codes of a quantized
// cache, else the 4 or 8 values unpack_vec reads.
template <typename T>
__device__ __forceinline__ void unpack_kv(const uint4& w, float* f) {
  if constexpr (Storage<T>::kDtype == ATTN_FP8_E4M3) {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      unpack_e4m3x2(ws[k], f[4 * k], f[4 * k + 1]);
      unpack_e4m3x2(ws[k] >> 16, f[4 * k + 2], f[4 * k + 3]);
    }
  } else if constexpr (Storage<T>::kDtype == ATTN_I8) {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int b = 0; b < 4; ++b) f[4 * k + b] = (float)(int8_t)(ws[k] >> (8 * b));
  } else {
    unpack_vec<T>(w, f);
  }
}

}  // namespace attn
