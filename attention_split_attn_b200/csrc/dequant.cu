// dequant.cu -- e4m3 / int8 K/V caches widened for the prefill tensor cores.
//
// TensorFold PR #911 ("--kv-cache fp8": its prefill kernel stages e4m3 rows
// widened to bf16) and TensorFold PR #2595 (an int8 cache with a K and a V
// scale per key) keep one F32 scale per (cell, KV head); a cache value is the
// code times its scale.  attn_prefill computes on those values: this kernel
// writes code * scale, rounded once to F16, into a contiguous
// [n_cells][n_head_kv][head_dim] copy of K and of V in the caller's
// workspace (and a BF16 Q into an F16 copy, since the tensor cores take both
// operands in one type), and the tensor-core prefill then runs on the copies
// as on any F16 cache.  F16 rather than BF16: one rounding of code * scale to
// BF16 alone moves the result by an NMSE near 7e-6 on N(0,1) data, F16 by
// about 1e-7.  The e4m3 NaN code stays NaN (so the prefill's non-finite-V
// handling applies unchanged); a value beyond F16's range becomes infinite.
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "quant.cuh"

namespace attn {
namespace {

constexpr int kDqThreads = 256;

template <typename OT>
__device__ __forceinline__ uint32_t dq_pack(float lo, float hi) {
  if constexpr (Storage<OT>::kDtype == ATTN_BF16) {
    __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&b);
  } else {
    __half2 b = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&b);
  }
}

// One thread per 16 codes of one (cell, KV head) row of K or V: a 16-byte
// load of codes, one scale, a 32-byte store.  blockIdx.y: 0 = K, 1 = V,
// 2 = the BF16 Q to F16 (8 values per thread).
template <typename CT, typename OT>
__global__ void __launch_bounds__(kDqThreads) dequant_kernel(const DequantPlan p) {
  const int which = blockIdx.y;
  if (which == 2) {
    const int per_vec = p.D / 8;
    const int64_t nq = (int64_t)p.R * p.Hq * per_vec;
    for (int64_t i = (int64_t)blockIdx.x * kDqThreads + threadIdx.x; i < nq; i += (int64_t)gridDim.x * kDqThreads) {
      const int64_t rh = i / per_vec;          // row * Hq + h
      const int chunk = (int)(i % per_vec);
      const int64_t r = rh / p.Hq;
      const int h = (int)(rh % p.Hq);
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.q) + r * p.q_sr +
                                                           (int64_t)h * p.q_sh) + chunk);
      float f[8];
      unpack_vec<__nv_bfloat16>(w, f);
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) o[e] = dq_pack<__half>(f[2 * e], f[2 * e + 1]);
      reinterpret_cast<uint4*>(static_cast<__half*>(p.q_out) + rh * p.D)[chunk] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    return;
  }
  const uint8_t* codes = static_cast<const uint8_t*>(which ? p.v : p.k);
  const float* scales = which ? p.v_scale : p.k_scale;
  OT* out = static_cast<OT*>(which ? p.v_out : p.k_out);
  const int per_row = p.D / 16;
  const int64_t n = (int64_t)p.N * p.Hkv * per_row;
  for (int64_t i = (int64_t)blockIdx.x * kDqThreads + threadIdx.x; i < n; i += (int64_t)gridDim.x * kDqThreads) {
    const int64_t row = i / per_row;          // cell * Hkv + g
    const int chunk = (int)(i % per_row);
    const int64_t c = row / p.Hkv;
    const int g = (int)(row % p.Hkv);
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(codes + c * p.sc + (int64_t)g * p.sh) + chunk);
    const float s = __ldg(scales + c * p.ss + g);
    float f[16];
    unpack_kv<CT>(w, f);
    uint32_t o[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = dq_pack<OT>(f[2 * e] * s, f[2 * e + 1] * s);
    uint4* dst = reinterpret_cast<uint4*>(out + row * p.D) + 2 * chunk;
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

template <typename CT, typename OT>
cudaError_t launch_dequant_t(const DequantPlan& p, int sms, cudaStream_t stream) {
  const int64_t n = std::max<int64_t>((int64_t)p.N * p.Hkv * (p.D / 16), p.q_out ? (int64_t)p.R * p.Hq * (p.D / 8) : 0);
  const int64_t want = (n + kDqThreads - 1) / kDqThreads;
  const unsigned blocks = (unsigned)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)sms * 8));
  dequant_kernel<CT, OT><<<dim3(blocks, p.q_out ? 3 : 2), kDqThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dequant(const DequantPlan& p, int sms, cudaStream_t stream) {
  if ((int64_t)p.N * p.Hkv == 0 && !p.q_out) return cudaSuccess;
  return p.code_type == ATTN_FP8_E4M3 ? launch_dequant_t<e4m3_code, __half>(p, sms, stream)
                                      : launch_dequant_t<i8_code, __half>(p, sms, stream);
}

}  // namespace attn
