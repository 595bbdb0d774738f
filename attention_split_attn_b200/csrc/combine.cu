// combine.cu -- split_k_reduce: fold the split partial records of every
// (row, q head) with the sink, in slot order.
//
// The pages' combine (TensorFold PR #2595: attn_decode writes fp32 partials,
// attn_merge folds them into bf16 rows; strix-llama.cpp PR #119:
// flash_attn_split_k_reduce after a row split) with HartsyInference PR #910's
// rules: a NaN in any record's max, or in the sink, gives NaN in every element
// (it must not turn into 0); a row whose max is -inf is +0; otherwise
//   M = max(m_s, sigma),  L = sum_s l_s e^(m_s - M) + e^(sigma - M),
//   out[d] = sum_s o_s[d] e^(m_s - M) / L,
// so a NaN in one record's o reaches that element even when its weight is 0.
//
// One warp per (row, q head).  Records are taken 32 at a time: lane j loads
// record j's (m, l) and computes its weight, then each lane folds its D/32
// output elements over the 32 records with eight vector loads in flight.
#include "common.cuh"
#include "internal.h"

namespace attn {

namespace {

// Warp whose run holds flattened tile t (runs are [T w / W, T (w + 1) / W)).
__device__ __forceinline__ int64_t warp_of_tile(int64_t t, int64_t T, int64_t W) {
  return ((t + 1) * W + T - 1) / T - 1;
}

struct SlotList {
  int64_t n;          // number of records
  int64_t first;      // slice scheme: first slot; balanced scheme: home slot
  int64_t w_first;    // balanced scheme: warp of the pair's first tile
  int64_t T, W;
  int mode;
  // k-th record of the list; -1 for a record that does not exist (an empty
  // warp run inside the pair, possible only when there are more warps than tiles)
  __device__ __forceinline__ int64_t slot(int64_t k) const {
    if (mode == 0) return first + k;
    if (k == 0) return first;
    const int64_t w = w_first + k;
    return (T * w / W < T * (w + 1) / W) ? w : -1;
  }
};

template <int D>
__global__ void __launch_bounds__(128) combine_kernel(const CombinePlan p) {
  constexpr int EPL = D / 32;                 // output elements per lane: 2, 4 or 8
  pdl_wait_prior_grid();
  const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= (int64_t)p.R * p.Hq) return;
  const int r = (int)(wid / p.Hq), h = (int)(wid % p.Hq);
  const int g = h / p.G, hh = h % p.G;

  SlotList sl;
  sl.mode = p.mode;
  sl.T = sl.W = 1;
  sl.w_first = 0;
  if (p.mode == 0) {
    int n_used;
    if (p.n_used) {
      n_used = min(__ldg(p.n_used + r), p.part.S);
    } else {
      int32_t b = p.row_begin ? __ldg(p.row_begin + r) : 0;
      int32_t e = p.row_end ? __ldg(p.row_end + r) : p.N;
      b = max(b, 0);
      e = min(e, p.N);
      const int64_t len = e > b ? (int64_t)e - b : 0;
      n_used = len == 0 ? 0 : (int)min((int64_t)p.part.S, (len + p.C - 1) / p.C);
    }
    sl.n = n_used;
    sl.first = ((int64_t)r * p.Hkv + g) * p.part.S;
  } else {
    const int64_t nt = p.row_tiles[r + 1] - p.row_tiles[r];
    sl.T = (int64_t)p.Hkv * p.row_tiles[p.R];
    sl.W = p.W;
    if (nt == 0) {
      sl.n = 0;
      sl.first = 0;
    } else {
      const int64_t start = (int64_t)p.Hkv * p.row_tiles[r] + g * nt;
      sl.w_first = warp_of_tile(start, sl.T, sl.W);
      const int64_t w_last = warp_of_tile(start + nt - 1, sl.T, sl.W);
      sl.n = w_last - sl.w_first + 1;
      sl.first = p.W + (int64_t)r * p.Hkv + g;
    }
  }

  const float sigma = p.sinks ? __ldg(p.sinks + h) : neg_inf();
  const float2* ml = reinterpret_cast<const float2*>(p.part.ml);
  // pass 1: the max
  float M = sigma;
  for (int64_t k0 = 0; k0 < sl.n; k0 += 32) {
    const int64_t s = k0 + lane < sl.n ? sl.slot(k0 + lane) : -1;
    if (s >= 0) M = fmax_nan(M, ml[s * p.G + hh].x);
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) M = fmax_nan(M, __shfl_xor_sync(0xffffffffu, M, off));
  const int64_t obase = (int64_t)r * p.out.sr + (int64_t)h * p.out.sh + lane * EPL;
  if (isnan(M) || M == neg_inf()) {
    const float val = isnan(M) ? qnan() : 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) store_from_float(p.out.out, obase + i, p.out.type, val);
    return;
  }
  // pass 2: weights, L, O -- in record order
  float L = 0.f;
  float O[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) O[i] = 0.f;
  for (int64_t k0 = 0; k0 < sl.n; k0 += 32) {
    const int64_t s_mine = k0 + lane < sl.n ? sl.slot(k0 + lane) : -1;
    float f = 0.f;
    if (s_mine >= 0) {
      const float2 x = ml[s_mine * p.G + hh];
      f = ex2((x.x - M) * kLog2e);
      L = fmaf(x.y, f, L);
    }
    const int cnt = (sl.n - k0) < 32 ? (int)(sl.n - k0) : 32;
    for (int j0 = 0; j0 < cnt; j0 += 8) {
      float v[8][EPL];
      int64_t sj[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        sj[j] = __shfl_sync(0xffffffffu, s_mine, (j0 + j) & 31);
        if (j0 + j < cnt && sj[j] >= 0) {
          const float* src = p.part.o + (sj[j] * p.G + hh) * D + lane * EPL;
#pragma unroll
          for (int i = 0; i < EPL; i += 2) {
            const float2 y = *reinterpret_cast<const float2*>(src + i);
            v[j][i] = y.x;
            v[j][i + 1] = y.y;
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float fj = __shfl_sync(0xffffffffu, f, (j0 + j) & 31);
        if (j0 + j < cnt && sj[j] >= 0) {
#pragma unroll
          for (int i = 0; i < EPL; ++i) O[i] = fmaf(v[j][i], fj, O[i]);
        }
      }
    }
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
  L += ex2((sigma - M) * kLog2e);
#pragma unroll
  for (int i = 0; i < EPL; ++i) store_from_float(p.out.out, obase + i, p.out.type, O[i] / L);
}

}  // namespace

cudaError_t launch_combine(const CombinePlan& p, cudaStream_t stream) {
  const int64_t warps = (int64_t)p.R * p.Hq;
  const int threads = 128;
  const int64_t blocks = (warps * 32 + threads - 1) / threads;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = p.use_pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  switch (p.D) {
    case 64: return cudaLaunchKernelEx(&cfg, combine_kernel<64>, p);
    case 128: return cudaLaunchKernelEx(&cfg, combine_kernel<128>, p);
    default: return cudaLaunchKernelEx(&cfg, combine_kernel<256>, p);
  }
}

}  // namespace attn
