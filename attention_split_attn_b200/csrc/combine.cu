// combine.cu -- split_k_reduce: fold the split partial records of every
// (row, q head) with the sink, in record order.
//
// The pages' combine (TensorFold PR #2595: attn_decode writes fp32 partials,
// attn_merge folds them into bf16 rows; strix-llama.cpp PR #119:
// flash_attn_split_k_reduce after a row split) with HartsyInference PR #910's
// rules: a NaN in any record's max, or in the sink, gives NaN in every element
// (it must not turn into 0); a row whose max is -inf is +0; NaN in one
// record's o reaches that element even when the record's weight is 0.
//
// One warp per (row, q head), one online pass over the records in order:
//   M' = max(M, m_k);  L = L e^(M - M') + l_k e^(m_k - M');
//   O = O e^(M - M') + o_k e^(m_k - M')        (per output element)
// then the sink: M_f = max(M, sigma), out = O e^(M - M_f) / (L e^(M - M_f) +
// e^(sigma - M_f)).  Each lane owns D/32 output elements; the records are read
// BATCH at a time with all their loads in flight, so a row with up to BATCH
// records costs one round trip to L2.
#include "common.cuh"
#include "decode_tile.cuh"
#include "internal.h"

namespace attn {

namespace {

// Warp whose run holds flattened tile t (runs are [T w / W, T (w + 1) / W)).
__device__ __forceinline__ int64_t warp_of_tile(int64_t t, int64_t T, int64_t W) {
  return ((t + 1) * W + T - 1) / T - 1;
}

// The records of one (row, KV head), in order.
//  mode 0 (slices): slots first .. first + n - 1.
//  mode 1 (balanced): the pair's home slot W + pair (from the warp in which
//  the pair starts), then the own slot of each later warp whose run starts
//  inside the pair: warps w_first + 1 .. w_last when T >= W (every run holds
//  a tile); when T < W every non-empty run holds one tile, so record k comes
//  from the warp of tile start + k.
struct SlotList {
  int64_t n, first, w_first, start, T, W;
  int mode;
  __device__ __forceinline__ int64_t slot(int64_t k) const {
    if (mode == 0) return first + k;
    if (k == 0) return first;
    return T >= W ? w_first + k : warp_of_tile(start + k, T, W);
  }
};

template <int D>
__global__ void __launch_bounds__(128) combine_kernel(const CombinePlan p) {
  constexpr int EPL = D / 32;                 // output elements per lane: 2, 4 or 8
  constexpr int BATCH = 8;                    // records in flight per round
  pdl_wait_prior_grid();
  const int64_t wid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= (int64_t)p.R * p.Hq) return;
  const int r = (int)(wid / p.Hq), h = (int)(wid % p.Hq);
  const int g = h / p.G, hh = h % p.G;

  SlotList sl;
  sl.mode = p.mode;
  sl.T = sl.W = 1;
  sl.w_first = sl.start = 0;
  if (p.mode == 0) {
    int n_used;
    if (p.n_used) {
      n_used = min(__ldg(p.n_used + r), p.part.S);
    } else if (p.row_len) {
      const int64_t len = max(__ldg(p.row_len + r), 0);
      n_used = len == 0 ? 0 : (int)min((int64_t)p.part.S, (len + p.C - 1) / p.C);
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
      sl.start = (int64_t)p.Hkv * p.row_tiles[r] + g * nt;
      sl.w_first = warp_of_tile(sl.start, sl.T, sl.W);
      sl.n = sl.T >= sl.W ? warp_of_tile(sl.start + nt - 1, sl.T, sl.W) - sl.w_first + 1 : nt;
      sl.first = p.W + (int64_t)r * p.Hkv + g;
    }
  }

  const float sigma = p.sinks ? __ldg(p.sinks + h) : neg_inf();
  const float2* ml = reinterpret_cast<const float2*>(p.part.ml);
  float M = neg_inf(), L = 0.f, O[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) O[i] = 0.f;
  for (int64_t k0 = 0; k0 < sl.n; k0 += BATCH) {
    float2 mlk[BATCH];
    float v[BATCH][EPL];
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      if (k0 + j < sl.n) {
        const int64_t rec = sl.slot(k0 + j) * p.G + hh;
        mlk[j] = ml[rec];
        const float* src = p.part.o + rec * D + lane * EPL;
#pragma unroll
        for (int i = 0; i < EPL; i += 2) {
          const float2 x = *reinterpret_cast<const float2*>(src + i);
          v[j][i] = x.x;
          v[j][i + 1] = x.y;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      if (k0 + j < sl.n) {
        const float mn = fmax_nan(M, mlk[j].x);
        const float mu = (mn == neg_inf()) ? 0.f : mn;
        const float c = ex2((M - mu) * kLog2e);
        const float f = ex2((mlk[j].x - mu) * kLog2e);
        L = fmaf(L, c, mlk[j].y * f);
#pragma unroll
        for (int i = 0; i < EPL; ++i) O[i] = fmaf(O[i], c, v[j][i] * f);
        M = mn;
      }
    }
  }
  const int64_t obase = (int64_t)r * p.out.sr + (int64_t)h * p.out.sh + lane * EPL;
#pragma unroll
  for (int i = 0; i < EPL; ++i) store_from_float(p.out.out, obase + i, p.out.type, fold_with_sink(M, L, O[i], sigma));
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
