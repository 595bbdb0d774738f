// decode_slice.cu -- split-K decode attention on a (rows, heads, slices) grid
// (attn_decode with a forced slice count, every FP32 or mixed-dtype cache, and
// the e4m3 / int8 caches with per (cell, KV head) scales).
//
// Work decomposition (TensorFold PR #2595, "What this changes": the
// attn_decode grid is (rows, heads, slices) so that rows sharing a key slice
// run back to back and share its K/V in L2; each work-group's arithmetic does
// not depend on the grid order, so outputs are bit-identical across orders).
// One CTA = one (row r, KV head g, slice s).  The slice is a run of cells of
// row r cut at multiples of 32 cells from row_begin[r] (32-key slices, same
// page); the CTA computes, for every query head of KV head g (GQA sharing),
// the online-softmax partial (m, l, o[D]) of its slice, and the combine
// (combine.cu) folds the partials of a row in slice order with the sink
// (attn_merge on the same page; flash_attn_split_k_reduce in strix-llama.cpp
// PR #119).  With one slice per row the CTA folds the sink itself and writes
// the row.
//
// Two kernels:
//  * decode_slice_kernel (any cache dtype, CUDA cores): one producer warp
//    streams 32-cell K and V tiles into a 4-stage ring with 3-D TMA loads on
//    mbarriers; four consumer warps (per group of up to 8 q heads) score keys
//    from shared memory with 16-byte vector reads, LPK lanes per key row and a
//    shuffle reduction of the dot product; each (warp, lane group) keeps its
//    own running (m, l, o) with one max per 32-cell tile (TensorFold PR #985,
//    "64-key softmax tiles"); the streams are merged in a fixed order.
//  * decode_warp_kernel (16-bit cache, Q in the cache dtype): a CTA is one
//    warp that streams 16-cell tiles of its slice through a 3-stage TMA ring
//    and folds them with tensor-core MMAs (decode_tile.cuh).
//
// Semantics (HartsyInference PR #910): the max propagates NaN; exp(-inf - -inf)
// is guarded (an all -inf stream uses 0 as its reference); excluded cells
// (outside the slice, other sequence, causal, mask == -inf) never contribute,
// not even through 0 * NaN, because their V vector is zeroed; visible cells
// always contribute p * v, so a NaN in a visible V reaches the output even
// when p underflows to 0.
#include "common.cuh"
#include "decode_tile.cuh"
#include "internal.h"
#include "mma.cuh"
#include "quant.cuh"

namespace attn {

namespace {

constexpr int kTileKeys = 32;   // cells per TMA tile (a multiple of the 32-cell slice grid)
constexpr int kKeyWarps = 4;    // consumer warps per head group

template <typename KT, int D>
struct DecodeGeom {
  static constexpr int ES = sizeof(KT);
  static constexpr int EPV = 16 / ES;                  // elements per 16-byte vector
  static constexpr int VPR = D / EPV;                  // vectors per key row
  static constexpr int LPK = VPR < 32 ? VPR : 32;      // lanes per key
  static constexpr int VPL = VPR / LPK;                // vectors per lane
  static constexpr int EPL = VPL * EPV;                // elements per lane
  static constexpr int KPI = 32 / LPK;                 // keys per warp step
  static constexpr int KPS = kTileKeys / (kKeyWarps * KPI);  // keys per stream per tile
  static constexpr int NST = kKeyWarps * KPI;          // streams per head group
  static constexpr int ROW_BYTES = D * ES;
  static constexpr int TILE_BYTES = kTileKeys * ROW_BYTES;
  static constexpr int NSTAGE = (2 * TILE_BYTES * 4 <= 65536) ? 4 : ((2 * TILE_BYTES * 3 <= 98304) ? 3 : 2);
  static_assert(KPS >= 1, "tile too small for the warp layout");
  static_assert(VPR % LPK == 0, "head_dim not a multiple of the lane layout");
};

template <typename KT, int D, int HPW, int HG>
struct DecodeSmem {
  using Geo = DecodeGeom<KT, D>;
  static constexpr int kStageBytes = 2 * Geo::TILE_BYTES;                 // K + V tile
  static constexpr int kRingBytes = Geo::NSTAGE * kStageBytes;
  static constexpr int kMergeO = HG * Geo::NST * HPW * D * 4;             // stream outputs
  static constexpr int kMergeML = HG * Geo::NST * HPW * 4 * 2;            // stream m, l
  static constexpr int kMergeBytes = kMergeO + kMergeML;
  static constexpr int kDataBytes = kRingBytes > kMergeBytes ? kRingBytes : kMergeBytes;
  static constexpr int kBarOffset = (kDataBytes + 127) / 128 * 128;
  static constexpr int kTotal = kBarOffset + 2 * Geo::NSTAGE * 8 + 16;
};

template <typename KT, int D, int HPW, int HG>
__global__ void __launch_bounds__(32 * (kKeyWarps * HG + 1))
decode_slice_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const DecodePlan p) {
  using Geo = DecodeGeom<KT, D>;
  using Sm = DecodeSmem<KT, D, HPW, HG>;
  constexpr int NCW = kKeyWarps * HG;
  constexpr bool kQuant = is_code_type<KT>();
  constexpr int NS = Geo::NSTAGE;
  extern __shared__ __align__(1024) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Sm::kBarOffset);
  uint64_t* empty = full + NS;
  int* abort_flag = reinterpret_cast<int*>(empty + NS);

  // ---- which unit ----------------------------------------------------------
  const int64_t bid = blockIdx.x;
  int r, g, s;
  if (p.grid_order == 0) {
    r = (int)(bid % p.R);
    g = (int)((bid / p.R) % p.Hkv);
    s = (int)(bid / ((int64_t)p.R * p.Hkv));
  } else {
    s = (int)(bid % p.S);
    g = (int)((bid / p.S) % p.Hkv);
    r = (int)(bid / ((int64_t)p.S * p.Hkv));
  }
  RowCtx rc;
  const int32_t raw_b = p.f.row_begin ? __ldg(p.f.row_begin + r) : 0;
  const int32_t raw_e = p.f.row_end ? __ldg(p.f.row_end + r) : p.N;
  rc.pos_base = raw_b;
  rc.begin = max(raw_b, 0);
  rc.end = min(raw_e, p.N);
  if (rc.end < rc.begin) rc.end = rc.begin;
  {
    const int64_t b = rc.begin, e = rc.end;
    const int64_t sb = b + (int64_t)s * p.C;
    const int64_t se = (s == p.S - 1) ? e : min(e, sb + p.C);
    rc.s_begin = (int32_t)min(sb, e);
    rc.s_end = (int32_t)max(min(se, e), (int64_t)rc.s_begin);
  }
  // An empty slice of a split row writes nothing: split_k_reduce reads only
  // the slices that hold cells.  With one slice the CTA must still write the
  // row (zeros or the sink's NaN).
  if (p.S > 1 && rc.s_begin >= rc.s_end) {
    pdl_launch_dependents();
    return;
  }
  rc.row_seq = p.f.row_seq ? __ldg(p.f.row_seq + r) : 0;
  rc.row_pos = p.f.row_pos ? (int64_t)__ldg(p.f.row_pos + r) : (int64_t)raw_e - raw_b - 1;
  const bool has_filter = (p.f.cell_seq && p.f.row_seq) || p.f.causal || p.f.mask;
  const int n_tiles = (rc.s_end - rc.s_begin + kTileKeys - 1) / kTileKeys;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], NCW);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();

  KT* ring = reinterpret_cast<KT*>(smem);
  constexpr int kStageElems = 2 * kTileKeys * D;   // K tile then V tile

  if (warp == NCW) {
    // ---------------- producer: TMA K/V tiles into the ring -----------------
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int issued = 0;
      for (int t = 0; t < n_tiles; ++t) {
        const int st = t % NS;
        if (t >= NS) {
          if (!mbar_wait_bounded(&empty[st], ((t / NS) & 1) ^ 1, p.status)) {
            atomicExch(abort_flag, 1);
            break;
          }
        }
        if (*(volatile int*)abort_flag) break;
        KT* sk = ring + st * kStageElems;
        KT* sv = sk + kTileKeys * D;
        mbar_arrive_expect_tx(&full[st], 2 * Geo::TILE_BYTES);
        const int c0 = rc.s_begin + t * kTileKeys;
        tma_load_3d(sk, &tmK, &full[st], 0, g, c0, pol);
        tma_load_3d(sv, &tmV, &full[st], 0, g, c0, pol);
        issued = t + 1;
      }
      // Never leave the CTA with copies in flight: wait (bounded) for every
      // issued tile the consumers may not have waited for.
      if (*(volatile int*)abort_flag) {
        for (int t = max(0, issued - NS); t < issued; ++t)
          mbar_wait_bounded(&full[t % NS], (t / NS) & 1, nullptr);
      }
    }
    return;
  }

  // ---------------- consumers ------------------------------------------------
  const int hg = warp / kKeyWarps;          // head group
  const int kw = warp % kKeyWarps;          // key warp within the group
  const int kg = lane / Geo::LPK;           // key lane-group within the warp
  const int dl = lane % Geo::LPK;           // lane within the key's row
  const int h_base = g * p.G + hg * HPW;    // first q head of this warp

  // q (scaled) for this lane's elements of each head
  float qf[HPW][Geo::EPL];
  float slope[HPW];
#pragma unroll
  for (int h = 0; h < HPW; ++h) {
    const bool hv = (hg * HPW + h) < p.G;
    const int hq = h_base + h;
    slope[h] = (hv && p.lg.slopes) ? __ldg(p.lg.slopes + hq) : 0.f;
#pragma unroll
    for (int v = 0; v < Geo::VPL; ++v)
#pragma unroll
      for (int e = 0; e < Geo::EPV; ++e) {
        const int d = (v * Geo::LPK + dl) * Geo::EPV + e;
        qf[h][v * Geo::EPV + e] =
            hv ? load_as_float(p.q.q, (int64_t)r * p.q.sr + (int64_t)hq * p.q.sh + d, p.q.type) * p.lg.scale
               : 0.f;
      }
  }

  float m[HPW], l[HPW], o[HPW][Geo::EPL];
#pragma unroll
  for (int h = 0; h < HPW; ++h) {
    m[h] = neg_inf();
    l[h] = 0.f;
#pragma unroll
    for (int e = 0; e < Geo::EPL; ++e) o[h][e] = 0.f;
  }
  const float softcap = p.lg.softcap;
  const bool alibi = p.lg.slopes != nullptr;

  for (int t = 0; t < n_tiles; ++t) {
    const int st = t % NS;
    if (!mbar_wait_bounded(&full[st], (t / NS) & 1, p.status)) {
      atomicExch(abort_flag, 1);
      break;
    }
    if (*(volatile int*)abort_flag) break;
    const KT* sk = ring + st * kStageElems;
    const KT* sv = sk + kTileKeys * D;
    const int tile0 = rc.s_begin + t * kTileKeys;

    float x[Geo::KPS][HPW];
    bool vis[Geo::KPS];
#pragma unroll
    for (int i = 0; i < Geo::KPS; ++i) {
      const int j = (i * kKeyWarps + kw) * Geo::KPI + kg;
      const int c = tile0 + j;
      bool vk = c < rc.s_end;
      float mval = 0.f;
      int64_t cpos = (int64_t)c - rc.pos_base;
      if (has_filter && vk) vk = cell_visible(p.f, rc, r, c, mval, cpos);
      else if (alibi && p.f.cell_pos && vk) cpos = __ldg(p.f.cell_pos + c);
      vis[i] = vk;
      float kf[Geo::EPL];
#pragma unroll
      for (int v = 0; v < Geo::VPL; ++v) {
        const uint4 w = *reinterpret_cast<const uint4*>(sk + j * D + (v * Geo::LPK + dl) * Geo::EPV);
        unpack_kv<KT>(w, kf + v * Geo::EPV);
      }
      float acc[HPW];
#pragma unroll
      for (int h = 0; h < HPW; ++h) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < Geo::EPL; ++e) a = fmaf(qf[h][e], kf[e], a);
        acc[h] = a;
      }
#pragma unroll
      for (int off = Geo::LPK / 2; off >= 1; off >>= 1)
#pragma unroll
        for (int h = 0; h < HPW; ++h) acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], off);
      const float negdist = -(float)(rc.row_pos >= cpos ? rc.row_pos - cpos : cpos - rc.row_pos);
      // quantized cache: q.(s_k code) = s_k (q.code), the dequantized dot product
      const float ks = kQuant ? (vk ? __ldg(p.k_scale + (int64_t)c * p.scale_sc + g) : 0.f) : 1.f;
#pragma unroll
      for (int h = 0; h < HPW; ++h) {
        float xv = kQuant ? acc[h] * ks : acc[h];
        if (softcap > 0.f) xv = softcap * tanhf(xv / softcap);
        if (alibi) xv = fmaf(slope[h], negdist, xv);
        xv += mval;
        x[i][h] = vk ? xv : neg_inf();
      }
    }
    // one running max per tile and stream
    float mu[HPW];
#pragma unroll
    for (int h = 0; h < HPW; ++h) {
      float mt = x[0][h];
#pragma unroll
      for (int i = 1; i < Geo::KPS; ++i) mt = fmax_nan(mt, x[i][h]);
      const float mn = fmax_nan(m[h], mt);
      mu[h] = (mn == neg_inf()) ? 0.f : mn;
      const float corr = ex2((m[h] - mu[h]) * kLog2e);
      l[h] *= corr;
#pragma unroll
      for (int e = 0; e < Geo::EPL; ++e) o[h][e] *= corr;
      m[h] = mn;
    }
#pragma unroll
    for (int i = 0; i < Geo::KPS; ++i) {
      const int j = (i * kKeyWarps + kw) * Geo::KPI + kg;
      float vf[Geo::EPL];
#pragma unroll
      for (int v = 0; v < Geo::VPL; ++v) {
        uint4 w = *reinterpret_cast<const uint4*>(sv + j * D + (v * Geo::LPK + dl) * Geo::EPV);
        if (!vis[i]) w = make_uint4(0u, 0u, 0u, 0u);
        unpack_kv<KT>(w, vf + v * Geo::EPV);
      }
      // quantized cache: p (s_v code) = (p s_v) code
      const float vs = kQuant ? (vis[i] ? __ldg(p.v_scale + (int64_t)(tile0 + j) * p.scale_sc + g) : 0.f) : 1.f;
#pragma unroll
      for (int h = 0; h < HPW; ++h) {
        const float pr = ex2((x[i][h] - mu[h]) * kLog2e);
        l[h] += pr;
        const float pv = kQuant ? pr * vs : pr;
#pragma unroll
        for (int e = 0; e < Geo::EPL; ++e) o[h][e] = fmaf(pv, vf[e], o[h][e]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }

  // ---------------- merge the streams of this CTA ----------------------------
  named_bar_sync(1, NCW * 32);          // every consumer is done with the ring
  float* sO = reinterpret_cast<float*>(smem);
  float* sM = sO + HG * Geo::NST * HPW * D;
  float* sL = sM + HG * Geo::NST * HPW;
  const int stream = kw * Geo::KPI + kg;
#pragma unroll
  for (int h = 0; h < HPW; ++h) {
    const int slot = (hg * Geo::NST + stream) * HPW + h;
#pragma unroll
    for (int v = 0; v < Geo::VPL; ++v)
#pragma unroll
      for (int e = 0; e < Geo::EPV; ++e)
        sO[slot * D + (v * Geo::LPK + dl) * Geo::EPV + e] = o[h][v * Geo::EPV + e];
    if (dl == 0) {
      sM[slot] = m[h];
      sL[slot] = l[h];
    }
  }
  named_bar_sync(1, NCW * 32);

  const bool aborted = *(volatile int*)abort_flag != 0;
  const int G = p.G;
  for (int idx = threadIdx.x; idx < G * D; idx += NCW * 32) {
    const int hh = idx / D, d = idx % D;     // hh: head within the KV group
    const int hgi = hh / HPW, h = hh % HPW;
    float M = neg_inf();
    for (int k = 0; k < Geo::NST; ++k) M = fmax_nan(M, sM[(hgi * Geo::NST + k) * HPW + h]);
    const float Mu = (M == neg_inf()) ? 0.f : M;
    float L = 0.f, O = 0.f;
    for (int k = 0; k < Geo::NST; ++k) {
      const int slot = (hgi * Geo::NST + k) * HPW + h;
      const float f = ex2((sM[slot] - Mu) * kLog2e);
      L = fmaf(sL[slot], f, L);
      O = fmaf(sO[slot * D + d], f, O);
    }
    if (aborted) { M = qnan(); L = qnan(); O = qnan(); }
    const int hq = g * G + hh;
    if (p.S == 1) {
      const float sigma = p.lg.sinks ? __ldg(p.lg.sinks + hq) : neg_inf();
      store_from_float(p.out.out, (int64_t)r * p.out.sr + (int64_t)hq * p.out.sh + d, p.out.type,
                       fold_with_sink(M, L, O, sigma));
    } else {
      const int64_t slot = (((int64_t)r * p.Hkv + g) * p.S + s) * G + hh;
      p.part.o[slot * D + d] = O;
      if (d == 0) {
        p.part.ml[slot * 2] = M;
        p.part.ml[slot * 2 + 1] = L;
      }
    }
  }
}

template <int D>
struct WarpRing {
  static constexpr int NS = (D <= 128) ? 3 : 2;      // ring stages
  static constexpr int BAR_OFF = NS * WarpStage<D>::BYTES;
  static constexpr int TOTAL = BAR_OFF + NS * 8 + 1024;   // + alignment slack for the swizzle
};

template <typename KT, int D, int NH>
__global__ void __launch_bounds__(32)
decode_warp_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   const DecodePlan p) {
  constexpr int NS = WarpRing<D>::NS;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + WarpRing<D>::BAR_OFF);
  const int lane = threadIdx.x;

  const int64_t bid = blockIdx.x;
  int r, g, s;
  if (p.grid_order == 0) {
    r = (int)(bid % p.R);
    g = (int)((bid / p.R) % p.Hkv);
    s = (int)(bid / ((int64_t)p.R * p.Hkv));
  } else {
    s = (int)(bid % p.S);
    g = (int)((bid / p.S) % p.Hkv);
    r = (int)(bid / ((int64_t)p.S * p.Hkv));
  }
  RowCtx rc;
  const int32_t raw_b = p.f.row_begin ? __ldg(p.f.row_begin + r) : 0;
  const int32_t raw_e = p.f.row_end ? __ldg(p.f.row_end + r) : p.N;
  rc.pos_base = raw_b;
  rc.begin = max(raw_b, 0);
  rc.end = min(raw_e, p.N);
  if (rc.end < rc.begin) rc.end = rc.begin;
  {
    const int64_t b = rc.begin, e = rc.end;
    const int64_t sb = b + (int64_t)s * p.C;
    const int64_t se = (s == p.S - 1) ? e : min(e, sb + p.C);
    rc.s_begin = (int32_t)min(sb, e);
    rc.s_end = (int32_t)max(min(se, e), (int64_t)rc.s_begin);
  }
  if (p.S > 1 && rc.s_begin >= rc.s_end) {
    pdl_launch_dependents();
    return;
  }
  rc.row_seq = p.f.row_seq ? __ldg(p.f.row_seq + r) : 0;
  rc.row_pos = p.f.row_pos ? (int64_t)__ldg(p.f.row_pos + r) : (int64_t)raw_e - raw_b - 1;
  const bool has_filter = (p.f.cell_seq && p.f.row_seq) || p.f.causal || p.f.mask;
  const int n_tiles = (rc.s_end - rc.s_begin + kWarpTile - 1) / kWarpTile;

  if (lane == 0) {
    for (int i = 0; i < NS; ++i) mbar_init(&full[i], 1);
    fence_mbar_init();
  }
  __syncwarp();
  pdl_launch_dependents();
  uint64_t pol = 0;
  if (lane == 0) {
    pol = policy_evict_first();
    for (int t = 0; t < min(NS, n_tiles); ++t)
      issue_warp_tile<D>(smem + t * WarpStage<D>::BYTES, &full[t], &tmK, &tmV, g, rc.s_begin + t * kWarpTile,
                         pol);
  }
  WarpTileState<KT, D, NH> st;
  st.reset();
  st.init_offsets(lane);
  st.load_q(p, r, g * p.G, lane);

  int consumed = 0;
  bool aborted = false;
  for (int t = 0; t < n_tiles; ++t) {
    const int stg = t % NS;
    if (!mbar_wait_bounded(&full[stg], (t / NS) & 1, p.status)) {
      aborted = true;
      break;
    }
    unsigned char* stage = smem + stg * WarpStage<D>::BYTES;
    st.load_tile(stage);
    consumed = t + 1;
    auto refill = [&]() {
      __syncwarp();
      if (lane == 0 && t + NS < n_tiles) {
        // the lanes' shared-memory reads of this stage precede its async refill
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        issue_warp_tile<D>(stage, &full[stg], &tmK, &tmV, g, rc.s_begin + (t + NS) * kWarpTile, pol);
      }
    };
    if (decltype(st)::kEarlyRelease) refill();
    st.compute(p, rc, r, rc.s_begin + t * kWarpTile, has_filter, lane, stage);
    if (!decltype(st)::kEarlyRelease) refill();
  }
  if (aborted) {
    // leave no copy in flight: wait (bounded) for every issued, unconsumed tile
    if (lane == 0)
      for (int t = consumed; t < min(n_tiles, consumed + NS); ++t)
        mbar_wait_bounded(&full[t % NS], (t / NS) & 1, nullptr);
    __syncwarp();
  }
  st.finish_sums();
  if (p.S == 1)
    st.write_final(p, r, g * p.G, lane, aborted);
  else
    st.write_partial(p.part.o, p.part.ml, ((int64_t)r * p.Hkv + g) * p.S + s, p.G, lane, aborted);
}

template <typename KT, int D, int HPW, int HG>
cudaError_t launch_decode_t(const DecodePlan& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                            cudaStream_t stream) {
  using Sm = DecodeSmem<KT, D, HPW, HG>;
  auto kern = decode_slice_kernel<KT, D, HPW, HG>;
  static std::atomic<unsigned long long> smem_set{0ull};
  cudaError_t e = set_smem_limit_once(smem_set, kern, Sm::kTotal);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (int64_t)p.R * p.Hkv * p.S;
  const int threads = 32 * (kKeyWarps * HG + 1);
  kern<<<dim3((unsigned)blocks), threads, Sm::kTotal, stream>>>(tmK, tmV, p);
  return cudaGetLastError();
}

template <typename KT, int D, int NH>
cudaError_t launch_decode_mma_t(const DecodePlan& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                                cudaStream_t stream) {
  auto kern = decode_warp_kernel<KT, D, NH>;
  static std::atomic<unsigned long long> smem_set{0ull};
  cudaError_t e = set_smem_limit_once(smem_set, kern, WarpRing<D>::TOTAL);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (int64_t)p.R * p.Hkv * p.S;
  kern<<<dim3((unsigned)blocks), 32, WarpRing<D>::TOTAL, stream>>>(tmK, tmV, p);
  return cudaGetLastError();
}

template <typename KT>
cudaError_t launch_decode_mma(const DecodePlan& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                              cudaStream_t stream) {
  const bool h16 = p.G > 8;
  switch (p.D) {
    case 64: return h16 ? launch_decode_mma_t<KT, 64, 16>(p, tmK, tmV, stream)
                        : launch_decode_mma_t<KT, 64, 8>(p, tmK, tmV, stream);
    case 128: return h16 ? launch_decode_mma_t<KT, 128, 16>(p, tmK, tmV, stream)
                         : launch_decode_mma_t<KT, 128, 8>(p, tmK, tmV, stream);
    default: return h16 ? launch_decode_mma_t<KT, 256, 16>(p, tmK, tmV, stream)
                        : launch_decode_mma_t<KT, 256, 8>(p, tmK, tmV, stream);
  }
}

template <typename KT, int D>
cudaError_t launch_decode_d(const DecodePlan& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                            cudaStream_t stream) {
  if (p.hg == 2) return launch_decode_t<KT, D, 8, 2>(p, tmK, tmV, stream);
  switch (p.hpw) {
    case 1: return launch_decode_t<KT, D, 1, 1>(p, tmK, tmV, stream);
    case 2: return launch_decode_t<KT, D, 2, 1>(p, tmK, tmV, stream);
    case 4: return launch_decode_t<KT, D, 4, 1>(p, tmK, tmV, stream);
    default: return launch_decode_t<KT, D, 8, 1>(p, tmK, tmV, stream);
  }
}

template <typename KT>
cudaError_t launch_decode_k(const DecodePlan& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                            cudaStream_t stream) {
  switch (p.D) {
    case 64: return launch_decode_d<KT, 64>(p, tmK, tmV, stream);
    case 128: return launch_decode_d<KT, 128>(p, tmK, tmV, stream);
    default: return launch_decode_d<KT, 256>(p, tmK, tmV, stream);
  }
}

}  // namespace

bool decode_uses_mma(int kv_type, int q_type, const void* q, int64_t q_sr, int64_t q_sh) {
  // Q must already be in the cache dtype (no extra rounding) and its pairs of
  // elements 4-byte aligned for the A-fragment loads.
  return (kv_type == ATTN_F16 || kv_type == ATTN_BF16) && q_type == kv_type &&
         (reinterpret_cast<uintptr_t>(q) & 3u) == 0 && (q_sr % 2) == 0 && (q_sh % 2) == 0;
}

bool decode_shape_supported(int kv_type, int D, int G) {
  return (kv_type == ATTN_F32 || kv_type == ATTN_F16 || kv_type == ATTN_BF16 || kv_type == ATTN_FP8_E4M3 ||
          kv_type == ATTN_I8) &&
         (D == 64 || D == 128 || D == 256) && G >= 1 && G <= 16;
}

cudaError_t launch_decode_slices(const DecodePlan& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                                 cudaStream_t stream) {
  if (p.mma) {
    if (p.kv_type == ATTN_F16) return launch_decode_mma<__half>(p, tmK, tmV, stream);
    return launch_decode_mma<__nv_bfloat16>(p, tmK, tmV, stream);
  }
  switch (p.kv_type) {
    case ATTN_F32: return launch_decode_k<float>(p, tmK, tmV, stream);
    case ATTN_F16: return launch_decode_k<__half>(p, tmK, tmV, stream);
    case ATTN_FP8_E4M3: return launch_decode_k<e4m3_code>(p, tmK, tmV, stream);
    case ATTN_I8: return launch_decode_k<i8_code>(p, tmK, tmV, stream);
    default: return launch_decode_k<__nv_bfloat16>(p, tmK, tmV, stream);
  }
}

}  // namespace attn
