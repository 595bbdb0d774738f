// selected.cu -- maskless selected-key attention (attn_selected).
//
// strix-llama.cpp PR #115 / #119 (FLASH_ATTN_EXT with a selection list src[5];
// flash_attn_sel.comp): a query row's visibility is exactly the cells named in
// its selection list; the list is sorted, invalid and duplicate entries are
// skipped (as the CPU path does), and K/V are gathered in blocks of 32 cells;
// with too few work-groups the rows are split into parts and
// flash_attn_split_k_reduce folds them.  Semantics of the logits, sinks, NaN
// and empty rows as everywhere else (HartsyInference PR #910).
//
// B200 design:
//  * select_compact_kernel: one CTA per row loads the list into shared memory,
//    replaces entries outside [0, n_cells) by a sentinel, bitonic-sorts it and
//    keeps each valid value once (flag + block scan).  The compacted list and
//    its length go to the workspace (and to the caller's optional outputs).
//  * selected_kernel: one CTA per (row, KV head, part).  A producer warp gathers
//    each 32-cell block with one cp.async.bulk per K row and per V row (the
//    cache row of a cell and head is D contiguous elements), completing on an
//    mbarrier.  Rows land D*2+16 bytes apart so eight rows read at one column
//    by ldmatrix fall in eight different bank groups.  The head dimension is
//    split over D/64 consumer warps: warp w computes the partial scores of
//    S^T = K Q^T over its 64 dimensions (m16n8k16, the q heads in N), the
//    warps add their partials through shared memory in a fixed order, every
//    warp then runs the same online softmax on the full scores, and warp w
//    accumulates O^T += V^T P^T for its 64 dimensions.  Each consumer warp
//    releases a stage as soon as it holds the block's fragments.
#include "common.cuh"
#include "decode_tile.cuh"
#include "internal.h"
#include "mma.cuh"

namespace attn {

namespace {

constexpr int kSelTile = 32;   // cells per gathered block
constexpr int kSortThreads = 1024;

// ---- a2: sort + dedup of the selection lists ---------------------------------
__global__ void __launch_bounds__(kSortThreads) select_compact_kernel(const SelectedPlan p) {
  extern __shared__ int32_t sbuf[];           // [n_pow2] keys, then [kSortThreads/32] scan
  const int r = blockIdx.x, tid = threadIdx.x;
  const int n = p.n_sel, np2 = p.n_pow2;
  const int32_t* list = p.sel + (int64_t)r * p.sel_stride;
  constexpr int32_t kSentinel = 0x7fffffff;
  for (int i = tid; i < np2; i += kSortThreads) {
    int32_t e = i < n ? __ldg(list + i) : kSentinel;
    sbuf[i] = (e >= 0 && e < p.N) ? e : kSentinel;
  }
  __syncthreads();
  // bitonic sort, ascending
  for (int k = 2; k <= np2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < np2; i += kSortThreads) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const int32_t a = sbuf[i], b = sbuf[ixj];
          const bool up = (i & k) == 0;
          if ((a > b) == up) {
            sbuf[i] = b;
            sbuf[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  // keep the first of each run of equal valid values; scan the flags in
  // chunks of kSortThreads
  int32_t* warp_tot = sbuf + np2;
  const int lane = tid & 31, wid = tid >> 5;
  int carry = 0;
  int32_t* out = p.compact + (int64_t)r * n;
  for (int base = 0; base < np2; base += kSortThreads) {
    const int i = base + tid;
    const int32_t v = i < np2 ? sbuf[i] : kSentinel;
    const int flag = (v != kSentinel && (i == 0 || sbuf[i - 1] != v)) ? 1 : 0;
    int x = flag;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) warp_tot[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int t = warp_tot[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, t, off);
        if (lane >= off) t += y;
      }
      warp_tot[lane] = t;
    }
    __syncthreads();
    const int pos = carry + x - flag + (wid > 0 ? warp_tot[wid - 1] : 0);
    if (flag) {
      out[pos] = v;
      if (p.sorted_out) p.sorted_out[(int64_t)r * n + pos] = v;
    }
    carry += warp_tot[31];
    __syncthreads();
  }
  if (tid == 0) {
    p.count[r] = carry;
    if (p.count_out) p.count_out[r] = carry;
  }
  if (p.sorted_out)
    for (int i = carry + tid; i < n; i += kSortThreads) p.sorted_out[(int64_t)r * n + i] = -1;
}

// ---- the attention kernel --------------------------------------------------------
template <typename KT, int D, int NH>
struct SelCfg {
  static constexpr int NW = D / 64;                   // consumer warps (64 dims each)
  static constexpr int NT = NH / 8;                   // head n-tiles
  static constexpr int RS = D * 2 + 16;               // shared-memory row stride (bytes)
  static constexpr int TILE_BYTES = kSelTile * RS;    // K or V block
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int NS = D == 256 ? 2 : 3;         // ring stages
  static constexpr int EXCH_FLOATS = NW * 32 * 8 * NT;   // partial S^T of every consumer warp
  static constexpr int EXCH_OFF = NS * STAGE_BYTES;
  static constexpr int BAR_OFF = EXCH_OFF + 2 * EXCH_FLOATS * 4;
  static constexpr int TOTAL = BAR_OFF + 2 * NS * 8 + 16;
  static constexpr int THREADS = 32 * (NW + 1);
};

template <typename KT, int D, int NH>
__global__ void __launch_bounds__(SelCfg<KT, D, NH>::THREADS)
selected_kernel(const SelectedPlan p) {
  using C = SelCfg<KT, D, NH>;
  using Op = MmaType<KT>;
  constexpr int NW = C::NW, NT = C::NT, NS = C::NS;
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty = full + NS;
  int* abort_flag = reinterpret_cast<int*>(empty + NS);
  float* exch = reinterpret_cast<float*>(smem + C::EXCH_OFF);

  const int64_t bid = blockIdx.x;
  const int r = (int)(bid % p.R);
  const int g = (int)((bid / p.R) % p.Hkv);
  const int part = (int)(bid / ((int64_t)p.R * p.Hkv));
  const int count = __ldg(p.count + r);
  const int c_begin = min(count, part * p.C);
  const int c_end = (part == p.S - 1) ? count : min(count, c_begin + p.C);
  if (p.S > 1 && c_begin >= c_end) {
    pdl_launch_dependents();
    return;
  }
  const int n_tiles = (c_end - c_begin + kSelTile - 1) / kSelTile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], NW);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_launch_dependents();
  const int32_t* cells = p.compact + (int64_t)r * p.n_sel;
  const KT* kbase = static_cast<const KT*>(p.k);
  const KT* vbase = static_cast<const KT*>(p.v);

  if (warp == NW) {
    // ---------------- producer: gather 32-cell blocks ----------------
    int issued = 0;
    for (int t = 0; t < n_tiles; ++t) {
      const int st = t % NS;
      if (t >= NS) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait_bounded(&empty[st], ((t / NS) & 1) ^ 1, p.status);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          if (lane == 0) atomicExch(abort_flag, 1);
          break;
        }
      }
      const int idx = c_begin + t * kSelTile + lane;
      const bool valid = idx < c_end;
      const int c = valid ? __ldg(cells + idx) : 0;
      const unsigned m = __ballot_sync(0xffffffffu, valid);
      unsigned char* sk = smem + st * C::STAGE_BYTES;
      if (lane == 0) mbar_arrive_expect_tx(&full[st], (uint32_t)__popc(m) * 2u * D * 2u);
      __syncwarp();
      if (valid) {
        const int64_t off = (int64_t)c * p.kv_sc + (int64_t)g * p.kv_sh;
        bulk_load(sk + lane * C::RS, kbase + off, D * 2, &full[st]);
        bulk_load(sk + C::TILE_BYTES + lane * C::RS, vbase + off, D * 2, &full[st]);
      }
      issued = t + 1;
    }
    if (lane == 0 && *(volatile int*)abort_flag)
      for (int t = max(0, issued - NS); t < issued; ++t) mbar_wait_bounded(&full[t % NS], (t / NS) & 1, nullptr);
    return;
  }

  // ---------------- consumers: warp w owns dims [64w, 64w + 64) ----------------
  const int grp = lane >> 2, tig = lane & 3;
  const int G = p.G, h0 = g * G;
  const int dw = warp * 64;
  uint32_t qb[4][NT][2];
  {
    const KT* qrow = static_cast<const KT*>(p.q) + (int64_t)r * p.q_sr;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int hh = nt * 8 + grp;
      const bool hv = hh < G;
      const KT* qh = qrow + (int64_t)(h0 + hh) * p.q_sh + dw;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        qb[kk][nt][0] = hv ? *reinterpret_cast<const uint32_t*>(qh + kk * 16 + 2 * tig) : 0u;
        qb[kk][nt][1] = hv ? *reinterpret_cast<const uint32_t*>(qh + kk * 16 + 8 + 2 * tig) : 0u;
      }
    }
  }
  const float scale = p.lg.scale, softcap = p.lg.softcap;
  const bool alibi = p.lg.slopes != nullptr;
  float slope[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int hh = nt * 8 + 2 * tig + e;
      slope[nt][e] = (alibi && hh < G) ? __ldg(p.lg.slopes + h0 + hh) : 0.f;
    }
  const int64_t row_pos = p.row_pos ? (int64_t)__ldg(p.row_pos + r) : (int64_t)p.N - 1;

  // ldmatrix byte offsets inside a stage
  uint32_t koff[2][4], voff[4][2];
  {
    const int mi = lane >> 3;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int row = mt * 16 + (lane & 7) + (mi & 1) * 8;
        const int chunk = (dw >> 3) + 2 * kk + (mi >> 1);
        koff[mt][kk] = row * C::RS + chunk * 16;
      }
#pragma unroll
    for (int m4 = 0; m4 < 4; ++m4)
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
        const int row = ks * 16 + (lane & 7) + (mi >> 1) * 8;
        const int chunk = (dw >> 3) + 2 * m4 + (mi & 1);
        voff[m4][ks] = C::TILE_BYTES + row * C::RS + chunk * 16;
      }
  }

  float acc[4][NT][4];
#pragma unroll
  for (int m4 = 0; m4 < 4; ++m4)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[m4][nt][0] = acc[m4][nt][1] = acc[m4][nt][2] = acc[m4][nt][3] = 0.f;
  float m[NT][2], l[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) m[nt][0] = m[nt][1] = neg_inf(), l[nt][0] = l[nt][1] = 0.f;
  bool aborted = false;

  for (int t = 0; t < n_tiles; ++t) {
    const int st = t % NS;
    // Every consumer warp takes part in the exchange barrier below, so after a
    // timeout (here or in another warp) a warp stops waiting but keeps looping
    // on whatever the stage holds; its output is poisoned at the end.
    if (!aborted && *(volatile int*)abort_flag) aborted = true;
    if (!aborted && !mbar_wait_bounded(&full[st], (t / NS) & 1, p.status)) {
      atomicExch(abort_flag, 1);
      aborted = true;
    }
    __syncwarp();
    const uint32_t sbase = smem_u32(smem + st * C::STAGE_BYTES);
    uint32_t ka[2][4][4], va[4][2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        ldsm_x4(ka[mt][kk][0], ka[mt][kk][1], ka[mt][kk][2], ka[mt][kk][3], sbase + koff[mt][kk]);
#pragma unroll
    for (int m4 = 0; m4 < 4; ++m4)
#pragma unroll
      for (int ks = 0; ks < 2; ++ks)
        ldsm_x4_trans(va[m4][ks][0], va[m4][ks][1], va[m4][ks][2], va[m4][ks][3], sbase + voff[m4][ks]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);

    // partial S^T over this warp's dims: [2 m-tiles of 16 cells][NT][4]
    float sc[2][NT][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) sc[mt][nt][0] = sc[mt][nt][1] = sc[mt][nt][2] = sc[mt][nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) Op::mma(sc[mt][nt], ka[mt][kk], qb[kk][nt][0], qb[kk][nt][1]);
    if (NW > 1) {
      // add the partials of all warps, in warp order
      float* buf = exch + (t & 1) * C::EXCH_FLOATS;
      float4* mine = reinterpret_cast<float4*>(buf + (warp * 32 + lane) * 8 * NT);
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mine[mt * NT + nt] = make_float4(sc[mt][nt][0], sc[mt][nt][1], sc[mt][nt][2], sc[mt][nt][3]);
      named_bar_sync(1, NW * 32);
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float4 s = reinterpret_cast<const float4*>(buf + lane * 8 * NT)[mt * NT + nt];
#pragma unroll
          for (int w = 1; w < NW; ++w) {
            const float4 x = reinterpret_cast<const float4*>(buf + (w * 32 + lane) * 8 * NT)[mt * NT + nt];
            s.x += x.x; s.y += x.y; s.z += x.z; s.w += x.w;
          }
          sc[mt][nt][0] = s.x; sc[mt][nt][1] = s.y; sc[mt][nt][2] = s.z; sc[mt][nt][3] = s.w;
        }
    }

    // logits: this lane's cells are 16*mt + grp + 8*kr
    const int tile0 = c_begin + t * kSelTile;
    bool vis[2][2];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int kr = 0; kr < 2; ++kr) {
        const int idx = tile0 + mt * 16 + grp + 8 * kr;
        const bool vk = idx < c_end;
        vis[mt][kr] = vk;
        float negdist = 0.f;
        if (alibi && vk) {
          const int c = __ldg(cells + idx);
          const int64_t cpos = p.cell_pos ? (int64_t)__ldg(p.cell_pos + c) : (int64_t)c;
          negdist = -(float)(row_pos >= cpos ? row_pos - cpos : cpos - row_pos);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            float x = sc[mt][nt][2 * kr + e] * scale;
            if (softcap > 0.f) x = softcap * tanhf(x / softcap);
            if (alibi) x = fmaf(slope[nt][e], negdist, x);
            sc[mt][nt][2 * kr + e] = vk ? x : neg_inf();
          }
      }

    // online softmax per head (a column of S^T), one max per block
    float corr[NT][2];
    bool changed = false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float mt_ = fmax_nan(fmax_nan(sc[0][nt][e], sc[0][nt][2 + e]), fmax_nan(sc[1][nt][e], sc[1][nt][2 + e]));
        mt_ = fmax_nan(mt_, __shfl_xor_sync(0xffffffffu, mt_, 4));
        mt_ = fmax_nan(mt_, __shfl_xor_sync(0xffffffffu, mt_, 8));
        mt_ = fmax_nan(mt_, __shfl_xor_sync(0xffffffffu, mt_, 16));
        const float mo = m[nt][e];
        const float mn = fmax_nan(mo, mt_);
        const float mu = (mn == neg_inf()) ? 0.f : mn;
        corr[nt][e] = ex2((mo - mu) * kLog2e);
        changed |= !(mo == mn);
        m[nt][e] = mn;
        float lsum = 0.f;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const float p0 = ex2((sc[mt][nt][e] - mu) * kLog2e);
          const float p1 = ex2((sc[mt][nt][2 + e] - mu) * kLog2e);
          sc[mt][nt][e] = p0;
          sc[mt][nt][2 + e] = p1;
          lsum += p0 + p1;
        }
        l[nt][e] = fmaf(l[nt][e], corr[nt][e], lsum);
      }
    if (__any_sync(0xffffffffu, changed)) {
#pragma unroll
      for (int m4 = 0; m4 < 4; ++m4)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          acc[m4][nt][0] *= corr[nt][0];
          acc[m4][nt][1] *= corr[nt][1];
          acc[m4][nt][2] *= corr[nt][0];
          acc[m4][nt][3] *= corr[nt][1];
        }
    }
    // cells past the end of the list: clear their V values (their rows in the
    // stage are stale); this lane's V^T registers 0,1 hold cells 16ks+2tig,+1
    // and registers 2,3 cells 16ks+8+2tig,+1
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      const unsigned lo = __ballot_sync(0xffffffffu, vis[ks][0]);
      const unsigned hi = __ballot_sync(0xffffffffu, vis[ks][1]);
      if ((lo & hi & 0x11111111u) != 0x11111111u) {
        auto bit = [](unsigned mm, int cell) { return (mm >> (4 * cell)) & 1u; };
        const uint32_t m01 = (bit(lo, 2 * tig) ? 0x0000ffffu : 0u) | (bit(lo, 2 * tig + 1) ? 0xffff0000u : 0u);
        const uint32_t m23 = (bit(hi, 2 * tig) ? 0x0000ffffu : 0u) | (bit(hi, 2 * tig + 1) ? 0xffff0000u : 0u);
#pragma unroll
        for (int m4 = 0; m4 < 4; ++m4) {
          va[m4][ks][0] &= m01;
          va[m4][ks][1] &= m01;
          va[m4][ks][2] &= m23;
          va[m4][ks][3] &= m23;
        }
      }
    }
    // O^T += V^T P^T over this warp's dims
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      uint32_t pb[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        pb[nt][0] = movm_trans(Op::pack(sc[ks][nt][0], sc[ks][nt][1]));
        pb[nt][1] = movm_trans(Op::pack(sc[ks][nt][2], sc[ks][nt][3]));
      }
#pragma unroll
      for (int m4 = 0; m4 < 4; ++m4)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) Op::mma(acc[m4][nt], va[m4][ks], pb[nt][0], pb[nt][1]);
    }
  }

  // ---------------- epilogue ----------------
  aborted = aborted || (*(volatile int*)abort_flag != 0);
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float v = l[nt][e];
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      l[nt][e] = v;
    }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int hh = nt * 8 + 2 * tig + e;
      if (hh >= G) continue;
      const int hq = h0 + hh;
      if (p.S == 1) {
        const float sigma = p.lg.sinks ? __ldg(p.lg.sinks + hq) : neg_inf();
        const int64_t ob = (int64_t)r * p.out.sr + (int64_t)hq * p.out.sh;
#pragma unroll
        for (int m4 = 0; m4 < 4; ++m4)
#pragma unroll
          for (int dr = 0; dr < 2; ++dr) {
            const int d = dw + m4 * 16 + grp + 8 * dr;
            const float v = aborted ? qnan() : fold_with_sink(m[nt][e], l[nt][e], acc[m4][nt][2 * dr + e], sigma);
            store_from_float(p.out.out, ob + d, p.out.type, v);
          }
      } else {
        const int64_t rec = (((int64_t)r * p.Hkv + g) * p.S + part) * G + hh;
        float* o = p.part.o + rec * D;
#pragma unroll
        for (int m4 = 0; m4 < 4; ++m4)
#pragma unroll
          for (int dr = 0; dr < 2; ++dr)
            o[dw + m4 * 16 + grp + 8 * dr] = aborted ? qnan() : acc[m4][nt][2 * dr + e];
        if (warp == 0 && grp == 0) {
          p.part.ml[rec * 2] = aborted ? qnan() : m[nt][e];
          p.part.ml[rec * 2 + 1] = aborted ? qnan() : l[nt][e];
        }
      }
    }
}

template <typename KT, int D, int NH>
cudaError_t launch_selected_t(const SelectedPlan& p, cudaStream_t stream) {
  using C = SelCfg<KT, D, NH>;
  auto kern = selected_kernel<KT, D, NH>;
  static std::atomic<unsigned long long> smem_set{0ull};
  cudaError_t e = set_smem_limit_once(smem_set, kern, C::TOTAL);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (int64_t)p.R * p.Hkv * p.S;
  kern<<<dim3((unsigned)blocks), C::THREADS, C::TOTAL, stream>>>(p);
  return cudaGetLastError();
}

template <typename KT>
cudaError_t launch_selected_k(const SelectedPlan& p, cudaStream_t stream) {
  const bool h16 = p.G > 8;
  switch (p.D) {
    case 64: return h16 ? launch_selected_t<KT, 64, 16>(p, stream) : launch_selected_t<KT, 64, 8>(p, stream);
    case 128: return h16 ? launch_selected_t<KT, 128, 16>(p, stream) : launch_selected_t<KT, 128, 8>(p, stream);
    default: return h16 ? launch_selected_t<KT, 256, 16>(p, stream) : launch_selected_t<KT, 256, 8>(p, stream);
  }
}

}  // namespace

int selected_pow2(int n_sel) {
  int np2 = 1;
  while (np2 < n_sel) np2 <<= 1;
  return np2;
}

cudaError_t launch_select_compact(const SelectedPlan& p, cudaStream_t stream) {
  // at most 4096 keys + the scan scratch: 16.5 KB, under the default limit
  const size_t smem = ((size_t)p.n_pow2 + kSortThreads / 32) * sizeof(int32_t);
  select_compact_kernel<<<dim3((unsigned)p.R), kSortThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_selected(const SelectedPlan& p, cudaStream_t stream) {
  if (p.kv_type == ATTN_F16) return launch_selected_k<__half>(p, stream);
  return launch_selected_k<__nv_bfloat16>(p, stream);
}

}  // namespace attn
