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
//  * compaction, one CTA per row: for caches up to 256K cells a bitmap in
//    shared memory (set a bit per valid entry, read the bits back in order
//    with a popcount prefix scan); above that a bitonic sort of the list with
//    invalid entries turned into a sentinel, keeping the first of each run.
//    The compacted list and its length go to the workspace (and to the
//    caller's optional outputs).
//  * selected_kernel: one CTA per (row, KV head, part) with D/64 warps; warp w
//    owns head dims [64w, 64w + 64).  Each warp gathers its column slice of
//    every 32-cell block itself with 16-byte cp.async copies (rows past the
//    list end zero-filled) into its own ring -- per-thread copies gather rows
//    that mostly sit in L2 much faster than one bulk copy per row -- with rows
//    144 bytes apart so ldmatrix reads are free of bank conflicts.  The warp
//    computes the partial scores of S^T = K Q^T over its 64 dimensions
//    (m16n8k16, the q heads in N), the warps add their partials through shared
//    memory in a fixed order, every warp then runs the same online softmax on
//    the full scores, and warp w accumulates O^T += V^T P^T for its dims.
//    A warp refills a stage as soon as it holds the block's fragments.
#include "common.cuh"
#include "decode_tile.cuh"
#include "internal.h"
#include "mma.cuh"

namespace attn {

namespace {

constexpr int kSelTile = 32;   // cells per gathered block
constexpr int kSortThreads = 1024;

// ---- a2: sort + dedup of the selection lists ---------------------------------
// For caches of at most kBitmapCells cells: one bit per cell in shared memory.
// Setting the bit of every valid entry drops duplicates; reading the bits in
// cell order (a popcount prefix over the words gives each bit its position)
// yields the distinct valid entries in ascending order -- the same list the
// sort-and-unique below produces, in O(n_sel + n_cells / 32).
constexpr int kBitmapCells = 256 * 1024;

__global__ void __launch_bounds__(kSortThreads) select_bitmap_kernel(const SelectedPlan p) {
  extern __shared__ uint32_t bits[];          // [ceil(N / 32)] words, then [32] scan scratch
  const int r = blockIdx.x, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int n = p.n_sel;
  const int nw = (p.N + 31) / 32;
  uint32_t* warp_tot = bits + nw;
  for (int i = tid; i < nw; i += kSortThreads) bits[i] = 0u;
  __syncthreads();
  const int32_t* list = p.sel + (int64_t)r * p.sel_stride;
  for (int i = tid; i < n; i += kSortThreads) {
    const int32_t e = __ldg(list + i);
    if (e >= 0 && e < p.N) atomicOr(&bits[e >> 5], 1u << (e & 31));
  }
  __syncthreads();
  int32_t* out = p.compact + (int64_t)r * n;
  int carry = 0;
  for (int base = 0; base < nw; base += kSortThreads) {
    const int i = base + tid;
    uint32_t w = i < nw ? bits[i] : 0u;
    const int cnt = __popc(w);
    int x = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) warp_tot[wid] = (uint32_t)x;
    __syncthreads();
    if (wid == 0) {
      int t = (int)warp_tot[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, t, off);
        if (lane >= off) t += y;
      }
      warp_tot[lane] = (uint32_t)t;
    }
    __syncthreads();
    int pos = carry + x - cnt + (wid > 0 ? (int)warp_tot[wid - 1] : 0);
    while (w) {
      const int b = __ffs(w) - 1;
      w &= w - 1;
      const int32_t v = i * 32 + b;
      out[pos] = v;
      if (p.sorted_out) p.sorted_out[(int64_t)r * n + pos] = v;
      ++pos;
    }
    carry += (int)warp_tot[31];
    __syncthreads();
  }
  if (tid == 0) {
    p.count[r] = carry;
    if (p.count_out) p.count_out[r] = carry;
  }
  if (p.sorted_out)
    for (int i = carry + tid; i < n; i += kSortThreads) p.sorted_out[(int64_t)r * n + i] = -1;
}

// Larger caches: bitonic sort of the list in shared memory, then keep the
// first of each run of equal valid values.
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
// Warp w owns head dims [64w, 64w + 64) and gathers exactly that slice of each
// 32-cell block's K and V rows itself: 16-byte cp.async copies (L2 only; per-
// thread copies gather L2-resident rows far faster than one bulk copy per
// row) into the warp's own ring, rows past the end of the list zero-filled.
// The warps meet only to add their partial scores.
template <typename KT, int D, int NH>
struct SelCfg {
  static constexpr int NW = D / 64;                   // warps (64 dims each)
  static constexpr int NT = NH / 8;                   // head n-tiles
  // A warp's slice of a cell row is 128 bytes; rows are stored unpadded with
  // 16-byte chunk k of row i at chunk k ^ (i & 7), so the 8 lanes copying one
  // row and the 8 rows one ldmatrix reads both cover all 32 banks.
  static constexpr int RS = 64 * 2;                   // row stride of a warp's slice (bytes)
  static constexpr int TILE_BYTES = kSelTile * RS;    // K or V slice of a block
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int NS = NW == 4 ? 2 : 3;          // ring stages per warp
  static constexpr int RING_BYTES = NS * STAGE_BYTES;
  static constexpr int EXCH_FLOATS = NW * 32 * 8 * NT;   // partial S^T of every warp
  static constexpr int EXCH_OFF = NW * RING_BYTES;
  static constexpr int TOTAL = EXCH_OFF + EXCH_FLOATS * 4;
  static constexpr int THREADS = 32 * NW;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// BIAS: add the F32 mask bias of each listed cell (unified-cache route only).
template <typename KT, int D, int NH, bool BIAS>
__global__ void __launch_bounds__(SelCfg<KT, D, NH>::THREADS)
selected_kernel(const SelectedPlan p) {
  using C = SelCfg<KT, D, NH>;
  using Op = MmaType<KT>;
  constexpr int NW = C::NW, NT = C::NT, NS = C::NS;
  extern __shared__ __align__(128) unsigned char smem[];
  float* exch = reinterpret_cast<float*>(smem + C::EXCH_OFF);

  const int64_t bid = blockIdx.x;
  const int r = (int)(bid % p.R);
  const int g = (int)((bid / p.R) % p.Hkv);
  const int part = (int)(bid / ((int64_t)p.R * p.Hkv));
  const int count = __ldg(p.count + r);
  const int c_begin = min(count, part * p.C);
  const int c_end = (part == p.S - 1) ? count : min(count, c_begin + p.C);
  pdl_launch_dependents();
  if (p.S > 1 && c_begin >= c_end) return;
  const int n_tiles = (c_end - c_begin + kSelTile - 1) / kSelTile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t* cells = p.compact + (int64_t)r * p.n_sel;
  const KT* kbase = static_cast<const KT*>(p.k);
  const KT* vbase = static_cast<const KT*>(p.v);
  const int dw = warp * 64;
  const uint32_t ring = smem_u32(smem + warp * C::RING_BYTES);

  // block t's cell of this lane's row (-1 past the end of the list)
  auto block_cell = [&](int t) {
    const int idx = c_begin + t * kSelTile + lane;
    return (t < n_tiles && idx < c_end) ? __ldg(cells + idx) : -1;
  };
  // gather this warp's slice of block t into stage t % NS: lane l copies
  // 16-byte chunk l % 8 of rows l / 8 + 4 i; one commit group per block
  auto issue = [&](int t, int cl) {
    if (t < n_tiles) {
      const uint32_t st = ring + (t % NS) * C::STAGE_BYTES;
      const int chunk = lane & 7;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int row = (lane >> 3) + 4 * i;
        const int c = __shfl_sync(0xffffffffu, cl, row);
        const bool valid = c >= 0;
        const int64_t off = (int64_t)(valid ? c : 0) * p.kv_sc + (int64_t)g * p.kv_sh + dw + chunk * 8;
        const uint32_t so = (uint32_t)(row * C::RS + ((chunk ^ (row & 7)) << 4));
        cp_async16(st + so, kbase + off, valid);
        cp_async16(st + C::TILE_BYTES + so, vbase + off, valid);
      }
    }
    cp_async_commit();
  };
#pragma unroll
  for (int t = 0; t < NS; ++t) issue(t, block_cell(t));

  const int grp = lane >> 2, tig = lane & 3;
  const int G = p.G, h0 = g * G;
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
        const int chunk = 2 * kk + (mi >> 1);
        koff[mt][kk] = row * C::RS + ((chunk ^ (row & 7)) << 4);
      }
#pragma unroll
    for (int m4 = 0; m4 < 4; ++m4)
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
        const int row = ks * 16 + (lane & 7) + (mi >> 1) * 8;
        const int chunk = 2 * m4 + (mi & 1);
        voff[m4][ks] = C::TILE_BYTES + row * C::RS + ((chunk ^ (row & 7)) << 4);
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
  for (int t = 0; t < n_tiles; ++t) {
    const int st = t % NS;
    const int cl_next = block_cell(t + NS);   // indices of the block to gather next
    cp_async_wait<NS - 1>();                  // this lane's copies of block t are done
    __syncwarp();                             // ... and every other lane's
    const uint32_t sbase = ring + st * C::STAGE_BYTES;
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
    __syncwarp();                             // every lane holds block t: refill its stage
    issue(t + NS, cl_next);

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
      // add the partials of all warps, in warp order; layout [warp][fragment
      // index][lane] so a warp's float4 stores and loads are contiguous
      float4* buf = reinterpret_cast<float4*>(exch);
      named_bar_sync(1, NW * 32);   // every warp has read the previous block's sums
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          buf[(warp * 2 * NT + mt * NT + nt) * 32 + lane] =
              make_float4(sc[mt][nt][0], sc[mt][nt][1], sc[mt][nt][2], sc[mt][nt][3]);
      named_bar_sync(1, NW * 32);
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float4 s = buf[(mt * NT + nt) * 32 + lane];
#pragma unroll
          for (int w = 1; w < NW; ++w) {
            const float4 x = buf[(w * 2 * NT + mt * NT + nt) * 32 + lane];
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
        float negdist = 0.f, bias = 0.f;
        if ((alibi || BIAS) && vk) {
          const int c = __ldg(cells + idx);
          if (alibi) {
            const int64_t cpos = p.cell_pos ? (int64_t)__ldg(p.cell_pos + c) : (int64_t)c;
            negdist = -(float)(row_pos >= cpos ? row_pos - cpos : cpos - row_pos);
          }
          if (BIAS) bias = __ldg(p.mask + (int64_t)r * p.mask_sr + c);   // F32, added unnarrowed
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            float x = sc[mt][nt][2 * kr + e] * scale;
            if (softcap > 0.f) x = softcap * tanhf(x / softcap);
            if (alibi) x = fmaf(slope[nt][e], negdist, x);
            if (BIAS) x += bias;
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
  cp_async_wait<0>();                         // no copy is left in flight at exit
  constexpr bool aborted = false;             // (no barrier waits in this kernel)
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
  auto kern = p.mask ? selected_kernel<KT, D, NH, true> : selected_kernel<KT, D, NH, false>;
  static std::atomic<unsigned long long> smem_set{0ull}, smem_set_b{0ull};
  cudaError_t e = set_smem_limit_once(p.mask ? smem_set_b : smem_set, kern, C::TOTAL);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (int64_t)p.R * p.Hkv * p.S;
  kern<<<dim3((unsigned)blocks), C::THREADS, C::TOTAL, stream>>>(p);
  return cudaGetLastError();
}

// ---- unified-cache route: the visible cells of each row, in order ------------
// One CTA of 1024 threads per row.  Each round covers 4096 cells as four
// 1024-cell sub-chunks: the loads of all four go out first, then each
// sub-chunk is compacted in order (warp ballots, a prefix over the 32 warp
// counts in shared memory).
constexpr int kVisThreads = 1024;

__global__ void __launch_bounds__(kVisThreads) visible_list_kernel(const SelectedPlan p, const RowFilter f) {
  __shared__ int wcount[32];
  __shared__ int base_sh;
  const int r = blockIdx.x, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  // positions default from the range as given; the scan covers its part inside [0, n_cells)
  const int32_t raw_b = f.row_begin ? __ldg(f.row_begin + r) : 0;
  const int32_t raw_e = f.row_end ? __ldg(f.row_end + r) : p.N;
  const int32_t rb = max(raw_b, 0);
  const int32_t re = min(raw_e, p.N);
  const int32_t rs = f.row_seq ? __ldg(f.row_seq + r) : 0;
  const int64_t rp = f.row_pos ? (int64_t)__ldg(f.row_pos + r) : (int64_t)raw_e - raw_b - 1;
  const float* mrow = f.mask ? f.mask + (int64_t)r * f.mask_sr : nullptr;
  int32_t* out = p.compact + (int64_t)r * p.n_sel;
  if (tid == 0) base_sh = 0;
  __syncthreads();
  for (int64_t c0 = rb; c0 < re; c0 += 4 * kVisThreads) {
    bool vis[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int64_t c = c0 + k * kVisThreads + tid;
      bool v = c < re;
      if (v && f.cell_seq) v = __ldg(f.cell_seq + c) == rs;
      if (v && f.causal) {
        const int64_t cp = f.cell_pos ? (int64_t)__ldg(f.cell_pos + c) : c - raw_b;
        v = cp <= rp;
      }
      if (v && mrow) v = !(__ldg(mrow + c) == neg_inf());
      vis[k] = v;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const unsigned bal = __ballot_sync(0xffffffffu, vis[k]);
      if (lane == 0) wcount[wid] = __popc(bal);
      __syncthreads();
      if (wid == 0) {
        const int x = wcount[lane];
        int incl = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        wcount[lane] = incl - x;   // exclusive prefix of the warp counts
      }
      __syncthreads();
      const int base = base_sh;
      if (vis[k]) out[base + wcount[wid] + __popc(bal & ((1u << lane) - 1u))] = (int32_t)(c0 + k * kVisThreads + tid);
      __syncthreads();
      if (tid == kVisThreads - 1) base_sh = base + wcount[31] + __popc(bal);
      __syncthreads();
    }
  }
  if (tid == 0) p.count[r] = base_sh;
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
  if (p.N <= kBitmapCells) {
    // one bit per cell (at most 32 KB) + the scan scratch
    const size_t smem = ((size_t)(p.N + 31) / 32 + 32) * sizeof(uint32_t);
    static std::atomic<unsigned long long> smem_set{0ull};
    cudaError_t e = set_smem_limit_once(smem_set, select_bitmap_kernel, (kBitmapCells / 32 + 32) * 4);
    if (e != cudaSuccess) return e;
    select_bitmap_kernel<<<dim3((unsigned)p.R), kSortThreads, smem, stream>>>(p);
    return cudaGetLastError();
  }
  // at most 4096 keys + the scan scratch: 16.5 KB, under the default limit
  const size_t smem = ((size_t)p.n_pow2 + kSortThreads / 32) * sizeof(int32_t);
  select_compact_kernel<<<dim3((unsigned)p.R), kSortThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_visible_lists(const SelectedPlan& p, const RowFilter& f, cudaStream_t stream) {
  visible_list_kernel<<<dim3((unsigned)p.R), kVisThreads, 0, stream>>>(p, f);
  return cudaGetLastError();
}

cudaError_t launch_selected(const SelectedPlan& p, cudaStream_t stream) {
  if (p.kv_type == ATTN_F16) return launch_selected_k<__half>(p, stream);
  return launch_selected_k<__nv_bfloat16>(p, stream);
}

}  // namespace attn
