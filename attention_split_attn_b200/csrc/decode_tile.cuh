// decode_tile.cuh -- the per-warp tensor-core tile step shared by the decode
// kernels for 16-bit caches (the (rows, heads, slices) slice kernel and the
// balanced persistent kernel).
//
// A warp owns one (row, KV head) at a time and folds 16-cell tiles into a
// running state with the roles of the contraction transposed so the q heads
// sit in the narrow N = 8 dimension of m16n8k16:
//   S^T[16 cells x heads] = K[16 x D] . Q^T[D x heads]    (K by ldmatrix)
//   O^T[D x heads]       += V^T[D x 16] . P^T[16 x heads]  (V by ldmatrix.trans)
// P^T is the S^T accumulator after the softmax, re-packed to the cache dtype
// and transposed in registers with movmatrix.  A head's running max and sum
// (a column of S^T) are reduced over the 8 lanes holding its cells with warp
// shuffles; the max is updated once per tile (TensorFold PR #985's tile-wise
// max).  Semantics as in decode.cu (HartsyInference PR #910).
#pragma once

#include "common.cuh"
#include "internal.h"
#include "mma.cuh"

namespace attn {

constexpr int kWarpTile = 16;   // cells per warp tile = one MMA m-tile

struct RowCtx {
  int32_t begin, end;        // the row's cell range, clipped to [0, n_cells)
  int32_t pos_base;          // row_begin as given (not clipped): cell c's default position is c - pos_base
  int32_t s_begin, s_end;    // the cells this unit may use
  int32_t row_seq;
  int64_t row_pos;
};

__device__ __forceinline__ bool cell_visible(const RowFilter& f, const RowCtx& rc, int r, int c,
                                             float& mval, int64_t& cpos) {
  bool vis = true;
  if (f.cell_seq != nullptr && f.row_seq != nullptr) vis = (__ldg(f.cell_seq + c) == rc.row_seq);
  cpos = f.cell_pos ? (int64_t)__ldg(f.cell_pos + c) : (int64_t)c - rc.pos_base;
  if (f.causal) vis = vis && (cpos <= rc.row_pos);
  mval = 0.f;
  if (f.mask != nullptr) {
    mval = __ldg(f.mask + (int64_t)r * f.mask_sr + c);
    vis = vis && !(mval == neg_inf());
  }
  return vis;
}

// Final fold of one (row, head): state (M, L, O) with the sink.
__device__ __forceinline__ float fold_with_sink(float M, float L, float O, float sigma) {
  const float Mf = fmax_nan(M, sigma);
  if (isnan(Mf)) return qnan();
  if (Mf == neg_inf()) return 0.f;
  const float f = ex2((M - Mf) * kLog2e);
  const float Lf = L * f + ex2((sigma - Mf) * kLog2e);
  return (O * f) / Lf;
}

__device__ __forceinline__ unsigned char* align1024(unsigned char* p) {
  const uint32_t a = smem_u32(p);
  return p + (((a + 1023u) & ~1023u) - a);
}

// Byte layout of one ring stage: K tile then V tile, each D/64 swizzled
// sub-tiles of [16 rows][128 B].
template <int D>
struct WarpStage {
  static constexpr int TILE_BYTES = kWarpTile * D * 2;
  static constexpr int BYTES = 2 * TILE_BYTES;
};

// TMA of one 16-cell K/V tile of KV head g starting at cell c0.
template <int D>
__device__ __forceinline__ void issue_warp_tile(unsigned char* stage, uint64_t* bar, const CUtensorMap* tmK,
                                                const CUtensorMap* tmV, int g, int c0, uint64_t pol) {
  mbar_arrive_expect_tx(bar, WarpStage<D>::BYTES);
#pragma unroll
  for (int sub = 0; sub < D / 64; ++sub) {
    tma_load_3d(stage + sub * (kWarpTile * 128), tmK, bar, sub * 64, g, c0, pol);
    tma_load_3d(stage + WarpStage<D>::TILE_BYTES + sub * (kWarpTile * 128), tmV, bar, sub * 64, g, c0, pol);
  }
}

template <typename KT, int D, int NH>
struct WarpTileState {
  static constexpr int NT = NH / 8;          // head n-tiles
  static constexpr int KSTEPS = D / 16;
  uint32_t qb[KSTEPS][NT][2];                // Q^T as B fragments
  float slope[NT][2];
  float acc[KSTEPS][NT][4];                  // O^T
  float m[NT][2], l[NT][2];

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] = acc[mt][nt][3] = 0.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) m[nt][0] = m[nt][1] = neg_inf(), l[nt][0] = l[nt][1] = 0.f;
  }

  // Q rows of q heads h0 .. h0+G-1 of query row r (column n = head nt*8 + grp).
  __device__ __forceinline__ void load_q(const DecodePlan& p, int r, int h0, int lane) {
    const int grp = lane >> 2, tig = lane & 3;
    const KT* qrow = static_cast<const KT*>(p.q.q) + (int64_t)r * p.q.sr;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int hh = nt * 8 + grp;
      const bool hv = hh < p.G;
      const KT* qh = qrow + (int64_t)(h0 + hh) * p.q.sh;
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        qb[kk][nt][0] = hv ? *reinterpret_cast<const uint32_t*>(qh + kk * 16 + 2 * tig) : 0u;
        qb[kk][nt][1] = hv ? *reinterpret_cast<const uint32_t*>(qh + kk * 16 + 8 + 2 * tig) : 0u;
      }
    }
    const bool alibi = p.lg.slopes != nullptr;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int hh = nt * 8 + 2 * tig + e;
        slope[nt][e] = (alibi && hh < p.G) ? __ldg(p.lg.slopes + h0 + hh) : 0.f;
      }
  }

  // ldmatrix byte offsets inside a stage; identical for every tile.
  uint32_t koff[KSTEPS], voff[KSTEPS];
  __device__ __forceinline__ void init_offsets(int lane) {
    const int mi = lane >> 3;
    const int keyk = (lane & 7) + (mi & 1) * 8, keyv = (lane & 7) + (mi >> 1) * 8;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      koff[kk] = swz_offset<kWarpTile>(keyk, 2 * kk + (mi >> 1));
      voff[kk] = WarpStage<D>::TILE_BYTES + swz_offset<kWarpTile>(keyv, 2 * kk + (mi & 1));
    }
  }

  // The whole tile as MMA fragments: K (A operand of S^T = K Q^T) and V^T
  // (A operand of O^T += V^T P^T).  Once every lane has them the stage can be
  // refilled while the tile is still being computed.
  // With head_dim 256 the V fragments would not fit beside the rest, so V
  // stays in shared memory until the PV product and the stage is refilled
  // only after compute() (kEarlyRelease false).
  static constexpr bool kEarlyRelease = D <= 128;
  uint32_t ka[KSTEPS][4], va[KSTEPS][4];
  __device__ __forceinline__ void load_v(uint32_t base) {
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) ldsm_x4_trans(va[kk][0], va[kk][1], va[kk][2], va[kk][3], base + voff[kk]);
  }
  __device__ __forceinline__ void load_tile(unsigned char* stage) {
    __syncwarp();   // the lanes left their barrier waits independently
    const uint32_t base = smem_u32(stage);
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) ldsm_x4(ka[kk][0], ka[kk][1], ka[kk][2], ka[kk][3], base + koff[kk]);
    if (kEarlyRelease) load_v(base);
  }

  // (one-byte caches load per-cell scales ahead; 16-bit caches have none)
  __device__ __forceinline__ void prefetch(const DecodePlan&, int, int, int) {}
  __device__ __forceinline__ void take_prefetched() {}

  // Fold the loaded tile: cells tile0 .. tile0+15 of the row; only cells
  // < rc.s_end that pass the row filter count.
  __device__ __forceinline__ void compute(const DecodePlan& p, const RowCtx& rc, int r, int tile0,
                                          bool has_filter, int lane, unsigned char* stage) {
    using Op = MmaType<KT>;
    const int grp = lane >> 2, tig = lane & 3;
    const float scale = p.lg.scale, softcap = p.lg.softcap;
    const bool alibi = p.lg.slopes != nullptr;

    float sc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) Op::mma(sc[nt], ka[kk], qb[kk][nt][0], qb[kk][nt][1]);

    bool vis[2];
#pragma unroll
    for (int kr = 0; kr < 2; ++kr) {
      const int c = tile0 + grp + 8 * kr;
      bool vk = c < rc.s_end;
      float mval = 0.f;
      float negdist = 0.f;
      if (has_filter || alibi) {
        int64_t cpos = (int64_t)c - rc.pos_base;
        if (has_filter && vk) vk = cell_visible(p.f, rc, r, c, mval, cpos);
        else if (alibi && p.f.cell_pos && vk) cpos = __ldg(p.f.cell_pos + c);
        negdist = -(float)(rc.row_pos >= cpos ? rc.row_pos - cpos : cpos - rc.row_pos);
      }
      vis[kr] = vk;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float x = sc[nt][2 * kr + e] * scale;
          if (softcap > 0.f) x = softcap * tanhf(x / softcap);
          if (alibi) x = fmaf(slope[nt][e], negdist, x);
          x += mval;
          sc[nt][2 * kr + e] = vk ? x : neg_inf();
        }
    }

    float corr[NT][2];
    bool changed = false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float mt = fmax_nan(sc[nt][e], sc[nt][2 + e]);
        mt = fmax_nan(mt, __shfl_xor_sync(0xffffffffu, mt, 4));
        mt = fmax_nan(mt, __shfl_xor_sync(0xffffffffu, mt, 8));
        mt = fmax_nan(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
        const float mo = m[nt][e];
        const float mn = fmax_nan(mo, mt);
        const float mu = (mn == neg_inf()) ? 0.f : mn;
        corr[nt][e] = ex2((mo - mu) * kLog2e);
        changed |= !(mo == mn);   // NaN compares unequal: a NaN max always rescales
        m[nt][e] = mn;
        const float p0 = ex2((sc[nt][e] - mu) * kLog2e);
        const float p1 = ex2((sc[nt][2 + e] - mu) * kLog2e);
        l[nt][e] = fmaf(l[nt][e], corr[nt][e], p0 + p1);
        sc[nt][e] = p0;
        sc[nt][2 + e] = p1;
      }
    // Rescale O only when some head's max moved (corr == 1 exactly otherwise).
    if (__any_sync(0xffffffffu, changed)) {
#pragma unroll
      for (int mt2 = 0; mt2 < KSTEPS; ++mt2)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          acc[mt2][nt][0] *= corr[nt][0];
          acc[mt2][nt][1] *= corr[nt][1];
          acc[mt2][nt][2] *= corr[nt][0];
          acc[mt2][nt][3] *= corr[nt][1];
        }
    }

    if (!kEarlyRelease) load_v(smem_u32(stage));

    // Excluded cells must not reach O even through 0 * NaN: clear their V
    // values in the fragments.  This lane's V^T fragments hold cells 2tig,
    // 2tig+1 (registers 0, 1) and 2tig+8, 2tig+9 (registers 2, 3).
    const unsigned vis_lo = __ballot_sync(0xffffffffu, vis[0]);   // lane 4*j holds cell j
    const unsigned vis_hi = __ballot_sync(0xffffffffu, vis[1]);   // lane 4*j holds cell j+8
    if ((vis_lo & vis_hi & 0x11111111u) != 0x11111111u) {
      auto bit = [](unsigned m, int cell) { return (m >> (4 * cell)) & 1u; };
      const uint32_t m01 = (bit(vis_lo, 2 * tig) ? 0x0000ffffu : 0u) | (bit(vis_lo, 2 * tig + 1) ? 0xffff0000u : 0u);
      const uint32_t m23 = (bit(vis_hi, 2 * tig) ? 0x0000ffffu : 0u) | (bit(vis_hi, 2 * tig + 1) ? 0xffff0000u : 0u);
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        va[kk][0] &= m01;
        va[kk][1] &= m01;
        va[kk][2] &= m23;
        va[kk][3] &= m23;
      }
    }

    uint32_t pb[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      pb[nt][0] = movm_trans(Op::pack(sc[nt][0], sc[nt][1]));
      pb[nt][1] = movm_trans(Op::pack(sc[nt][2], sc[nt][3]));
    }
#pragma unroll
    for (int mt2 = 0; mt2 < KSTEPS; ++mt2)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) Op::mma(acc[mt2][nt], va[mt2], pb[nt][0], pb[nt][1]);
  }

  // Sum the row sums over the 8 lanes that hold a head's cells.
  __device__ __forceinline__ void finish_sums() {
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
  }

  // Write (m, l, O) of heads h0.. as partial slot `slot` of a [slots][G][D]
  // store (o) and [slots][G][2] store (ml).
  __device__ __forceinline__ void write_partial(float* po, float* pml, int64_t slot, int G, int lane,
                                                bool poison) {
    const int grp = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int hh = nt * 8 + 2 * tig + e;
        if (hh >= G) continue;
        float* o = po + (slot * G + hh) * D;
#pragma unroll
        for (int mt2 = 0; mt2 < KSTEPS; ++mt2)
#pragma unroll
          for (int dr = 0; dr < 2; ++dr) o[mt2 * 16 + grp + 8 * dr] = poison ? qnan() : acc[mt2][nt][2 * dr + e];
        if (grp == 0) {
          pml[(slot * G + hh) * 2] = poison ? qnan() : m[nt][e];
          pml[(slot * G + hh) * 2 + 1] = poison ? qnan() : l[nt][e];
        }
      }
  }

  // Fold with the sinks and store the final rows of heads h0.. of row r.
  __device__ __forceinline__ void write_final(const DecodePlan& p, int r, int h0, int lane, bool poison) {
    const int grp = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int hh = nt * 8 + 2 * tig + e;
        if (hh >= p.G) continue;
        const int hq = h0 + hh;
        const float sigma = p.lg.sinks ? __ldg(p.lg.sinks + hq) : neg_inf();
        const int64_t ob = (int64_t)r * p.out.sr + (int64_t)hq * p.out.sh;
#pragma unroll
        for (int mt2 = 0; mt2 < KSTEPS; ++mt2)
#pragma unroll
          for (int dr = 0; dr < 2; ++dr) {
            const int d = mt2 * 16 + grp + 8 * dr;
            const float v = poison ? qnan() : fold_with_sink(m[nt][e], l[nt][e], acc[mt2][nt][2 * dr + e], sigma);
            store_from_float(p.out.out, ob + d, p.out.type, v);
          }
      }
  }
};

}  // namespace attn
