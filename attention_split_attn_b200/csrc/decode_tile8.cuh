// decode_tile8.cuh -- the per-warp tensor-core tile step of the balanced
// decode kernel for one-byte caches: e4m3 or int8 codes with one F32 scale
// per (cell, KV head) for K and one for V (TensorFold PR #911: e4m3 rows with
// an fp32 scale per position and key head; TensorFold PR #2595: an int8
// cache with K and V scales per key).
//
// A tile is 16 cells x D codes of K and of V of one KV head, staged by TMA in
// 128-byte-swizzled boxes of 128 codes.  The codes are widened in registers
// to f16 -- exact for both formats (e4m3 by the hardware conversion, which
// also turns the S.1111.111 code into NaN; int8 by the 1024 + x bit trick)
// -- and the two products run as mma.sync m16n8k16 f16 with f32 accumulation,
// with the roles of decode_tile.cuh (q heads in the narrow N dimension):
//   S^T[16 cells x heads] = Kc[16 x D] . Q'^T,   Q'_h = 2^E_h q_h in f16
//   O^T[D x heads]       += Vc^T[D x 16] . P'^T,  P'_c = p_c v_scale[c] / vref
// E_h puts head h's largest |q| in [2^14, 2^15), so Q' holds every bf16 / f16
// query value exactly except components more than 2^31 below the largest,
// whose rounding stays below the f32 accumulation error.  The logit is then
// x_c = scale k_scale[c] 2^-E_h S, exactly the dot product of q with the
// dequantized key.  O is kept in units of vref, the largest |v_scale| of the
// visible cells met so far (rescaled when it grows, like the running max), so
// P' stays in [0, 1] and keeps f16 precision whatever the scales' magnitude.
//
// Fragment layouts.  An MMA's reduction index may be permuted freely as long
// as both operands agree, so each lane reads whole 16-byte chunks:
//  * K (A of S^T): for 128-code block b and j in {0, 1}, lane (grp, tig)
//    loads chunk c = 2 tig + j of cells grp and grp + 8; its four 4-code words
//    feed k-steps kk = 8b + 4j + t: bytes 4t, 4t+1 are reduction slots 2tig,
//    2tig+1 and bytes 4t+2, 4t+3 slots 2tig+8, 2tig+9.  The Q' fragments of
//    k-step kk take head dims 128b + 16c + 4t + {0, 1} and {2, 3}.  Chunks
//    2tig + j of two rows that differ in bit 0 land on 8 distinct 16-byte
//    bank groups under the swizzle, so the loads are conflict-free.
//  * V (A of O^T): lane grp owns head dims [DL grp, DL grp + DL), DL = D / 8;
//    it loads them for cells 2tig, 2tig+1, 2tig+8, 2tig+9 (16 bytes each per
//    128 dims); m-tile mt of O^T has rows d = DL grp + 2mt (row grp) and
//    DL grp + 2mt + 1 (row grp + 8).  Byte pairs of two cells are interleaved
//    with one prmt each before widening.
// Semantics as in decode_tile.cuh (HartsyInference PR #910).
#pragma once

#include "common.cuh"
#include "decode_tile.cuh"
#include "internal.h"
#include "mma.cuh"
#include "quant.cuh"

namespace attn {

// f16 mma (A: 16x16 f16, B: 16x8 f16, C/D f32)
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Two codes (low byte = the low f16 lane) to an exact f16x2.
template <typename CT>
__device__ __forceinline__ uint32_t codes_to_f16x2(uint32_t two) {
  if constexpr (Storage<CT>::kDtype == ATTN_FP8_E4M3) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((unsigned short)(two & 0xffffu)));
    return h2;
  } else {
    // int8 x -> the f16 whose bits are 0x6400 | (x ^ 0x80), i.e. 1024 + x + 128, minus 1152
    const uint32_t t = prmt(two ^ 0x8080u, 0x64646464u, 0x5140u);   // [x0^80, 64, x1^80, 64]
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(t), "r"(0x64806480u));
    return r;
  }
}

template <typename CT, int D, int NH>
struct WarpTileState8 {
  static constexpr int NT = NH / 8;          // head n-tiles
  static constexpr int KSTEPS = D / 16;      // k-steps of S^T, m-tiles of O^T
  static constexpr int NB = D / 128;         // 128-code blocks per cell row
  static constexpr int DL = D / 8;           // head dims of O^T per lane
  static constexpr int TILE_BYTES = kWarpTile * D;   // K or V codes of one tile
  static constexpr int BYTES = 2 * TILE_BYTES;
  static constexpr bool kEarlyRelease = true;
  uint32_t qb[KSTEPS][NT][2];                // Q'^T as B fragments (f16, permuted)
  float colsc[NT][2];                        // scale 2^-E of the heads of this lane's S^T columns
  float slope[NT][2];
  float acc[KSTEPS][NT][4];                  // O^T in units of vref
  float m[NT][2], l[NT][2];
  float vref;                                // largest |v_scale| of the visible cells so far (0: none)
  int scale_head_;                           // KV head of the current (row, KV head): its scale column
  uint32_t ka[KSTEPS][4];                    // K codes widened (A fragments of S^T)
  uint32_t vw[4][NB * 4];                    // V codes: this lane's 16-byte chunks of its 4 cells
  uint32_t koff[NB][2][2], voff[4][NB];      // shared-memory byte offsets inside a stage
  // this lane's cells' K and V scales (cells grp, grp + 8): the current tile's,
  // and the next tile's, loaded one tile ahead so their latency hides behind
  // a tile's work
  float cur_ks[2], cur_vs[2], nxt_ks[2], nxt_vs[2];

  __device__ __forceinline__ void prefetch(const DecodePlan& p, int g, int tile0, int lane) {
#pragma unroll
    for (int kr = 0; kr < 2; ++kr) {
      const int c = tile0 + (lane >> 2) + 8 * kr;
      const int64_t si = (int64_t)c * p.scale_sc + g;
      nxt_ks[kr] = c < p.N ? __ldg(p.k_scale + si) : 0.f;
      nxt_vs[kr] = c < p.N ? __ldg(p.v_scale + si) : 0.f;
    }
  }
  __device__ __forceinline__ void take_prefetched() {
    cur_ks[0] = nxt_ks[0]; cur_ks[1] = nxt_ks[1];
    cur_vs[0] = nxt_vs[0]; cur_vs[1] = nxt_vs[1];
  }

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] = acc[mt][nt][3] = 0.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) m[nt][0] = m[nt][1] = neg_inf(), l[nt][0] = l[nt][1] = 0.f;
    vref = 0.f;
  }

  // Q' of q heads h0 .. h0+G-1 of row r in the permuted B layout, with each
  // head's power-of-two scale; Q in bf16 or f16 (the cache's query dtype).
  __device__ __forceinline__ void load_q(const DecodePlan& p, int r, int h0, int lane) {
    const int grp = lane >> 2, tig = lane & 3;
    scale_head_ = h0 / p.G;
    const bool bf = p.q.type == ATTN_BF16;
    const uint16_t* qrow = static_cast<const uint16_t*>(p.q.q) + (int64_t)r * p.q.sr;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int hh = nt * 8 + grp;
      const bool hv = hh < p.G;
      const uint16_t* qh = qrow + (int64_t)(h0 + hh) * p.q.sh;
      // this lane's dims: 128 b + 16 (2 tig + j) + 0..15, as floats
      float qf[NB][2][16];
      float amax = 0.f;
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int d0 = 128 * b + 16 * (2 * tig + j);
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const uint4 w = hv ? *reinterpret_cast<const uint4*>(qh + d0 + 8 * v) : make_uint4(0u, 0u, 0u, 0u);
            float f[8];
            if (bf) unpack_vec<__nv_bfloat16>(w, f);
            else unpack_vec<__half>(w, f);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              qf[b][j][8 * v + e] = f[e];
              amax = fmaxf(amax, fabsf(f[e]));
            }
          }
        }
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      // 2^E puts amax in [2^14, 2^15): E = 14 - floor(log2 amax)
      int E = 0;
      if (amax > 0.f && amax < 3.0e38f) E = 14 - (((int)(__float_as_uint(amax) >> 23) & 0xff) - 127);
      E = max(-100, min(E, 100));
      const float up = __uint_as_float((uint32_t)(E + 127) << 23);   // 2^E
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int kk = 8 * b + 4 * j + t;
            const __half2 lo = __floats2half2_rn(qf[b][j][4 * t] * up, qf[b][j][4 * t + 1] * up);
            const __half2 hi = __floats2half2_rn(qf[b][j][4 * t + 2] * up, qf[b][j][4 * t + 3] * up);
            qb[kk][nt][0] = *reinterpret_cast<const uint32_t*>(&lo);
            qb[kk][nt][1] = *reinterpret_cast<const uint32_t*>(&hi);
          }
      // this lane's S^T columns are heads 2 tig, 2 tig + 1: their scales from
      // the lanes holding those heads' Q (grp = 2 tig + e)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int Ee = __shfl_sync(0xffffffffu, E, (2 * tig + e) * 4);
        colsc[nt][e] = __uint_as_float((uint32_t)(127 - Ee) << 23);   // 2^-E
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

  __device__ __forceinline__ void init_offsets(int lane) {
    const int grp = lane >> 2, tig = lane & 3;
    // sub-tile b of K: 16 rows x 128 B at b * 2048; chunk c of row r at (c ^ (r & 7)) * 16
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int row = grp + 8 * h, c = 2 * tig + j;
          koff[b][j][h] = (uint32_t)(b * (kWarpTile * 128) + row * 128 + ((c ^ (row & 7)) << 4));
        }
    // V: cells 2tig, 2tig+1, 2tig+8, 2tig+9; this lane's dims DL grp .. DL grp + DL
    const int cells[4] = {2 * tig, 2 * tig + 1, 2 * tig + 8, 2 * tig + 9};
#pragma unroll
    for (int ci = 0; ci < 4; ++ci)
#pragma unroll
      for (int q = 0; q < NB; ++q) {
        const int d0 = DL * grp + 16 * q;           // a 16-byte chunk of this lane's dims
        const int b = d0 >> 7, c = (d0 & 127) >> 4, row = cells[ci];
        voff[ci][q] = (uint32_t)(TILE_BYTES + b * (kWarpTile * 128) + row * 128 + ((c ^ (row & 7)) << 4));
      }
  }

  // Widen the tile's K codes into A fragments and keep the V codes of this
  // lane; after this every lane is done with the stage.
  __device__ __forceinline__ void load_tile(unsigned char* stage) {
    __syncwarp();
    const uint32_t base = smem_u32(stage);
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        uint4 r0, r1;
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(r0.x), "=r"(r0.y), "=r"(r0.z), "=r"(r0.w) : "r"(base + koff[b][j][0]));
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(r1.x), "=r"(r1.y), "=r"(r1.z), "=r"(r1.w) : "r"(base + koff[b][j][1]));
        const uint32_t w0[4] = {r0.x, r0.y, r0.z, r0.w}, w1[4] = {r1.x, r1.y, r1.z, r1.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int kk = 8 * b + 4 * j + t;
          ka[kk][0] = codes_to_f16x2<CT>(w0[t]);         // row grp, slots 2tig, 2tig+1
          ka[kk][1] = codes_to_f16x2<CT>(w1[t]);         // row grp+8
          ka[kk][2] = codes_to_f16x2<CT>(w0[t] >> 16);   // row grp, slots 2tig+8, 2tig+9
          ka[kk][3] = codes_to_f16x2<CT>(w1[t] >> 16);
        }
      }
#pragma unroll
    for (int ci = 0; ci < 4; ++ci)
#pragma unroll
      for (int q = 0; q < NB; ++q)
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(vw[ci][4 * q]), "=r"(vw[ci][4 * q + 1]), "=r"(vw[ci][4 * q + 2]), "=r"(vw[ci][4 * q + 3])
                     : "r"(base + voff[ci][q]));
  }

  // Fold the loaded tile: cells tile0 .. tile0+15 of the row; only cells
  // < rc.s_end that pass the row filter count.
  __device__ __forceinline__ void compute(const DecodePlan& p, const RowCtx& rc, int r, int tile0,
                                          bool has_filter, int lane, unsigned char* /*stage*/) {
    const int grp = lane >> 2, tig = lane & 3;
    const float scale = p.lg.scale, softcap = p.lg.softcap;
    const bool alibi = p.lg.slopes != nullptr;

    float sc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_f16(sc[nt], ka[kk], qb[kk][nt][0], qb[kk][nt][1]);

    bool vis[2];
    float vs[2];
#pragma unroll
    for (int kr = 0; kr < 2; ++kr) {
      const int c = tile0 + grp + 8 * kr;
      bool vk = c < rc.s_end;
      float mval = 0.f, negdist = 0.f;
      if (has_filter || alibi) {
        int64_t cpos = (int64_t)c - rc.pos_base;
        if (has_filter && vk) vk = cell_visible(p.f, rc, r, c, mval, cpos);
        else if (alibi && p.f.cell_pos && vk) cpos = __ldg(p.f.cell_pos + c);
        negdist = -(float)(rc.row_pos >= cpos ? rc.row_pos - cpos : cpos - rc.row_pos);
      }
      vis[kr] = vk;
      const float ks = vk ? cur_ks[kr] : 0.f;
      vs[kr] = vk ? cur_vs[kr] : 0.f;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float x = sc[nt][2 * kr + e] * (ks * colsc[nt][e]) * scale;
          if (softcap > 0.f) x = softcap * tanhf(x / softcap);
          if (alibi) x = fmaf(slope[nt][e], negdist, x);
          x += mval;
          sc[nt][2 * kr + e] = vk ? x : neg_inf();
        }
    }

    // the V reference: the largest |v_scale| of the visible cells so far
    // (NaN-propagating: a NaN scale on a visible cell makes the row NaN)
    float vt = fmax_nan(vis[0] ? fabsf(vs[0]) : 0.f, vis[1] ? fabsf(vs[1]) : 0.f);
    vt = fmax_nan(vt, __shfl_xor_sync(0xffffffffu, vt, 4));
    vt = fmax_nan(vt, __shfl_xor_sync(0xffffffffu, vt, 8));
    vt = fmax_nan(vt, __shfl_xor_sync(0xffffffffu, vt, 16));
    const float vnew = fmax_nan(vref, vt);
    const bool vgrow = !(vnew == vref);   // warp-uniform (NaN compares unequal)
    const float vcorr = vgrow ? (vref / vnew) : 1.f;   // 0 when vref was 0
    vref = vnew;

    float corr[NT][2];
    bool changed = vgrow;
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
        changed |= !(mo == mn);
        m[nt][e] = mn;
        const float p0 = ex2((sc[nt][e] - mu) * kLog2e);
        const float p1 = ex2((sc[nt][2 + e] - mu) * kLog2e);
        l[nt][e] = fmaf(l[nt][e], corr[nt][e], p0 + p1);
        sc[nt][e] = p0;
        sc[nt][2 + e] = p1;
      }
    if (__any_sync(0xffffffffu, changed)) {
#pragma unroll
      for (int mt2 = 0; mt2 < KSTEPS; ++mt2)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          acc[mt2][nt][0] *= corr[nt][0] * vcorr;
          acc[mt2][nt][1] *= corr[nt][1] * vcorr;
          acc[mt2][nt][2] *= corr[nt][0] * vcorr;
          acc[mt2][nt][3] *= corr[nt][1] * vcorr;
        }
    }

    // P' = p v_scale / vref (0 for an invisible cell or while vref is 0)
    const float inv = vref > 0.f ? 1.f / vref : 0.f;
    const float f0 = vs[0] * inv, f1 = vs[1] * inv;
    uint32_t pb[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const __half2 a = __floats2half2_rn(sc[nt][0] * f0, sc[nt][1] * f0);
      const __half2 b = __floats2half2_rn(sc[nt][2] * f1, sc[nt][3] * f1);
      pb[nt][0] = movm_trans(*reinterpret_cast<const uint32_t*>(&a));
      pb[nt][1] = movm_trans(*reinterpret_cast<const uint32_t*>(&b));
    }

    // V^T fragments; excluded cells must not reach O even through 0 * NaN,
    // so their codes are replaced by 0 before widening.  This lane's cells
    // are 2tig, 2tig+1 (registers 0, 1) and 2tig+8, 2tig+9 (registers 2, 3).
    const unsigned vis_lo = __ballot_sync(0xffffffffu, vis[0]);   // lane 4*j holds cell j
    const unsigned vis_hi = __ballot_sync(0xffffffffu, vis[1]);   // lane 4*j holds cell j+8
    auto bit = [](unsigned mm, int cell) { return (mm >> (4 * cell)) & 1u; };
    const uint32_t keep[4] = {bit(vis_lo, 2 * tig) ? 0xffffffffu : 0u, bit(vis_lo, 2 * tig + 1) ? 0xffffffffu : 0u,
                              bit(vis_hi, 2 * tig) ? 0xffffffffu : 0u, bit(vis_hi, 2 * tig + 1) ? 0xffffffffu : 0u};
#pragma unroll
    for (int q = 0; q < NB; ++q)
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t c0 = vw[0][4 * q + u] & keep[0], c1 = vw[1][4 * q + u] & keep[1];
        const uint32_t c8 = vw[2][4 * q + u] & keep[2], c9 = vw[3][4 * q + u] & keep[3];
        // bytes 4u .. 4u+3 of this lane's chunk q: dims DL grp + 16 q + 4u + {0..3}
        const uint32_t lo01 = prmt(c0, c1, 0x5140u), hi01 = prmt(c0, c1, 0x7362u);
        const uint32_t lo89 = prmt(c8, c9, 0x5140u), hi89 = prmt(c8, c9, 0x7362u);
        // m-tile mt covers dims DL grp + 2 mt (row grp) and + 1 (row grp + 8)
        const int mt_a = 8 * q + 2 * u, mt_b = mt_a + 1;
        uint32_t va[4], vb[4];
        va[0] = codes_to_f16x2<CT>(lo01);          // dim +4u,   cells 2tig, 2tig+1
        va[1] = codes_to_f16x2<CT>(lo01 >> 16);    // dim +4u+1
        va[2] = codes_to_f16x2<CT>(lo89);
        va[3] = codes_to_f16x2<CT>(lo89 >> 16);
        vb[0] = codes_to_f16x2<CT>(hi01);          // dim +4u+2
        vb[1] = codes_to_f16x2<CT>(hi01 >> 16);    // dim +4u+3
        vb[2] = codes_to_f16x2<CT>(hi89);
        vb[3] = codes_to_f16x2<CT>(hi89 >> 16);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          mma_f16(acc[mt_a][nt], va, pb[nt][0], pb[nt][1]);
          mma_f16(acc[mt_b][nt], vb, pb[nt][0], pb[nt][1]);
        }
      }
  }

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

  // Head dim of O^T row `dr` (0: row grp, 1: row grp + 8) of m-tile mt.
  __device__ __forceinline__ static int dim_of(int grp, int mt, int dr) { return DL * grp + 2 * mt + dr; }

  // Write (m, l, O) of heads h0.. as partial slot `slot` (O in true units).
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
          for (int dr = 0; dr < 2; ++dr)
            o[dim_of(grp, mt2, dr)] = poison ? qnan() : acc[mt2][nt][2 * dr + e] * vref;
        if (grp == 0) {
          pml[(slot * G + hh) * 2] = poison ? qnan() : m[nt][e];
          pml[(slot * G + hh) * 2 + 1] = poison ? qnan() : l[nt][e];
        }
      }
  }
};

}  // namespace attn
