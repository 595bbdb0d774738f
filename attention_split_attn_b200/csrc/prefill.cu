// prefill.cu -- causal prefill on the sm_100a tensor cores (tcgen05 + TMEM).
//
// Many query rows attend over the cache with the semantics of decode
// (HartsyInference PR #910 "attention semantic correctness": softcap before
// ALiBi, F32 mask bias added unnarrowed, per-head sinks, +0 for rows with no
// visible cell, NaN propagated).  The two dense contractions, S = Q K^T and
// O += P V, run as tcgen05.mma (kind::f16, f32 accumulators in tensor memory);
// everything between them (logit transforms, visibility, online softmax) runs
// on the CUDA cores of two softmax warpgroups.
//
// Two kernels:
//  * prefill_classify_kernel tags each (128-row tile, 128-cell tile) as
//    skipped / full / mixed from the visibility rules and the mask, and each
//    (cell tile, KV head) whose V holds a non-finite value.  Skipped tiles are
//    never loaded; full tiles need no per-element visibility or mask work;
//    only mixed tiles read the mask.  (The split of masked work by tile class
//    follows the pages' observation that masked cells cost time in dense
//    paths: strix-llama.cpp PR #115 "Performance" discussion.)
//  * prefill_kernel: one CTA per (row tile, two q heads of one KV group).  Both
//    heads share every K and V tile, so each tile crosses L2 once per pair.
//    With fewer rows than a tile and several q heads per KV head (draft-tree
//    rows, short prefills) the rows are packed: a tile's 128 lanes hold
//    128 / G rows x the G heads of one KV group (lane t: row t / G, head
//    t % G, the Q box being G heads x 128 / G rows), one head slot per CTA,
//    so each K and V tile serves the whole group at once.
//      warp 0       TMA producer: Q of both heads once, then K_j into a
//                   one-tile K buffer and V_j into a two-tile V ring
//                   (128-byte swizzled boxes of 64 x 128).
//      warp 1       allocates 512 TMEM columns and issues the MMAs:
//                     S_i  (TMEM cols i*128 .. +128)  = Q_i K_j^T
//                     O_i  (TMEM cols 256 + i*D ..)  += P_i V_j
//                   P_i lives in the first 64 columns of S_i (16-bit, two
//                   values per column) and is the MMA's A operand straight
//                   from tensor memory.  Per head the tensor core runs
//                   P V(j), then S(j+1) over the same columns; while one
//                   head's softmax runs, the tensor core works for the other.
//      warps 2-5    softmax of head slot 0; warps 6-9: slot 1.  Thread t owns
//                   query row t of the tile (TMEM lane t): it reads its row of
//                   S with tcgen05.ld, applies the transforms, keeps the
//                   running max m and sum l, writes P (16-bit) over its row
//                   of S in tensor memory, and
//                   rescales its O row in TMEM only when the max grew by more
//                   than ln 256 (lazy rescaling: the weights stay <= 256, and
//                   m is the common reference of l and O, so the result is
//                   the same softmax).
//    Mixed tiles whose V has a non-finite value for this KV head take P V on
//    the CUDA cores instead, over each row's visible cells only, so that a NaN
//    in a cell a row cannot see never reaches that row through 0 * NaN.
//  All mbarrier waits are bounded; a timeout records ATTN_ERR_DEVICE_TIMEOUT,
//  raises a CTA-wide abort flag, drains copies in flight and frees TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace attn {
namespace {

constexpr int kPfRows = 128;   // query rows per tile (MMA M)
constexpr int kPfCells = 128;  // cells per tile (MMA N of S, K of P V)

__device__ __forceinline__ unsigned char* pf_align1024(unsigned char* p) {
  const uint32_t a = smem_u32(p);
  return p + (((a + 1023u) & ~1023u) - a);
}

// ---------------------------------------------------------------------------
// tile classifier
// ---------------------------------------------------------------------------

struct RowVis {
  int32_t rb, re, rs, rp;
};

__device__ __forceinline__ RowVis row_vis(const RowFilter& f, int r, int N) {
  RowVis v;
  v.rb = f.row_begin ? __ldg(f.row_begin + r) : 0;
  v.re = f.row_end ? __ldg(f.row_end + r) : N;
  v.rs = f.row_seq ? __ldg(f.row_seq + r) : 0;
  v.rp = f.row_pos ? __ldg(f.row_pos + r) : v.re - v.rb - 1;
  return v;
}

// Classification of tile b = (rt, kt) by one CTA of 256 threads: the tile's
// rows' (128, or 128 / G when rows are packed) range, sequence and position
// are staged in shared memory; warp w
// takes rows w, w + 8, ..., lane l cells 4l .. 4l + 3 of the tile, and each
// warp issues its 16 rows' 16-byte mask loads before using any of them (the
// scan is bound by DRAM latency otherwise).  A row's visibility bits are gathered from the lanes'
// nibbles by three shuffles per 8-lane group (word k = cells 32k .. 32k + 31).
constexpr int kClsThreads = 256;
constexpr int kClsRowsPerWarp = kPfRows / (kClsThreads / 32);   // 16

__device__ __forceinline__ void pf_classify_tile(const PrefillPlan& p, int64_t b, int4* rows_sh) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int rt = (int)(b / p.n_kt), kt = (int)(b % p.n_kt);
    if (tid < p.rpt) {
      const int r = rt * p.rpt + tid;
      const RowVis rv = r < p.R ? row_vis(p.f, r, p.N) : RowVis{0, 0, 0, 0};
      rows_sh[tid] = make_int4(rv.rb, rv.re, rv.rs, rv.rp);
    }
    const int c_base = kt * kPfCells + 4 * lane;
    bool cin[4];
    int32_t cs[4], cpg[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = c_base + e;
      cin[e] = c < p.N;
      cs[e] = (cin[e] && p.f.cell_seq) ? __ldg(p.f.cell_seq + c) : 0;
      cpg[e] = (cin[e] && p.f.cell_pos) ? __ldg(p.f.cell_pos + c) : 0;
    }
    // the 16 rows of each warp in two batches of 8: a batch's 16-byte mask
    // loads all go out before any is used, and the smaller register set lets
    // four CTAs share an SM
    bool any = false, notfull = false, bias = false, late = false;
#pragma unroll
    for (int hb = 0; hb < 2; ++hb) {
    float4 mv[kClsRowsPerWarp / 2];
    if (p.f.mask) {
      const bool vec = p.mask_vec && kt * kPfCells + kPfCells <= p.N;
#pragma unroll
      for (int i2 = 0; i2 < kClsRowsPerWarp / 2; ++i2) {
        const int i = hb * (kClsRowsPerWarp / 2) + i2;
        const int r = rt * p.rpt + warp + 8 * i;
        mv[i2] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (warp + 8 * i < p.rpt && r < p.R) {
          const float* mrow = p.f.mask + (int64_t)r * p.f.mask_sr + c_base;
          if (vec) {
            mv[i2] = __ldg(reinterpret_cast<const float4*>(mrow));
          } else {
            if (cin[0]) mv[i2].x = __ldg(mrow);
            if (cin[1]) mv[i2].y = __ldg(mrow + 1);
            if (cin[2]) mv[i2].z = __ldg(mrow + 2);
            if (cin[3]) mv[i2].w = __ldg(mrow + 3);
          }
        }
      }
    }
    if (hb == 0) __syncthreads();   // the rows' data staged
#pragma unroll
    for (int i2 = 0; i2 < kClsRowsPerWarp / 2; ++i2) {
      const int i = hb * (kClsRowsPerWarp / 2) + i2;
      const int rl = warp + 8 * i;
      if (rl >= p.rpt || rt * p.rpt + rl >= p.R) continue;   // warp-uniform
      const int4 rv = rows_sh[rl];
      const float mvals[4] = {mv[i2].x, mv[i2].y, mv[i2].z, mv[i2].w};
      uint32_t nib = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = c_base + e;
        bool vis = cin[e] && c >= rv.x && c < rv.y;
        if (p.f.cell_seq) vis = vis && cs[e] == rv.z;
        const int32_t cp = p.f.cell_pos ? cpg[e] : c - rv.x;
        if (p.f.causal) vis = vis && cp <= rv.w;
        bool zero_bias = true;
        if (p.f.mask && vis) {
          vis = !(mvals[e] == neg_inf());
          zero_bias = (mvals[e] == 0.f);
        }
        any |= vis;
        notfull |= !(vis && zero_bias);
        bias |= vis && !zero_bias;
        late |= vis && cp > rv.w;
        nib |= (vis ? 1u : 0u) << e;
      }
      if (p.bits) {
        uint32_t word = nib << (4 * (lane & 7));
        word |= __shfl_xor_sync(0xffffffffu, word, 1);
        word |= __shfl_xor_sync(0xffffffffu, word, 2);
        word |= __shfl_xor_sync(0xffffffffu, word, 4);
        if ((lane & 7) == 0) p.bits[((b * kPfRows + rl) << 2) + (lane >> 3)] = word;
      }
    }
    }
    const int a = __syncthreads_or(any ? 1 : 0);
    const int nf = __syncthreads_or(notfull ? 1 : 0);
    const int bs = __syncthreads_or(bias ? 1 : 0);
    const int lt = __syncthreads_or(late ? 1 : 0);
    if (tid == 0) {
      const int cl = !a ? kTileSkip : !nf ? kTileFull : (p.bits && !bs) ? kTileBits : kTileMixed;
      p.cls[b] = (uint8_t)(cl | (lt ? kTileLate : 0));
    }
}

// V scan and K norms of cell tile kt for KV head g by one CTA: every 16-byte
// chunk of a round is loaded before any is used.
__device__ __forceinline__ void pf_scan_tile(const PrefillPlan& p, int kt, int g, float* wmax) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // 16-byte chunks of the tile's rows of head g: 128 cells x D/8 chunks,
    // chunk i of this thread = tid + 256 i (per_row chunks of one cell sit in
    // per_row consecutive lanes; per_row divides 32).
    const int per_row = p.D / 8;
    const int n_chunk = kPfCells * per_row;
    constexpr int kPer = 4;   // chunks per thread per round (all loads of a round go out first)
    const uint16_t* vbase = static_cast<const uint16_t*>(p.v) + (int64_t)g * p.kv_sh;
    const uint16_t* kbase = static_cast<const uint16_t*>(p.k) + (int64_t)g * p.kv_sh;
    // A 16-bit value is non-finite iff its exponent field is all ones.
    const uint32_t e_lo = p.kv_type == ATTN_BF16 ? 0x7F80u : 0x7C00u;
    bool bad = false;
    float mx = 0.f;   // max over the tile's cells of |k_c|^2 (NaN-propagating)
    for (int base = 0; base < n_chunk; base += kPer * kClsThreads) {
      uint4 vw[kPer], kw[kPer];
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int i = base + tid + k * kClsThreads;
        const int c = kt * kPfCells + i / per_row;
        vw[k] = make_uint4(0u, 0u, 0u, 0u);
        kw[k] = make_uint4(0u, 0u, 0u, 0u);
        if (i < n_chunk && c < p.N) {
          vw[k] = __ldg(reinterpret_cast<const uint4*>(vbase + (int64_t)c * p.kv_sc) + (i % per_row));
          if (p.kn2) kw[k] = __ldg(reinterpret_cast<const uint4*>(kbase + (int64_t)c * p.kv_sc) + (i % per_row));
        }
      }
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const uint32_t ws[4] = {vw[k].x, vw[k].y, vw[k].z, vw[k].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) bad |= ((ws[q] & e_lo) == e_lo) | (((ws[q] >> 16) & e_lo) == e_lo);
      }
      if (p.kn2) {
        // the per_row chunks of one cell sit in per_row consecutive lanes
        // (per_row divides 32) or, at head dim 256, in one warp's 32 lanes
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
          const uint32_t ws[4] = {kw[k].x, kw[k].y, kw[k].z, kw[k].w};
          float ss = 0.f;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float lo, hi;
            if (p.kv_type == ATTN_BF16) {
              lo = __uint_as_float(ws[q] << 16);
              hi = __uint_as_float(ws[q] & 0xffff0000u);
            } else {
              lo = __half2float(__ushort_as_half((unsigned short)(ws[q] & 0xffffu)));
              hi = __half2float(__ushort_as_half((unsigned short)(ws[q] >> 16)));
            }
            ss = fmaf(lo, lo, ss);
            ss = fmaf(hi, hi, ss);
          }
          for (int o = min(per_row, 32) / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
          mx = fmax_nan(mx, ss);
        }
      }
    }
    const int any_bad = __syncthreads_or(bad ? 1 : 0);
    if (tid == 0) p.vbad[(int64_t)kt * p.Hkv + g] = any_bad ? 1 : 0;
    if (p.kn2) {
      for (int o = 16; o > 0; o >>= 1) mx = fmax_nan(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (lane == 0) wmax[warp] = mx;
      __syncthreads();
      if (tid == 0) {
        float m = wmax[0];
        for (int w8 = 1; w8 < kClsThreads / 32; ++w8) m = fmax_nan(m, wmax[w8]);
        p.kn2[(int64_t)kt * p.Hkv + g] = m;
      }
    }
}

// Blocks b < n_rt * n_kt classify tile b; the blocks after them scan one
// (cell tile, KV head) each.
__global__ void __launch_bounds__(kClsThreads, 4) prefill_classify_kernel(PrefillPlan p) {
  pdl_launch_dependents();   // the prefill kernel may start its prologue
  __shared__ int4 rows_sh[kPfRows];
  __shared__ float wmax[kClsThreads / 32];
  const int64_t b = blockIdx.x;
  if (b == 0)   // the row counters of split units start at zero in every call
    for (int64_t i = threadIdx.x; i < p.n_split * 2 * kPfRows; i += kClsThreads) p.split_cnt[i] = 0;
  const int64_t n_cls = (int64_t)p.n_rt * p.n_kt;
  if (b < n_cls) {
    pf_classify_tile(p, b, rows_sh);
  } else {
    const int64_t vb = b - n_cls;
    pf_scan_tile(p, (int)(vb / p.Hkv), (int)(vb % p.Hkv), wmax);
  }
}

// ---------------------------------------------------------------------------
// the tensor-core kernel: shared-memory layout and helpers
// ---------------------------------------------------------------------------

template <int D>
struct PfLayout {
  static constexpr int BOX = 128 * 128;                  // one TMA box: 128 rows x 128 B (64 values)
  static constexpr int TILE = kPfRows * D * 2;           // a Q, K or V tile: D/64 boxes
  // q heads per CTA (head slots): S and O of a head take 128 + D tensor-memory
  // columns, so two heads fit the 512 columns up to head dim 128, one at 256
  static constexpr int HPC = D <= 128 ? 2 : 1;
  static constexpr int NK = D == 64 ? 3 : D == 128 ? 2 : 1;   // K ring stages (one tile each)
  static constexpr int NV = D == 64 ? 4 : D == 128 ? 3 : 1;   // V ring stages
  static constexpr int OFF_Q = 0;                        // [HPC slots][TILE]
  static constexpr int OFF_K = OFF_Q + HPC * TILE;       // [NK][TILE]
  static constexpr int OFF_V = OFF_K + NK * TILE;        // [NV][TILE]
  static constexpr int OFF_BAR = OFF_V + NV * TILE;
  // q_full, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV], s_full[2],
  // p_full[2], pv_last[2] (the last P V of each head slot), mma_done, stall
  // (never arrived at: the bounded-wait test)
  static constexpr int N_BAR = 1 + 2 * NK + 2 * NV + 6 + 2;
  static constexpr int OFF_MISC = OFF_BAR + N_BAR * 8;   // TMEM base address, abort flag
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int SMEM = BYTES + 1024;              // slack for 1024-byte alignment
  static constexpr int THREADS = 384;                    // 12 warps: 3 warpgroups
  // Register split (setmaxnreg): the launch gives every thread LAUNCH_REGS;
  // warpgroup 0 (producer, MMA issuer, two idle warps) drops to LOW_REGS and
  // the two softmax warpgroups rise to HIGH_REGS.  The total stays within
  // what the launch holds, so the increase never waits.  The compiler
  // allocates each side within its share: at 56 / 224 the producer and the
  // MMA issuer spilled (740 bytes of spill loads per thread at head dim 128),
  // at 72 / 216 neither side does (about 30 bytes), which took the causal
  // prefill from 666 to 695 TFLOP/s.
  static constexpr int LAUNCH_REGS = 168;
  static constexpr int LOW_REGS = 72;
  static constexpr int HIGH_REGS = 216;
  static_assert(128 * LOW_REGS + 256 * HIGH_REGS <= THREADS * LAUNCH_REGS, "register split");
  static_assert(THREADS * LAUNCH_REGS <= 65536, "launch registers");
  static constexpr uint32_t TMEM_COLS = 512;             // S_s at 128 s, O_s at 256 + D s
  static_assert(HPC * 128 <= 256 && 256 + HPC * D <= (int)TMEM_COLS, "TMEM columns");
  static_assert(SMEM <= 232448, "shared memory");
};


// K and V rings: the i-th K (or V) tile the CTA loads goes to stage i % NK
// (i % NV); its "full" barrier completes phase i / NK for it, and the stage's
// "empty" barrier completes once the tensor core is done with it (K: every
// head's S of that tile; V: every head's P V), which the load of tile
// i + NK (i + NV) waits for.  With two K and three V stages the next tiles
// stream in a step or more ahead of the MMAs that read them.
template <int N>
__device__ __forceinline__ int pf_stage(int64_t i) { return (int)(i % N); }
template <int N>
__device__ __forceinline__ uint32_t pf_phase(int64_t i) { return (uint32_t)((i / N) & 1); }

struct PfBars {
  uint64_t *q_full, *k_full, *k_empty, *v_full, *v_empty, *s_full, *p_full, *pv_last, *mma_done, *stall;
};
template <int D>
__device__ __forceinline__ PfBars pf_bars(unsigned char* sm) {
  using L = PfLayout<D>;
  uint64_t* b = reinterpret_cast<uint64_t*>(sm + L::OFF_BAR);
  PfBars r;
  r.q_full = b;
  r.k_full = b + 1;
  r.k_empty = r.k_full + L::NK;
  r.v_full = r.k_empty + L::NK;
  r.v_empty = r.v_full + L::NV;
  r.s_full = r.v_empty + L::NV;
  r.p_full = r.s_full + 2;
  r.pv_last = r.s_full + 4;   // [2]: the last P V of each head slot retired
  r.mma_done = r.s_full + 6;
  r.stall = r.s_full + 7;
  return r;
}

// Bounded wait (at most p.wait_ns) that also gives up as soon as another
// thread of the CTA has raised the abort flag.
__device__ __forceinline__ bool pf_wait(uint64_t* bar, uint32_t parity, const PrefillPlan& p,
                                        volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t spin = 1;; ++spin) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((spin & 63u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > p.wait_ns) {
        record_status(p.status, ATTN_ERR_DEVICE_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// Warp-uniform form: every lane waits; the warp goes on only if all did.
__device__ __forceinline__ bool pf_wait_warp(uint64_t* bar, uint32_t parity, const PrefillPlan& p,
                                             volatile int* abort_flag) {
  const bool ok = pf_wait(bar, parity, p, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

// S (TMEM, 128 x 128 f32) = Q (128 x D) . K (128 x D)^T; both operands K-major
// 128-byte-swizzled boxes of 64 columns.  One MMA per 16 columns of D: inside a
// box the start address advances by 32 bytes, across boxes by one box.
// The descriptors come in prebuilt: a descriptor's start-address field is
// its low 14 bits (byte address >> 4), so the descriptor of base + off is
// desc(base) + (off >> 4) -- no carry, shared-memory addresses stay below
// 2^18 bytes.  One thread issues all MMAs while two softmax warps share its
// scheduler, so every instruction saved here shortens the tensor core's wait.
template <int D>
__device__ __forceinline__ void pf_issue_s(uint32_t d_tmem, uint64_t q_desc, uint64_t k_desc, uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint64_t off = (uint64_t)(((kk >> 2) * PfLayout<D>::BOX + (kk & 3) * 32) >> 4);
    umma_ss(d_tmem, q_desc + off, k_desc + off, idesc, kk > 0 ? 1u : 0u);
  }
}

// O (TMEM, 128 x D f32) (+)= P . V with P in tensor memory: P (16-bit, two
// values per 32-bit column, row i in lane i) sits in the first 64 columns of
// the head's S region, and each MMA takes 16 cells = 8 columns of it.  V (128
// cells x D, D contiguous) is MN-major: its 8-cell groups are 1024 bytes apart
// (SBO) and its 64-column boxes one box apart (LBO).
template <int D>
__device__ __forceinline__ void pf_issue_pv_ts(uint32_t d_tmem, uint32_t p_tmem, uint64_t v_desc, uint32_t idesc,
                                               bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < kPfCells / 16; ++kk)
    umma_ts(d_tmem, p_tmem + (uint32_t)kk * 8u, v_desc + (uint64_t)((kk * 2048) >> 4), idesc,
            (accumulate || kk > 0) ? 1u : 0u);
}

// Cell tiles of one row tile, skipping the empty ones, from the LAST to the
// first: under causality the nearest cells come first, and with ALiBi they
// carry the largest logits, so the running max is set by the first tile and
// the output rarely needs rescaling afterwards.  All roles walk this order.
struct PfTiles {
  const uint8_t* cls;    // this row tile's class row [n_kt]
  const uint8_t* vbad;   // [n_kt][Hkv]
  int n_kt, Hkv, g;
  int hi, lo;            // this CTA's tiles: kt in (lo, hi], not skipped (a part of a split unit)
  __device__ __forceinline__ int below(int kt) const {
    while (kt >= 0 && (cls[kt] & 3) == kTileSkip) --kt;
    return kt;
  }
  __device__ __forceinline__ int first() const { return hi; }
  __device__ __forceinline__ int next(int kt) const {
    const int n = below(kt - 1);
    return n > lo ? n : -1;
  }
  // Full, Mixed or Bits; MixedBadV for a non-full tile whose V (this KV head)
  // holds a non-finite value (P V then runs on the CUDA cores).
  __device__ __forceinline__ int code(int kt) const {
    const int c = cls[kt] & 3;
    if (c >= kTileMixed && vbad[(int64_t)kt * Hkv + g]) return kTileMixedBadV;
    return c;
  }
  __device__ __forceinline__ bool bits(int kt) const { return (cls[kt] & 3) == kTileBits; }
  __device__ __forceinline__ bool late(int kt) const { return (cls[kt] & kTileLate) != 0; }
};

// ---------------------------------------------------------------------------
// softmax warpgroups
// ---------------------------------------------------------------------------

// Softcap x = c * tanh(u / c) of a raw logit u = scale * q.k.
//  pf_cap_poly: the odd Taylor series of c tanh(u / c) through u^7,
//    u + u w (k3 + w (k5 + w k7)) with w = u^2 and k_n = t_n / c^(n-1)
//    (t_3 = -1/3, t_5 = 2/15, t_7 = -17/315); for |u| <= c/5 the truncation
//    is below 2e-8 c.  No branch, FMA pipe only.
//  pf_cap_exact: any u, tanh |y| = 1 - 2 / (e^{2|y|} + 1) with 2^x on the
//    special-function unit; NaN stays NaN, +-inf gives +-c.
__device__ __forceinline__ float pf_cap_poly(float u, float k3, float k5, float k7) {
  const float w = u * u;
  float h = fmaf(w, k7, k5);
  h = fmaf(w, h, k3);
  return fmaf(u * w, h, u);
}
__device__ __forceinline__ float pf_cap_exact(float u, float c) {
  const float e = ex2((2.f * kLog2e) * (fabsf(u) / c));
  const float t = 1.f - 2.f / (e + 1.f);
  return copysignf(c * t, u);
}
__device__ __forceinline__ float pf_softcap(float u, const PrefillPlan& p) {
  return fabsf(u) <= p.cap_lim ? pf_cap_poly(u, p.k3, p.k5, p.k7) : pf_cap_exact(u, p.lg.softcap);
}

__device__ __forceinline__ float pf_max8(const float* v) {
  return fmax_nan(fmax_nan(fmax_nan(v[0], v[1]), fmax_nan(v[2], v[3])),
                  fmax_nan(fmax_nan(v[4], v[5]), fmax_nan(v[6], v[7])));
}

// Logit transforms of one thread's row of a tile: x_i = softcap(scale s_i),
// then + slope * -|row_pos - cell_pos| (AL 1: cell positions c - row_begin,
// i.e. row_pos + row_begin - c0 - i = A - i; AL 2: explicit cell positions).
// The feature set is a template so the unrolled loop holds no branch.  Also
// returns the tile max (NaN-propagating, 8 independent partial maxima) and the
// largest |scale s_i| (the softcap polynomial's range check).
template <bool CAP, int AL>
__device__ __forceinline__ void pf_transform(const uint32_t* raw, float* x, float scale, float k3, float k5,
                                             float k7, float nslope, float A, float rpf, const int32_t* cpos,
                                             float& mt, float& umax) {
  float mx[8], ub[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) mx[k] = neg_inf(), ub[k] = 0.f;
#pragma unroll
  for (int i = 0; i < kPfCells; ++i) {
    float u = __uint_as_float(raw[i]) * scale;
    if (CAP) {
      ub[i & 7] = fmaxf(ub[i & 7], fabsf(u));
      u = pf_cap_poly(u, k3, k5, k7);
    }
    if (AL == 1) u = fmaf(nslope, fabsf(A - (float)i), u);
    if (AL == 2) u = fmaf(nslope, fabsf(rpf - (float)__ldg(cpos + i)), u);
    x[i] = u;
    mx[i & 7] = fmax_nan(mx[i & 7], u);
  }
  mt = pf_max8(mx);
  umax = fmaxf(fmaxf(fmaxf(ub[0], ub[1]), fmaxf(ub[2], ub[3])), fmaxf(fmaxf(ub[4], ub[5]), fmaxf(ub[6], ub[7])));
}

// The same with the exact softcap outside the polynomial's range (taken
// only when some |scale s_i| of the warp's rows exceeds it).
template <int AL>
__device__ __forceinline__ void pf_transform_exact(const uint32_t* raw, float* x, const PrefillPlan& p, float nslope,
                                                float A, float rpf, const int32_t* cpos, float& mt) {
  float mx[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) mx[k] = neg_inf();
#pragma unroll
  for (int i = 0; i < kPfCells; ++i) {
    float u = pf_softcap(__uint_as_float(raw[i]) * p.lg.scale, p);
    if (AL == 1) u = fmaf(nslope, fabsf(A - (float)i), u);
    if (AL == 2) u = fmaf(nslope, fabsf(rpf - (float)__ldg(cpos + i)), u);
    x[i] = u;
    mx[i & 7] = fmax_nan(mx[i & 7], u);
  }
  mt = pf_max8(mx);
}

// Full tiles whose ALiBi bias is linear in the cell index (every cell of the
// tile at or before every row of the warp, so -slope |row_pos - cell_pos| =
// C + slope i with C = -slope A), or that carry no ALiBi: packed f32x2
// arithmetic, two cells per instruction.  The tile is cut into 16 blocks of 8
// cells; x[i] holds y_i = softcap(scale s_i) + slope (i mod 8), and block m adds
// off_m = C + 8 slope m (added back by the max here and by the exponent
// later), which keeps the per-cell ramp to four register pairs.  The softcap
// is the odd Taylor polynomial through u^9 in the raw dot product s:
//   softcap(scale s) = s (scale + w (a3 + w (a5 + w (a7 + w a9)))),  w = s^2.
// CAPM: 0 no softcap; 1 softcap with a per-cell range check (returns the
// largest |s| in smax); 2 softcap on a tile whose range the caller has
// bounded (|s| <= |q| |k| <= s_lim).  Returns the tile max (NaN-propagating).
template <int CAPM, bool ALIBI>
__device__ __forceinline__ void pf_transform_fast(const uint32_t* raw, float* x, const PrefillPlan& p, float slope,
                                                  float C, float& mt, float& smax) {
  const float2 A9 = f2(p.a9), A7 = f2(p.a7), A5 = f2(p.a5), A3 = f2(p.a3), SC = f2(p.lg.scale);
  float2 R[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) R[q] = ALIBI ? f2(slope * (float)(2 * q), slope * (float)(2 * q + 1)) : f2(0.f);
  float sm[2] = {0.f, 0.f};
  float tmax = neg_inf();
#pragma unroll
  for (int mb = 0; mb < kPfCells / 8; ++mb) {
    float bm = neg_inf();
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = mb * 8 + 2 * q;
      const float2 sv = f2(__uint_as_float(raw[i]), __uint_as_float(raw[i + 1]));
      float2 y;
      if (CAPM > 0) {
        if (CAPM == 1) sm[q & 1] = fmax3(sm[q & 1], fabsf(sv.x), fabsf(sv.y));
        const float2 w = mul2(sv, sv);
        float2 h = fma2(w, A9, A7);
        h = fma2(w, h, A5);
        h = fma2(w, h, A3);
        const float2 t = fma2(w, h, SC);
        y = ALIBI ? fma2(sv, t, R[q]) : mul2(sv, t);
      } else {
        y = ALIBI ? fma2(sv, SC, R[q]) : mul2(sv, SC);
      }
      x[i] = y.x;
      x[i + 1] = y.y;
      bm = fmax3_nan(bm, y.x, y.y);
    }
    const float off = ALIBI ? fmaf(8.f * slope, (float)mb, C) : 0.f;
    tmax = fmax_nan(tmax, bm + off);
  }
  mt = tmax;
  smax = fmaxf(sm[0], sm[1]);
}

// Bits tiles on the packed path: cells whose visibility bit is clear become
// -inf (whatever their logit, NaN included), and the tile max is taken again
// over the visible cells, block offsets included.
__device__ __forceinline__ void pf_apply_bits(float* x, const uint32_t* vis, float boff, float bstep, float& mt) {
  float tmax = neg_inf();
#pragma unroll
  for (int mb = 0; mb < kPfCells / 8; ++mb) {
    const uint32_t w = vis[mb >> 2] >> ((mb & 3) * 8);
    float bm = neg_inf();
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      const int i = mb * 8 + e;
      x[i] = ((w >> e) & 1u) ? x[i] : neg_inf();
      x[i + 1] = ((w >> (e + 1)) & 1u) ? x[i + 1] : neg_inf();
      bm = fmax3_nan(bm, x[i], x[i + 1]);
    }
    tmax = fmax_nan(tmax, bm + fmaf(bstep, (float)mb, boff));
  }
  mt = tmax;
}

// Mixed tiles: per-cell visibility (range, sequence, causal, mask != -inf)
// and the mask bias; excluded cells become -inf and lose their bit in vis.
// With explicit cell positions the ALiBi term is added here (the transform
// skipped it: it may not read cell_pos past the cache end).
__device__ __forceinline__ void pf_visibility(float* x, uint32_t* vis, const PrefillPlan& p, const RowVis& rv,
                                           bool rvalid, int c0, const float* mrow, bool mask_vec, bool alibi_pos,
                                           float nslope, float& mt) {
  float mx[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) mx[k] = neg_inf();
  const bool whole = c0 + kPfCells <= p.N;
  float4 mv4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int i = 0; i < kPfCells; ++i) {
    const int c = c0 + i;
    const bool cin = c < p.N;
    bool vc = rvalid && cin && c >= rv.rb && c < rv.re;
    if (p.f.cell_seq) vc = vc && cin && __ldg(p.f.cell_seq + c) == rv.rs;
    int32_t cp = c - rv.rb;
    if (p.f.cell_pos && cin) cp = __ldg(p.f.cell_pos + c);
    if (p.f.causal) vc = vc && cp <= rv.rp;
    float mv = 0.f;
    if (mrow) {
      if (mask_vec && whole) {
        if ((i & 3) == 0) mv4 = __ldg(reinterpret_cast<const float4*>(mrow + c));
        mv = (i & 3) == 0 ? mv4.x : (i & 3) == 1 ? mv4.y : (i & 3) == 2 ? mv4.z : mv4.w;
      } else if (cin) {
        mv = __ldg(mrow + c);
      }
      vc = vc && !(mv == neg_inf());
    }
    float u = x[i];
    if (alibi_pos) u = fmaf(nslope, fabsf((float)(rv.rp - cp)), u);
    u += mv;
    u = vc ? u : neg_inf();
    if (!vc) vis[i >> 5] &= ~(1u << (i & 31));
    x[i] = u;
    mx[i & 7] = fmax_nan(mx[i & 7], u);
  }
  mt = pf_max8(mx);
}

template <typename KT>
__device__ __forceinline__ uint32_t pf_pack(float lo, float hi) {
  if constexpr (Storage<KT>::kDtype == ATTN_BF16) {
    __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&b);
  } else {
    __half2 b = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&b);
  }
}

template <typename KT>
__device__ __forceinline__ float pf_widen(uint16_t bits) {
  if constexpr (Storage<KT>::kDtype == ATTN_BF16) return __uint_as_float((uint32_t)bits << 16);
  else return __half2float(__ushort_as_half(bits));
}

// 32 consecutive output values of one (row, head) starting at element `i0`.
__device__ __forceinline__ void pf_store32(const OutSpec& o, int64_t i0, const float* v, bool vec) {
  if (vec && o.type == ATTN_F32) {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(o.out) + i0);
#pragma unroll
    for (int k = 0; k < 8; ++k) dst[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
  } else if (vec) {
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(o.out) + i0);
    const bool bf = o.type == ATTN_BF16;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        w[e] = bf ? pf_pack<__nv_bfloat16>(v[8 * k + 2 * e], v[8 * k + 2 * e + 1])
                  : pf_pack<__half>(v[8 * k + 2 * e], v[8 * k + 2 * e + 1]);
      dst[k] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e) store_from_float(o.out, i0 + e, o.type, v[e]);
  }
}

// Bound path (bf16 P only): one pass from the raw dot products of one
// thread's row of a full or bits tile to P.  The caller has bounded every
// logit of the tile by |scale| |q| max|k| plus the ALiBi ramp's largest value
// and moved the running max m to that bound when it grew by more than ln 256,
// so no per-cell max is needed (the weights stay <= 256; m only serves as the
// common reference of l and O, and bf16 keeps the full float exponent range
// for weights far below 1).  With log2(e) folded into the constants:
//   a_i = s_i (bsc + w (b3 + w (b5 + w (b7 [+ w b9])))) + L (ramp_i - m),  w = s_i^2,
// the softcap's odd series through u^DEG (DEG 0: no softcap), then
// p_i = 2^a_i.  The ramp is L (C + slope i - m) = rbase + (8 mb) ls + rq[i % 8]
// for block mb of 8 cells (one rounding per block, none carried along the
// row).  Cells whose bit in vis is clear (bits tiles) get p = 0.  Returns the
// sum of the p_i.
template <int DEG, bool ALIBI, bool BITS>
__device__ __forceinline__ float pf_tile_bound(const uint32_t* raw, uint32_t* pk, const PrefillPlan& p, float ls,
                                               float rbase, const uint32_t* vis) {
  const float2 B9 = f2(p.b9), B7 = f2(p.b7), B5 = f2(p.b5), B3 = f2(p.b3), BS = f2(p.bsc);
  float2 RQ[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) RQ[k] = ALIBI ? f2(ls * (float)(2 * k), ls * (float)(2 * k + 1)) : f2(0.f);
  float2 acc[4] = {f2(0.f), f2(0.f), f2(0.f), f2(0.f)};
#pragma unroll
  for (int mb = 0; mb < kPfCells / 8; ++mb) {
    const float2 RB = f2(ALIBI ? fmaf(8.f * ls, (float)mb, rbase) : rbase);
    const uint32_t vw = BITS ? (vis[mb >> 2] >> ((mb & 3) * 8)) : 0xffu;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = mb * 8 + 2 * k;
      const float2 sv = f2(__uint_as_float(raw[i]), __uint_as_float(raw[i + 1]));
      float2 t = BS;
      if (DEG > 0) {
        const float2 w = mul2(sv, sv);
        float2 h = DEG == 9 ? fma2(w, fma2(w, fma2(w, B9, B7), B5), B3) : fma2(w, fma2(w, B7, B5), B3);
        t = fma2(w, h, BS);
      }
      float2 a = fma2(sv, t, ALIBI ? add2(RB, RQ[k]) : RB);
      if (BITS) {
        a.x = ((vw >> (2 * k)) & 1u) ? a.x : neg_inf();
        a.y = ((vw >> (2 * k + 1)) & 1u) ? a.y : neg_inf();
      }
      const float p0 = ex2(a.x), p1 = ex2(a.y);
      acc[k] = add2(acc[k], f2(p0, p1));
      pk[i / 2] = pf_pack<__nv_bfloat16>(p0, p1);
    }
  }
  const float2 s = add2(add2(acc[0], acc[1]), add2(acc[2], acc[3]));
  return s.x + s.y;
}

// Lazy rescaling of the running state (m, l) by the tile max mt, then the
// weights p_i = 2^((x_i + off_m) log2 e - m log2 e) of one row of a tile, their
// sum into l, and P packed to 16 bits.  Block m of 8 cells adds the offset
// off_m = boff + bstep m (nonzero on the fast ALiBi path only), folded into
// one exponent bias per block.  The max is only raised when it grows by more
// than ln 256, so the weights stay below 256 and O is rescaled rarely.
template <typename KT>
__device__ __forceinline__ void pf_weights(const float* x, float boff, float bstep, float mt, float& m, float& l,
                                           float& mneg2, uint32_t* pk, bool& need, float& factor) {
  constexpr float kLazy = 5.545177444479562f;   // ln 256
  need = !(mt <= m + kLazy);   // NaN compares false: a NaN max always rescales
  factor = 1.f;
  if (need) {
    const float mn = fmax_nan(m, mt);
    factor = ex2((m - mn) * kLog2e);        // 0 when m was -inf
    l *= factor;
    m = mn;
    mneg2 = (m == neg_inf()) ? 0.f : -m * kLog2e;
  }
  float2 ls[4] = {f2(0.f), f2(0.f), f2(0.f), f2(0.f)};
  const float2 L2E = f2(kLog2e);
#pragma unroll
  for (int mb = 0; mb < kPfCells / 8; ++mb) {
    const float2 E = f2(fmaf(fmaf(bstep, (float)mb, boff), kLog2e, mneg2));
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = mb * 8 + 2 * q;
      const float2 a = fma2(f2(x[i], x[i + 1]), L2E, E);
      const float p0 = ex2(a.x), p1 = ex2(a.y);
      ls[q] = add2(ls[q], f2(p0, p1));
      pk[i / 2] = pf_pack<KT>(p0, p1);
    }
  }
  const float2 s4 = add2(add2(ls[0], ls[1]), add2(ls[2], ls[3]));
  l += s4.x + s4.y;
}

// P V on the CUDA cores for one thread's row of a tile whose V holds a
// non-finite value: o[0..D) (+)= sum over the row's visible cells c of
// P[c] V[c] (P 16-bit, two per word of pk; V in shared memory, 128-byte
// swizzled 64-column boxes), so that a cell the row cannot see never reaches
// it through 0 * NaN.  The cell loop is unrolled so that pk stays in registers.
template <typename KT, int D>
__device__ __forceinline__ void pf_pv_cuda_cores(const uint32_t* pk, const uint32_t* vis,
                                                 const unsigned char* Vs, uint32_t tO, bool first,
                                                 float factor) {
  using L = PfLayout<D>;
#pragma unroll 1
  for (int ch = 0; ch < D / 32; ++ch) {
    float o[32];
    uint32_t ou[32];
    if (!first) {
      tmem_ld32(tO + ch * 32, ou);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = __uint_as_float(ou[e]) * factor;
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = 0.f;
    }
#pragma unroll
    for (int c = 0; c < kPfCells; ++c) {
      if (!((vis[c >> 5] >> (c & 31)) & 1u)) continue;
      const uint32_t w = pk[c >> 1];
      const float pc = pf_widen<KT>((uint16_t)((c & 1) ? (w >> 16) : (w & 0xffffu)));
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8) {
        const int d = ch * 32 + q8 * 8;
        const uint32_t voff = (uint32_t)(d >> 6) * L::BOX + (uint32_t)c * 128u +
                              ((uint32_t)(((d & 63) >> 3) ^ (c & 7)) << 4);
        float vf[8];
        unpack_vec<KT>(*reinterpret_cast<const uint4*>(Vs + voff), vf);
#pragma unroll
        for (int e = 0; e < 8; ++e) o[q8 * 8 + e] = fmaf(pc, vf[e], o[q8 * 8 + e]);
      }
    }
#pragma unroll
    for (int e = 0; e < 32; ++e) ou[e] = __float_as_uint(o[e]);
    tmem_st32(tO + ch * 32, ou);
    tmem_wait_st();
  }
}

// A CTA's share of a split unit: part `part` of nparts; su = the unit's index
// among the split units (negative for a whole unit).
struct PfSplit {
  int nparts, part;
  int64_t su;
};

// The end of a part of a split unit, for one thread's row (kept out of line:
// it runs once per CTA and would otherwise crowd the softmax loop's
// registers; every lane of the warp calls it): store this row's (m, l, O),
// and let the last part to finish (one counter per row) fold all parts in
// part order with the sink.  Stores before the counter, the counter before
// the loads.
template <int D>
__device__ __noinline__ void pf_split_epilogue(const PrefillPlan& p, const PfSplit& split, uint32_t tO, bool has_o,
                                               float m, float l, bool rvalid, int r, int h, int slot, int row_t,
                                               bool out_vec) {
  constexpr int HPC = PfLayout<D>::HPC;
  auto rec = [&](int prt) { return ((split.su * split.nparts + prt) * HPC + slot) * kPfRows + row_t; };
  float* o = p.part_o + rec(split.part) * D;
#pragma unroll
  for (int ch = 0; ch < D / 32; ++ch) {
    uint32_t ou[32];
    if (has_o) {   // every lane of the warp reads tensor memory (.sync.aligned)
      tmem_ld32(tO + ch * 32, ou);
      tmem_wait_ld();
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) ou[e] = 0u;
    }
    if (rvalid) {
      float4* dst = reinterpret_cast<float4*>(o + ch * 32);
#pragma unroll
      for (int k4 = 0; k4 < 8; ++k4)
        dst[k4] = make_float4(__uint_as_float(ou[4 * k4]), __uint_as_float(ou[4 * k4 + 1]),
                              __uint_as_float(ou[4 * k4 + 2]), __uint_as_float(ou[4 * k4 + 3]));
    }
  }
  if (!rvalid) return;
  p.part_ml[rec(split.part) * 2] = m;
  p.part_ml[rec(split.part) * 2 + 1] = l;
  __threadfence();
  int* cnt = p.split_cnt + (split.su * 2 + slot) * kPfRows + row_t;
  if (atomicAdd(cnt, 1) != split.nparts - 1) return;   // not the last part
  *cnt = 0;                                              // ready for the next call
  __threadfence();
  const float sigma = p.lg.sinks ? __ldg(p.lg.sinks + h) : neg_inf();
  float Mf = sigma;
  for (int q = 0; q < split.nparts; ++q) Mf = fmax_nan(Mf, __ldcg(p.part_ml + rec(q) * 2));
  const bool is_nan = isnan(Mf), is_zero = (Mf == neg_inf());
  // weight of part q's O: e^(m_q - M) (0 for an empty part)
  auto weight = [&](int q) {
    return (is_nan || is_zero) ? 0.f : ex2((__ldcg(p.part_ml + rec(q) * 2) - Mf) * kLog2e);
  };
  float Lf = is_nan || is_zero ? 1.f : ex2((sigma - Mf) * kLog2e);
  for (int q = 0; q < split.nparts; ++q) Lf = fmaf(__ldcg(p.part_ml + rec(q) * 2 + 1), weight(q), Lf);
  const float inv = 1.f / Lf;
  const int64_t ob = (int64_t)r * p.out.sr + (int64_t)h * p.out.sh;
#pragma unroll 1
  for (int ch = 0; ch < D / 32; ++ch) {
    float v[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) v[e] = 0.f;
    for (int q = 0; q < split.nparts; ++q) {
      const float wgt = weight(q);
      const float4* src = reinterpret_cast<const float4*>(p.part_o + rec(q) * D + ch * 32);
#pragma unroll
      for (int k4 = 0; k4 < 8; ++k4) {
        const float4 x = __ldcg(src + k4);
        v[4 * k4] = fmaf(x.x, wgt, v[4 * k4]);
        v[4 * k4 + 1] = fmaf(x.y, wgt, v[4 * k4 + 1]);
        v[4 * k4 + 2] = fmaf(x.z, wgt, v[4 * k4 + 2]);
        v[4 * k4 + 3] = fmaf(x.w, wgt, v[4 * k4 + 3]);
      }
    }
#pragma unroll
    for (int e = 0; e < 32; ++e) v[e] = is_nan ? qnan() : (is_zero ? 0.f : v[e] * inv);
    pf_store32(p.out, ob + ch * 32, v, out_vec);
  }
}

template <typename KT, int D, bool PK>
__device__ __forceinline__ void pf_softmax(const PrefillPlan& p, const PfTiles& tiles, unsigned char* sm,
                                           const PfBars& B, volatile int* abort_flag, uint32_t tmem, int rt,
                                           int h, int slot, int quarter, int lane, const PfSplit& split) {
  // (h: this slot's q head; with packed rows, the KV group's first head)
  const bool out_vec = p.out_vec != 0, mask_vec = p.mask_vec != 0;
  using L = PfLayout<D>;
  uint64_t* s_full = B.s_full;
  uint64_t* p_full = B.p_full;
  // Bounded-wait test: wait on a barrier nothing arrives at; the wait gives
  // up after p.wait_ns, records the timeout and raises the abort flag, and
  // every role of the CTA then winds down.
  if (p.test_stall) {
    if (!pf_wait_warp(B.stall, 0u, p, abort_flag)) return;
  }
  const int row_t = quarter * 32 + lane;
  // packed rows: lane row_t holds row row_t / pack of the tile, head
  // h + row_t % pack (h is then the KV group's first head)
  // (PK: the launch has packed rows; the unpacked kernel compiles without them)
  const int pack = PK ? p.pack : 1, rpt = PK ? p.rpt : kPfRows;
  const int row_l = PK ? row_t / pack : row_t;
  if (PK) h += row_t % pack;
  const int r = rt * rpt + row_l;
  const bool rvalid = (!PK || row_t < pack * rpt) && r < p.R;
  const RowVis rv = rvalid ? row_vis(p.f, r, p.N) : RowVis{0, 0, 0, 0};
  const bool alibi = p.lg.slopes != nullptr;
  const float nslope = alibi ? -__ldg(p.lg.slopes + h) : 0.f;
  const float scale = p.lg.scale;
  const bool cap = p.lg.softcap > 0.f;
  const int al = !alibi ? 0 : (p.f.cell_pos ? 2 : 1);   // ALiBi: off, affine, explicit cell positions
  const float rpf = (float)rv.rp;
  const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
  const uint32_t tS = lane_base + (uint32_t)slot * 128u;
  const uint32_t tO = lane_base + 256u + (uint32_t)slot * D;
  const float* mrow = (p.f.mask && rvalid) ? p.f.mask + (int64_t)r * p.f.mask_sr : nullptr;

  float m = neg_inf(), l = 0.f, mneg2 = 0.f;    // mneg2 = -m * log2(e) (0 while m = -inf)
  int j = 0;
  bool ok = true;
  float qn2 = 0.f;   // |q_r|^2 of this row and head (softcap range bound)
  for (int kt = tiles.first(); kt >= 0; kt = tiles.next(kt), ++j) {
    // the tile's class, K-tile norm and this row's visibility bits are read
    // before the wait for S, so their latency overlaps it
    const int code = tiles.code(kt);
    const bool bits_tile = tiles.bits(kt);
    const float kn2_t = p.kn2 ? __ldg(p.kn2 + (int64_t)kt * p.Hkv + tiles.g) : 0.f;
    const uint4 bw = (bits_tile && rvalid) ? __ldg(reinterpret_cast<const uint4*>(
                                                 p.bits + ((((int64_t)rt * p.n_kt + kt) * kPfRows + row_l) << 2)))
                                           : make_uint4(0u, 0u, 0u, 0u);
    if (!pf_wait_warp(&s_full[slot], (uint32_t)(j & 1), p, abort_flag)) { ok = false; break; }
    tc_fence_after();
    if (j == 0 && p.kn2) {
      // the Q tile is resident (its load completed before the first S)
      if (!pf_wait_warp(B.q_full, 0u, p, abort_flag)) { ok = false; break; }
      const unsigned char* Qs = sm + L::OFF_Q + slot * L::TILE;
      float a = 0.f, b = 0.f;
#pragma unroll
      for (int k8 = 0; k8 < D / 8; ++k8) {
        const uint32_t off = (uint32_t)(k8 >> 3) * L::BOX + (uint32_t)row_t * 128u +
                             ((uint32_t)((k8 & 7) ^ (row_t & 7)) << 4);
        float v[8];
        unpack_vec<KT>(*reinterpret_cast<const uint4*>(Qs + off), v);
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          a = fmaf(v[e], v[e], a);
          b = fmaf(v[e + 1], v[e + 1], b);
        }
      }
      qn2 = a + b;
    }
    uint32_t vis[4] = {~0u, ~0u, ~0u, ~0u};
    uint32_t pk[kPfCells / 2];   // P of this row, packed to 16 bits
    bool need;                    // the running max grew: O needs rescaling
    float factor;                 // ... by this factor
    const int c0 = kt * kPfCells;
    const float A = (float)(rv.rp + rv.rb - c0);
    // Packed fast path: a full or bits tile with no ALiBi, or with affine
    // positions and no visible cell after its row (see pf_transform_fast).
    // Each path below reads S, computes the logits and then the weights on
    // its own, so only P crosses the join (it keeps register use low).
    bool fast = (code == kTileFull || bits_tile) && (!cap || p.cap_raw) &&
                (al == 0 || (al == 1 && !tiles.late(kt)));
    bool done = false;
    if constexpr (Storage<KT>::kDtype == ATTN_BF16) {
      if (fast && p.kn2) {
        // Bound path: every row's logits bounded by |scale| |q| max|k| (the
        // softcap never increases |u|) plus the ALiBi ramp at the row's
        // nearest visible cell of the tile; |scale| |q| max|k| <= 30 keeps the
        // bound within 60 of the true max, so visible weights never underflow.
        // The softcap series of degree 7 where |u| <= c / 3 for every row of
        // the warp (truncation below 1e-6 c), degree 9 where |u| <= 0.4 c
        // (below 3.7e-7 c).
        const float qk2 = qn2 * kn2_t;
        int deg = -1;
        if (cap) deg = __all_sync(0xffffffffu, qk2 <= p.bound7) ? 7 : __all_sync(0xffffffffu, qk2 <= p.bound9) ? 9 : -1;
        else deg = __all_sync(0xffffffffu, qk2 <= p.nc_lim2) ? 0 : -1;
        if (deg >= 0) {
          uint32_t raw[kPfCells];
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) tmem_ld32(tS + c4 * 32, raw + c4 * 32);
          // visible cells of this row in the tile: all (full) or the stored bits
          int i_lo = 0, i_hi = kPfCells - 1;
          if (bits_tile) {
            vis[0] = bw.x; vis[1] = bw.y; vis[2] = bw.z; vis[3] = bw.w;
            i_hi = vis[3] ? 96 + 31 - __clz(vis[3]) : vis[2] ? 64 + 31 - __clz(vis[2])
                 : vis[1] ? 32 + 31 - __clz(vis[1]) : vis[0] ? 31 - __clz(vis[0]) : -1;
            i_lo = vis[0] ? __ffs(vis[0]) - 1 : vis[1] ? 32 + __ffs(vis[1]) - 1
                 : vis[2] ? 64 + __ffs(vis[2]) - 1 : vis[3] ? 96 + __ffs(vis[3]) - 1 : -1;
          }
          const float slope = -nslope, C = nslope * A;
          // ramp C + slope i over the visible cells: largest at i_hi (slope >= 0) or i_lo
          const float ramp_max = al == 1 ? fmaf(slope >= 0.f ? (float)i_hi : (float)i_lo, slope, C) : 0.f;
          const float Mt = fabsf(scale) * sqrtf(qk2) + ramp_max;
          constexpr float kLazy = 5.545177444479562f;   // ln 256
          // a row that sees no cell of the tile leaves its state alone (a row
          // that never sees a cell keeps m = -inf and is written as +0)
          need = i_hi >= 0 && !(Mt <= m + kLazy);
          factor = 1.f;
          if (need) {
            factor = ex2((m - Mt) * kLog2e);   // 0 when m was -inf
            l *= factor;
            m = Mt;
            mneg2 = -m * kLog2e;
          }
          const float rbase = ((al == 1 ? C : 0.f) - m) * kLog2e, lsl = slope * kLog2e;
          tmem_wait_ld();
          float ts;
          if (al == 1) {
            if (bits_tile) ts = deg == 7 ? pf_tile_bound<7, true, true>(raw, pk, p, lsl, rbase, vis)
                              : deg == 9 ? pf_tile_bound<9, true, true>(raw, pk, p, lsl, rbase, vis)
                                         : pf_tile_bound<0, true, true>(raw, pk, p, lsl, rbase, vis);
            else ts = deg == 7 ? pf_tile_bound<7, true, false>(raw, pk, p, lsl, rbase, vis)
                      : deg == 9 ? pf_tile_bound<9, true, false>(raw, pk, p, lsl, rbase, vis)
                                 : pf_tile_bound<0, true, false>(raw, pk, p, lsl, rbase, vis);
          } else {
            if (bits_tile) ts = deg == 7 ? pf_tile_bound<7, false, true>(raw, pk, p, lsl, rbase, vis)
                              : deg == 9 ? pf_tile_bound<9, false, true>(raw, pk, p, lsl, rbase, vis)
                                         : pf_tile_bound<0, false, true>(raw, pk, p, lsl, rbase, vis);
            else ts = deg == 7 ? pf_tile_bound<7, false, false>(raw, pk, p, lsl, rbase, vis)
                      : deg == 9 ? pf_tile_bound<9, false, false>(raw, pk, p, lsl, rbase, vis)
                                 : pf_tile_bound<0, false, false>(raw, pk, p, lsl, rbase, vis);
          }
          l += i_hi >= 0 ? ts : 0.f;
          done = true;
          fast = false;
        }
      }
    }
    if (fast) {
      uint32_t raw[kPfCells];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) tmem_ld32(tS + c4 * 32, raw + c4 * 32);
      tmem_wait_ld();
      const float slope = -nslope, C = nslope * A;
      float x[kPfCells], mt, smax = 0.f;
      // every row's |q|^2 max |k|^2 within range: no per-cell check
      const bool bounded = cap && p.kn2 != nullptr &&
                           __all_sync(0xffffffffu, qn2 * kn2_t <= p.bound2);
      if (bounded) {
        if (al == 1) pf_transform_fast<2, true>(raw, x, p, slope, C, mt, smax);
        else pf_transform_fast<2, false>(raw, x, p, slope, C, mt, smax);
      } else if (cap) {
        if (al == 1) pf_transform_fast<1, true>(raw, x, p, slope, C, mt, smax);
        else pf_transform_fast<1, false>(raw, x, p, slope, C, mt, smax);
      } else {
        if (al == 1) pf_transform_fast<0, true>(raw, x, p, slope, C, mt, smax);
        else pf_transform_fast<0, false>(raw, x, p, slope, C, mt, smax);
      }
      // outside the polynomial's range: the tile goes to the scalar path
      // below, which reads S from tensor memory again
      if (cap && !bounded && __any_sync(0xffffffffu, !(smax <= p.s_lim))) {
        fast = false;
      } else {
        const float boff = al == 1 ? C : 0.f, bstep = al == 1 ? 8.f * slope : 0.f;
        if (bits_tile) {
          vis[0] = bw.x; vis[1] = bw.y; vis[2] = bw.z; vis[3] = bw.w;
          pf_apply_bits(x, vis, boff, bstep, mt);
        }
        pf_weights<KT>(x, boff, bstep, mt, m, l, mneg2, pk, need, factor);
      }
    }
    if (!fast && !done) {
      const int32_t* cpos = p.f.cell_pos ? p.f.cell_pos + c0 : nullptr;
      // full tiles: ALiBi in the transform; mixed tiles with explicit
      // positions: in the visibility pass (cell_pos may end inside the tile)
      const int al_t = (code == kTileFull || al == 1) ? al : 0;
      uint32_t raw[kPfCells];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) tmem_ld32(tS + c4 * 32, raw + c4 * 32);
      tmem_wait_ld();
      float x[kPfCells], mt, umax = 0.f;
      switch ((cap ? 3 : 0) + al_t) {
        case 0: pf_transform<false, 0>(raw, x, scale, p.k3, p.k5, p.k7, nslope, A, rpf, cpos, mt, umax); break;
        case 1: pf_transform<false, 1>(raw, x, scale, p.k3, p.k5, p.k7, nslope, A, rpf, cpos, mt, umax); break;
        case 2: pf_transform<false, 2>(raw, x, scale, p.k3, p.k5, p.k7, nslope, A, rpf, cpos, mt, umax); break;
        case 3: pf_transform<true, 0>(raw, x, scale, p.k3, p.k5, p.k7, nslope, A, rpf, cpos, mt, umax); break;
        case 4: pf_transform<true, 1>(raw, x, scale, p.k3, p.k5, p.k7, nslope, A, rpf, cpos, mt, umax); break;
        default: pf_transform<true, 2>(raw, x, scale, p.k3, p.k5, p.k7, nslope, A, rpf, cpos, mt, umax); break;
      }
      if (cap && __any_sync(0xffffffffu, !(umax <= p.cap_lim))) {
        // some logit outside the polynomial's range: redo the row from S
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) tmem_ld32(tS + c4 * 32, raw + c4 * 32);
        tmem_wait_ld();
        if (al_t == 0) pf_transform_exact<0>(raw, x, p, nslope, A, rpf, cpos, mt);
        else if (al_t == 1) pf_transform_exact<1>(raw, x, p, nslope, A, rpf, cpos, mt);
        else pf_transform_exact<2>(raw, x, p, nslope, A, rpf, cpos, mt);
      }
      if (code != kTileFull) pf_visibility(x, vis, p, rv, rvalid, c0, mrow, mask_vec, al == 2, nslope, mt);
      pf_weights<KT>(x, 0.f, 0.f, mt, m, l, mneg2, pk, need, factor);
    }

    // P V of the previous tile is complete: the tensor core issued it before
    // this tile's S, and S's completion covers every MMA issued before it.
    if (j > 0 && code != kTileMixedBadV && __any_sync(0xffffffffu, need)) {
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t o[32];
        tmem_ld32(tO + ch * 32, o);
        tmem_wait_ld();
        const float2 F = f2(factor);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float2 v = mul2(f2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), F);
          o[e] = __float_as_uint(v.x);
          o[e + 1] = __float_as_uint(v.y);
        }
        tmem_st32(tO + ch * 32, o);
        tmem_wait_st();
      }
    }

    if (code == kTileMixedBadV) {
      // P V on the CUDA cores over this row's visible cells only (V(j) is
      // released by the tensor core's commit after this head's p_full).
      const int stV = pf_stage<L::NV>(j);
      if (!pf_wait_warp(&B.v_full[stV], pf_phase<L::NV>(j), p, abort_flag)) { ok = false; break; }
      pf_pv_cuda_cores<KT, D>(pk, vis, sm + L::OFF_V + stV * L::TILE, tO, j == 0, factor);
    } else {
      // P into the first 64 columns of this head's S region (S is read)
      tmem_st32(tS, pk);
      tmem_st32(tS + 32, pk + 32);
      tmem_wait_st();
    }
    tc_fence_before();
    mbar_arrive(&p_full[slot]);
  }

  if (!ok) return;
  if (j > 0) {
    // the last P V of this head: a barrier with one phase per launch, so the
    // wait is exact (a parity wait on a barrier that completed a phase per
    // tile and was never waited for before could pass early)
    if (!pf_wait_warp(&B.pv_last[slot], 0u, p, abort_flag)) return;
    tc_fence_after();
  }
  if (split.nparts > 1) {
    pf_split_epilogue<D>(p, split, tO, j > 0, m, l, rvalid, r, h, slot, row_t, out_vec);
    return;
  }
  // Fold with the sink (an extra logit with no value vector) and normalise.
  const float sigma = p.lg.sinks ? __ldg(p.lg.sinks + h) : neg_inf();
  const float Mf = fmax_nan(m, sigma);
  const bool is_nan = isnan(Mf), is_zero = (Mf == neg_inf());
  float f = 0.f;
  if (!is_nan && !is_zero) {
    const float fo = ex2((m - Mf) * kLog2e);
    const float Lf = l * fo + ex2((sigma - Mf) * kLog2e);
    f = fo / Lf;
  }
  const int64_t ob = rvalid ? (int64_t)r * p.out.sr + (int64_t)h * p.out.sh : 0;
#pragma unroll
  for (int ch = 0; ch < D / 32; ++ch) {
    uint32_t ou[32];
    if (j > 0) {
      tmem_ld32(tO + ch * 32, ou);
      tmem_wait_ld();
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) ou[e] = 0u;
    }
    float v[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) v[e] = is_nan ? qnan() : (is_zero ? 0.f : __uint_as_float(ou[e]) * f);
    if (rvalid) pf_store32(p.out, ob + ch * 32, v, out_vec);
  }
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------

// One CTA per (row tile, KV head g, pair of q heads of g).  Heavier row tiles
// (later rows see more cells under causality) are launched first.
template <typename KT, int D, bool PK>
__global__ void __launch_bounds__(PfLayout<D>::THREADS, 1)
prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const PrefillPlan p) {
  using L = PfLayout<D>;
  constexpr int NK = L::NK, NV = L::NV;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = pf_align1024(smem_raw);
  const PfBars B = pf_bars<D>(sm);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // work unit (row tile, KV head, q head pair) and, for a split unit, the part
  int64_t unit = blockIdx.x;
  int part = 0, nparts = 1;
  if (unit >= p.n_full) {
    const int64_t q = unit - p.n_full;
    unit = p.n_full + q / p.k_split;
    part = (int)(q % p.k_split);
    nparts = p.k_split;
  }
  const int per_rt = p.Hkv * p.n_pairs;
  const int rt = p.n_rt - 1 - (int)(unit / per_rt);
  const int g = (int)(unit % per_rt) / p.n_pairs;
  const int pair = (int)(unit % per_rt) % p.n_pairs;
  const int h0 = g * p.G + L::HPC * pair;
  // packed rows: one slot holding all of the group's heads
  const int n_slots = PK ? 1 : min(L::HPC, p.G - L::HPC * pair);
  const int rpt = PK ? p.rpt : kPfRows;
  // bytes of a slot's Q tile as loaded: rpt rows x pack heads x D
  const uint32_t q_bytes = PK ? (uint32_t)(p.rpt * p.pack) * (uint32_t)(D * 2) : (uint32_t)L::TILE;

  if (threadIdx.x == 0) {
    mbar_init(B.q_full, 1);
    for (int s = 0; s < NK; ++s) { mbar_init(&B.k_full[s], 1); mbar_init(&B.k_empty[s], 1); }
    for (int s = 0; s < NV; ++s) { mbar_init(&B.v_full[s], 1); mbar_init(&B.v_empty[s], 1); }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&B.s_full[s], 1);
      mbar_init(&B.p_full[s], kPfRows);
      mbar_init(&B.pv_last[s], 1);
    }
    mbar_init(B.mma_done, 1);
    mbar_init(B.stall, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, L::TMEM_COLS);
  if (PK && p.pack * p.rpt < kPfRows) {
    // packed rows that leave lanes unused: zero those rows of the Q tile
    // (its load writes the others), so the unused lanes of S stay finite
    const int used = p.pack * p.rpt;
    for (int i = threadIdx.x; i < (kPfRows - used) * (D / 8); i += L::THREADS) {
      const int row = used + i % (kPfRows - used), chunk = i / (kPfRows - used);   // chunk: 16 bytes of D
      *reinterpret_cast<uint4*>(sm + L::OFF_Q + (chunk >> 3) * L::BOX + row * 128 + (chunk & 7) * 16) =
          make_uint4(0u, 0u, 0u, 0u);
    }
    fence_async_smem();   // visible to the tensor core
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait_prior_grid();   // tile classes from the classifier

  PfTiles tiles{p.cls + (int64_t)rt * p.n_kt, p.vbad, p.n_kt, p.Hkv, g, -1, -1};
  {
    // This CTA's tiles in walk order (nearest first): all of the row tile's
    // non-skipped tiles, or part `part` of nparts equal runs of them.  Every
    // warp finds the same bounds: lane l looks at tile top - l.
    const uint8_t* cls = tiles.cls;
    int cnt = 0;
    for (int base = 0; base < p.n_kt; base += 32) {
      const int kt = base + lane;
      cnt += __popc(__ballot_sync(0xffffffffu, kt < p.n_kt && (cls[kt] & 3) != kTileSkip));
    }
    const int a = (int)((int64_t)part * cnt / nparts), bnd = (int)((int64_t)(part + 1) * cnt / nparts);
    int hi = -1, lo = -1, running = 0;
    for (int top = p.n_kt - 1; top >= 0; top -= 32) {
      const int kt = top - lane;
      const bool ns = kt >= 0 && (cls[kt] & 3) != kTileSkip;
      const uint32_t bal = __ballot_sync(0xffffffffu, ns);
      const int rank = running + __popc(bal & ((1u << lane) - 1u));
      const uint32_t at_a = __ballot_sync(0xffffffffu, ns && rank == a);
      const uint32_t at_b = __ballot_sync(0xffffffffu, ns && rank == bnd);
      if (at_a) hi = top - (__ffs(at_a) - 1);
      if (at_b) lo = top - (__ffs(at_b) - 1);
      running += __popc(bal);
    }
    if (a >= bnd) hi = -1;   // an empty part (fewer tiles than parts)
    tiles.hi = hi;
    tiles.lo = lo;
  }
  const PfSplit split{nparts, part, unit - p.n_full};

  if (warp >= 4) {
    // ---- softmax warpgroups ----
    setmaxnreg_inc<L::HIGH_REGS>();
    const int slot = (warp >> 2) - 1;
    if (slot < n_slots)
      pf_softmax<KT, D, PK>(p, tiles, sm, B, abort_flag, tmem, rt, h0 + slot, slot, warp & 3, lane, split);
  } else {
  setmaxnreg_dec<L::LOW_REGS>();
  if (warp == 0) {
    // ---- TMA producer ----
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();
      int kt = tiles.first();
      // K and V loads issued; the i-th goes to K stage i % NK, V stage i % NV
      int64_t nK = 0, nV = 0;
      const bool any = kt >= 0;
      if (any) {
        mbar_arrive_expect_tx(B.q_full, (uint32_t)n_slots * q_bytes);
        for (int s = 0; s < n_slots; ++s)
#pragma unroll
          for (int bx = 0; bx < D / 64; ++bx)
            tma_load_3d(sm + L::OFF_Q + s * L::TILE + bx * L::BOX, &tmQ, B.q_full, bx * 64, h0 + s, rt * rpt,
                        pol);
      }
      for (; kt >= 0; kt = tiles.next(kt)) {
        // K of this tile once every head's S of the tile NK loads back is done
        const int sk = pf_stage<NK>(nK);
        if (nK >= NK && !pf_wait(&B.k_empty[sk], pf_phase<NK>(nK - NK), p, abort_flag)) break;
        mbar_arrive_expect_tx(&B.k_full[sk], (uint32_t)L::TILE);
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx)
          tma_load_3d(sm + L::OFF_K + sk * L::TILE + bx * L::BOX, &tmK, &B.k_full[sk], bx * 64, g, kt * kPfCells,
                      pol);
        ++nK;
        // V of this tile once every head's P V of the tile NV loads back is done
        const int sv = pf_stage<NV>(nV);
        if (nV >= NV && !pf_wait(&B.v_empty[sv], pf_phase<NV>(nV - NV), p, abort_flag)) break;
        mbar_arrive_expect_tx(&B.v_full[sv], (uint32_t)L::TILE);
#pragma unroll
        for (int bx = 0; bx < D / 64; ++bx)
          tma_load_3d(sm + L::OFF_V + sv * L::TILE + bx * L::BOX, &tmV, &B.v_full[sv], bx * 64, g, kt * kPfCells,
                      pol);
        ++nV;
      }
      // Leave no copy in flight (bounded; completed loads return at once):
      // the last NK K loads and the last NV V loads issued.
      for (int64_t k = nK > NK ? nK - NK : 0; k < nK; ++k)
        mbar_wait_bounded(&B.k_full[pf_stage<NK>(k)], pf_phase<NK>(k), nullptr);
      for (int64_t k = nV > NV ? nV - NV : 0; k < nV; ++k)
        mbar_wait_bounded(&B.v_full[pf_stage<NV>(k)], pf_phase<NV>(k), nullptr);
      if (any) mbar_wait_bounded(B.q_full, 0, nullptr);
    }
  } else if (warp == 1) {
    // ---- MMA issuer ----
    if (lane == 0) {
      constexpr int bf = Storage<KT>::kDtype == ATTN_BF16 ? 1 : 0;
      constexpr uint32_t idS = umma_idesc_f16(kPfRows, kPfCells, bf, 0, 0);
      constexpr uint32_t idO = umma_idesc_f16(kPfRows, D, bf, 0, 1);
      // descriptors of slot 0's Q, stage 0's K (K-major, 128-byte swizzle) and
      // stage 0's V (MN-major); other slots / stages are whole tiles further
      const uint64_t q_desc = umma_desc_sw128(smem_u32(sm + L::OFF_Q), 16, 1024);
      const uint64_t k_desc = umma_desc_sw128(smem_u32(sm + L::OFF_K), 16, 1024);
      const uint64_t v_desc = umma_desc_sw128(smem_u32(sm + L::OFF_V), L::BOX, 1024);
      constexpr uint64_t kTileDesc = (uint64_t)(L::TILE >> 4);
      int kt = tiles.first();
      bool ok = kt >= 0;
      if (ok) {
        ok = pf_wait(B.q_full, 0, p, abort_flag) && pf_wait(&B.k_full[0], 0, p, abort_flag);
        if (ok) {
          tc_fence_after();
          for (int s = 0; s < n_slots; ++s) {
            pf_issue_s<D>(tmem + (uint32_t)s * 128u, q_desc + (uint64_t)s * kTileDesc, k_desc, idS);
            umma_commit(&B.s_full[s]);
          }
          umma_commit(&B.k_empty[0]);
        }
      }
      for (int64_t j = 0; ok && kt >= 0; ++j) {
        const int kn = tiles.next(kt);
        const bool has_next = kn >= 0;
        const bool pv_mma = tiles.code(kt) != kTileMixedBadV;
        const int stV = pf_stage<NV>(j), stK = pf_stage<NK>(j + 1);
        // per head: P V of this tile (P in the head's S columns), then the
        // next tile's S over them
        for (int s = 0; s < n_slots && ok; ++s) {
          if (!pf_wait(&B.p_full[s], (uint32_t)(j & 1), p, abort_flag)) { ok = false; break; }
          if (s == 0 && !pf_wait(&B.v_full[stV], pf_phase<NV>(j), p, abort_flag)) { ok = false; break; }
          tc_fence_after();
          if (pv_mma)
            pf_issue_pv_ts<D>(tmem + 256u + (uint32_t)s * D, tmem + (uint32_t)s * 128u,
                              v_desc + (uint64_t)stV * kTileDesc, idO, j > 0);
          if (!has_next) umma_commit(&B.pv_last[s]);
          if (has_next) {
            if (s == 0 && !pf_wait(&B.k_full[stK], pf_phase<NK>(j + 1), p, abort_flag)) { ok = false; break; }
            tc_fence_after();
            pf_issue_s<D>(tmem + (uint32_t)s * 128u, q_desc + (uint64_t)s * kTileDesc, k_desc + (uint64_t)stK * kTileDesc,
                          idS);
            umma_commit(&B.s_full[s]);
            if (s == n_slots - 1) umma_commit(&B.k_empty[stK]);
          }
        }
        if (!ok) break;
        umma_commit(&B.v_empty[stV]);
        kt = kn;
      }
      umma_commit(B.mma_done);   // arrives once every MMA issued above has retired
    }
  }   // warps 2 and 3 have no role
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    mbar_wait_bounded(B.mma_done, 0, p.status);
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

template <typename KT, int D, bool PK>
cudaError_t launch_prefill_t(const PrefillPlan& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                             const CUtensorMap& tmV, cudaStream_t stream, cudaEvent_t after_classify) {
  using L = PfLayout<D>;
  auto kern = prefill_kernel<KT, D, PK>;
  static std::atomic<unsigned long long> smem_set{0ull};
  cudaError_t e = set_smem_limit_once(smem_set, kern, L::SMEM);
  if (e != cudaSuccess) return e;
  const int64_t n_cls = (int64_t)p.n_rt * p.n_kt, n_scan = (int64_t)p.n_kt * p.Hkv;
  if (n_cls + n_scan > 0) {
    prefill_classify_kernel<<<(unsigned)(n_cls + n_scan), kClsThreads, 0, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  } else if (p.n_split > 0) {
    // no classifier runs (no cells): zero the split units' row counters here
    if ((e = cudaMemsetAsync(p.split_cnt, 0, (size_t)p.n_split * 2 * kPfRows * sizeof(int), stream)) != cudaSuccess)
      return e;
  }
  if (after_classify) cudaEventRecord(after_classify, stream);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.n_full + p.n_split * p.k_split));
  cfg.blockDim = dim3(L::THREADS);
  cfg.dynamicSmemBytes = L::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = after_classify ? 0 : 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tmQ, tmK, tmV, p);
}

}  // namespace

cudaError_t launch_prefill(const PrefillPlan& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                           const CUtensorMap& tmV, cudaStream_t stream, cudaEvent_t after_classify) {
  const bool bf = p.kv_type == ATTN_BF16;
  if (p.D == 64)
    return bf ? (p.pack > 1 ? launch_prefill_t<__nv_bfloat16, 64, true>(p, tmQ, tmK, tmV, stream, after_classify)
                         : launch_prefill_t<__nv_bfloat16, 64, false>(p, tmQ, tmK, tmV, stream, after_classify))
              : (p.pack > 1 ? launch_prefill_t<__half, 64, true>(p, tmQ, tmK, tmV, stream, after_classify)
                         : launch_prefill_t<__half, 64, false>(p, tmQ, tmK, tmV, stream, after_classify));
  if (p.D == 256)
    return bf ? (p.pack > 1 ? launch_prefill_t<__nv_bfloat16, 256, true>(p, tmQ, tmK, tmV, stream, after_classify)
                         : launch_prefill_t<__nv_bfloat16, 256, false>(p, tmQ, tmK, tmV, stream, after_classify))
              : (p.pack > 1 ? launch_prefill_t<__half, 256, true>(p, tmQ, tmK, tmV, stream, after_classify)
                         : launch_prefill_t<__half, 256, false>(p, tmQ, tmK, tmV, stream, after_classify));
  return bf ? (p.pack > 1 ? launch_prefill_t<__nv_bfloat16, 128, true>(p, tmQ, tmK, tmV, stream, after_classify)
                         : launch_prefill_t<__nv_bfloat16, 128, false>(p, tmQ, tmK, tmV, stream, after_classify))
            : (p.pack > 1 ? launch_prefill_t<__half, 128, true>(p, tmQ, tmK, tmV, stream, after_classify)
                         : launch_prefill_t<__half, 128, false>(p, tmQ, tmK, tmV, stream, after_classify));
}

}  // namespace attn
