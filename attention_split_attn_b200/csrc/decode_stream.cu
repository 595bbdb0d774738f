// decode_stream.cu -- balanced persistent split-K decode for 16-bit caches
// (attn_decode with n_slices == 0 and Q in the cache dtype) and for one-byte
// caches (e4m3 / int8 codes with per (cell, KV head) scales, Q in bf16 or
// f16; the tile step of decode_tile8.cuh).
//
// The split-K idea of the pages (TensorFold PR #2595: split each row's keys
// into slices, fold the slice partials afterwards) with slices sized for the
// GPU instead of for the row: flatten every (row, KV head) pair's cells into
// 16-cell tiles, pair after pair, and give each of W resident warps
// (W = SMs x warps per SM) an equal contiguous run of that tile space.  A warp
// streams its run through one TMA ring without restarting at pair
// boundaries, folds it with the tensor-core tile step of decode_tile.cuh, and
// writes one partial record per pair it touches.  Every warp gets the same
// number of tiles (+-1), whatever the mix of row lengths, so no SM idles at
// the end of the launch.
//
// Record slots, with no prefix sums in the combine: the warp in which a pair
// STARTS writes the pair's "home" slot W + pair; any later warp that covers
// part of the pair covers it from the start of its own run, so it writes its
// own slot w (a run can start inside at most one pair).  The combine walks a
// pair's home slot, then the slots of the following warps up to the one that
// holds the pair's last tile, in tile order, so the result is deterministic.
//
// A planner kernel first writes row_tiles[r] (exclusive prefix of each row's
// tile count); the persistent kernel and the combine run behind it with
// programmatic dependent launch.  With at most kInlineRows rows every warp
// computes the prefix itself and no planner runs.
#include "common.cuh"
#include "decode_tile.cuh"
#include "decode_tile8.cuh"
#include "internal.h"
#include "mma.cuh"
#include "quant.cuh"

namespace attn {

namespace {

// Up to this many rows, every warp computes the row tile prefix itself (no
// planner kernel in front of the stream kernel).
constexpr int kInlineRows = 64;

// The tile step of a cache type: decode_tile.cuh for 16-bit values,
// decode_tile8.cuh for one-byte codes; ES bytes per element, so a stage is
// 16 cells x D elements of K then of V, each in D ES / 128 TMA boxes of 128
// bytes per cell.
template <typename KT, int D, int NH>
struct StreamTraits {
  using State = WarpTileState<KT, D, NH>;
  static constexpr int ES = 2;
};
template <int D, int NH>
struct StreamTraits<e4m3_code, D, NH> {
  using State = WarpTileState8<e4m3_code, D, NH>;
  static constexpr int ES = 1;
};
template <int D, int NH>
struct StreamTraits<i8_code, D, NH> {
  using State = WarpTileState8<i8_code, D, NH>;
  static constexpr int ES = 1;
};

template <int D, int ES>
struct StreamRing {
  static constexpr int NS = 2;                       // ring stages per warp
  static constexpr int TILE = kWarpTile * D * ES;    // K (or V) of one tile
  static constexpr int STAGE = 2 * TILE;
  static constexpr int BAR_OFF = NS * STAGE;
  static constexpr int RT_OFF = BAR_OFF + NS * 8;    // inline row tile prefix [kInlineRows + 1]
  static constexpr int TOTAL = RT_OFF + (kInlineRows + 1) * 8 + 1024;   // + alignment slack for the swizzle
};

// TMA of one 16-cell K/V tile of KV head g starting at cell c0 (boxes of 128
// bytes per cell, 128-byte swizzled, each sub-tile 16 x 128 B).
template <int D, int ES>
__device__ __forceinline__ void issue_stream_tile(unsigned char* stage, uint64_t* bar, const CUtensorMap* tmK,
                                                  const CUtensorMap* tmV, int g, int c0, uint64_t pol) {
  constexpr int TILE = kWarpTile * D * ES, NB = D * ES / 128, EPB = 128 / ES;
  mbar_arrive_expect_tx(bar, 2 * TILE);
#pragma unroll
  for (int sub = 0; sub < NB; ++sub) {
    tma_load_3d(stage + sub * (kWarpTile * 128), tmK, bar, sub * EPB, g, c0, pol);
    tma_load_3d(stage + TILE + sub * (kWarpTile * 128), tmV, bar, sub * EPB, g, c0, pol);
  }
}

__device__ __forceinline__ int64_t row_len(const DecodePlan& p, int r) {
  int32_t b = p.f.row_begin ? __ldg(p.f.row_begin + r) : 0;
  int32_t e = p.f.row_end ? __ldg(p.f.row_end + r) : p.N;
  b = max(b, 0);
  e = min(e, p.N);
  return e > b ? (int64_t)e - b : 0;
}

// row_tiles[r] = sum over r' < r of ceil(len_r' / 16); row_tiles[R] = total.
__global__ void __launch_bounds__(1024) decode_plan_kernel(const DecodePlan p) {
  pdl_launch_dependents();
  __shared__ long long wsum[32];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  long long carry = 0;
  for (int base = 0; base < p.R; base += 1024) {
    const int r = base + tid;
    const long long n = r < p.R ? (row_len(p, r) + kWarpTile - 1) / kWarpTile : 0;
    long long x = n;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) wsum[wid] = x;
    __syncthreads();
    if (wid == 0) {
      long long v = wsum[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += y;
      }
      wsum[lane] = v;
    }
    __syncthreads();
    const long long excl = x - n + (wid > 0 ? wsum[wid - 1] : 0);
    if (r < p.R) p.row_tiles[r] = carry + excl;
    carry += wsum[31];
    __syncthreads();
  }
  if (tid == 0) p.row_tiles[p.R] = carry;
}

// Position in the flattened tile space: row r, KV head g, tile j of nt.
struct Cursor {
  int r, g;
  int64_t j, nt;
  int32_t begin, end;        // the row's cell range, clipped to [0, n_cells)
  int32_t raw_b, raw_e;      // row_begin / row_end as given (default positions)
};

__device__ __forceinline__ void cursor_load_row(const DecodePlan& p, const int64_t* row_tiles, Cursor& c) {
  c.nt = row_tiles[c.r + 1] - row_tiles[c.r];
  int32_t b = p.f.row_begin ? __ldg(p.f.row_begin + c.r) : 0;
  int32_t e = p.f.row_end ? __ldg(p.f.row_end + c.r) : p.N;
  c.raw_b = b;
  c.raw_e = e;
  b = max(b, 0);
  e = min(e, p.N);
  c.begin = b;
  c.end = max(e, b);
}

// Move to the next tile; rows without tiles are skipped.
__device__ __forceinline__ void cursor_next(const DecodePlan& p, const int64_t* row_tiles, Cursor& c) {
  if (++c.j < c.nt) return;
  c.j = 0;
  if (++c.g < p.Hkv) return;
  c.g = 0;
  do {
    ++c.r;
    cursor_load_row(p, row_tiles, c);
  } while (c.nt == 0 && c.r + 1 < p.R);
}

// Fused append: when this tile holds the append cell of its (row, KV head)
// (cell row_end - 1), write the row's new K and V into the cache and over the
// staged copy of that cell (the TMA may have read the cell before or after
// the cache write), so the attention of this launch already sees them.  Each
// (row, KV head, tile) belongs to exactly one warp, so each new row is
// written once.  16-byte chunks, one per lane per pass; the staged rows are
// 128-byte swizzled (chunk k of cell row i at chunk k ^ (i & 7)).
template <int D>
__device__ __forceinline__ void append_patch(const DecodePlan& p, const Cursor& c, unsigned char* stage, int lane) {
  const int t0 = c.begin + (int)(c.j * kWarpTile);
  const int a = c.raw_e - 1;   // the append cell (inside [begin, end) whenever the row has cells)
  if (a < t0 || a >= t0 + kWarpTile || a < c.begin || a >= c.end) return;
  const int row = a - t0;
  constexpr int CH = D / 8;    // 16-byte chunks of one cell row of one head
  const int64_t src = (int64_t)c.r * p.new_sr + (int64_t)c.g * p.new_sh;
  const int64_t dst = (int64_t)a * p.kv_sc + (int64_t)c.g * p.kv_sh;
  for (int i = lane; i < 2 * CH; i += 32) {
    const bool is_v = i >= CH;
    const int ch = is_v ? i - CH : i;
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(is_v ? p.v_new : p.k_new) + src) + ch);
    reinterpret_cast<uint4*>(static_cast<uint16_t*>(is_v ? p.v_out : p.k_out) + dst)[ch] = w;
    const int sub = ch >> 3, k = ch & 7;
    const uint32_t off = (is_v ? (uint32_t)(kWarpTile * D * 2) : 0u) + (uint32_t)sub * (kWarpTile * 128) +
                         (uint32_t)row * 128u + ((uint32_t)(k ^ (row & 7)) << 4);
    *reinterpret_cast<uint4*>(stage + off) = w;
  }
  __syncwarp();
}

template <typename KT, int D, int NH>
__global__ void __launch_bounds__(32)
decode_stream_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const DecodePlan p) {
  using Tr = StreamTraits<KT, D, NH>;
  using Ring = StreamRing<D, Tr::ES>;
  constexpr int NS = Ring::NS;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Ring::BAR_OFF);
  const int lane = threadIdx.x;
  if (lane == 0) {
    for (int i = 0; i < NS; ++i) mbar_init(&full[i], 1);
    fence_mbar_init();
  }
  __syncwarp();
  pdl_launch_dependents();
  // The row tile prefix: from the planner, or (few rows) computed here
  // before waiting on the previous kernel in the stream, which may still be
  // reading a workspace this call is about to reuse.
  const int64_t* row_tiles = p.row_tiles;
  if (p.plan_inline) {
    int64_t* rt = reinterpret_cast<int64_t*>(smem + Ring::RT_OFF);
    int64_t carry = 0;
    for (int base = 0; base < p.R; base += 32) {
      const int r = base + lane;
      const int64_t n = r < p.R ? (row_len(p, r) + kWarpTile - 1) / kWarpTile : 0;
      int64_t x = n;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int64_t y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
      }
      if (r < p.R) rt[r] = carry + x - n;
      carry += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) rt[p.R] = carry;
    __syncwarp();
    row_tiles = rt;
  }
  pdl_wait_prior_grid();
  if (p.plan_inline && blockIdx.x == 0) {
    // the combine reads the prefix from the workspace
    for (int r = lane; r <= p.R; r += 32) p.row_tiles[r] = row_tiles[r];
  }

  const int64_t W = p.W, Hkv = p.Hkv;
  const int64_t T = Hkv * row_tiles[p.R];
  const int64_t w = p.grid_order ? W - 1 - blockIdx.x : blockIdx.x;
  const int64_t t0 = T * w / W, t1 = T * (w + 1) / W;
  if (t0 >= t1) return;

  // the row holding tile t0: the last r with Hkv * row_tiles[r] <= t0
  // (32-ary search: each round the lanes probe 32 evenly spaced rows)
  int lo = 0, hi = p.R;   // answer in [lo, hi)
  while (hi - lo > 1) {
    const int64_t span = hi - lo;
    const int64_t step = (span + 31) / 32;
    const int64_t probe = lo + lane * step;
    const bool ok = probe < hi && Hkv * row_tiles[probe] <= t0;
    const unsigned m = __ballot_sync(0xffffffffu, ok);
    const int k = 31 - __clz(m);       // lane 0 always qualifies (row_tiles[lo] <= t0)
    lo = (int)(lo + k * step);
    hi = (int)((int64_t)hi < lo + step ? (int64_t)hi : lo + step);
  }
  Cursor c;
  c.r = lo;
  cursor_load_row(p, row_tiles, c);
  {
    const int64_t off = t0 - Hkv * row_tiles[c.r];
    c.g = (int)(off / c.nt);
    c.j = off % c.nt;
  }
  Cursor ic = c;   // issue cursor (lane 0 runs it NS tiles ahead)
  const int64_t n = t1 - t0;
  uint64_t pol = 0;
  int64_t issued = 0;
  // The issue cursor only advances right before issuing a tile that exists,
  // so it never moves past the last tile of the run.
  if (lane == 0) {
    pol = policy_evict_first();
    for (; issued < (n < NS ? n : (int64_t)NS); ++issued) {
      if (issued > 0) cursor_next(p, row_tiles, ic);
      issue_stream_tile<D, Tr::ES>(smem + issued * Ring::STAGE, &full[issued], &tmK, &tmV, ic.g,
                                   ic.begin + (int)(ic.j * kWarpTile), pol);
    }
  }

  const bool has_filter = (p.f.cell_seq && p.f.row_seq) || p.f.causal || p.f.mask;
  auto make_ctx = [&](const Cursor& cc) {
    RowCtx rc;
    rc.begin = cc.begin;
    rc.end = cc.end;
    rc.pos_base = cc.raw_b;
    rc.s_begin = cc.begin;
    rc.s_end = cc.end;
    rc.row_seq = p.f.row_seq ? __ldg(p.f.row_seq + cc.r) : 0;
    rc.row_pos = p.f.row_pos ? (int64_t)__ldg(p.f.row_pos + cc.r) : (int64_t)cc.raw_e - cc.raw_b - 1;
    return rc;
  };
  RowCtx rc = make_ctx(c);
  typename Tr::State st;
  st.reset();
  st.init_offsets(lane);
  st.load_q(p, c.r, c.g * p.G, lane);

  bool aborted = false;
  int64_t k = 0;
  if constexpr (Tr::ES == 1) st.prefetch(p, c.g, c.begin + (int)(c.j * kWarpTile), lane);
  for (; k < n; ++k) {
    const int stg = (int)(k % NS);
    if constexpr (Tr::ES == 1) {
      st.take_prefetched();
      if (k + 1 < n) {   // the next tile's per-cell scales, a tile ahead
        Cursor nc = c;
        cursor_next(p, row_tiles, nc);
        st.prefetch(p, nc.g, nc.begin + (int)(nc.j * kWarpTile), lane);
      }
    }
    if (!mbar_wait_bounded(&full[stg], (uint32_t)((k / NS) & 1), p.status)) {
      aborted = true;
      break;
    }
    unsigned char* stage = smem + stg * Ring::STAGE;
    if (Tr::ES == 2 && p.k_new) append_patch<D>(p, c, stage, lane);
    st.load_tile(stage);
    auto refill = [&]() {
      __syncwarp();
      if (lane == 0 && issued < n) {
        // the lanes' shared-memory reads of this stage precede its async refill
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        cursor_next(p, row_tiles, ic);
        issue_stream_tile<D, Tr::ES>(stage, &full[stg], &tmK, &tmV, ic.g, ic.begin + (int)(ic.j * kWarpTile), pol);
        ++issued;
      }
    };
    if (decltype(st)::kEarlyRelease) refill();
    st.compute(p, rc, c.r, c.begin + (int)(c.j * kWarpTile), has_filter, lane, stage);
    if (!decltype(st)::kEarlyRelease) refill();
    const bool last = (k + 1 == n);
    if (c.j + 1 == c.nt || last) {
      // the pair ends here (or this warp's run does): emit its record
      st.finish_sums();
      const int64_t pair = (int64_t)c.r * Hkv + c.g;
      const int64_t pair_start = Hkv * row_tiles[c.r] + (int64_t)c.g * c.nt;
      const int64_t slot = pair_start >= t0 ? W + pair : w;
      st.write_partial(p.part.o, p.part.ml, slot, p.G, lane, false);
      if (!last) {
        cursor_next(p, row_tiles, c);
        rc = make_ctx(c);
        st.reset();
        st.load_q(p, c.r, c.g * p.G, lane);
      }
    } else {
      ++c.j;
    }
  }
  if (aborted) {
    // poison the record in progress and leave no copy in flight
    const int64_t pair = (int64_t)c.r * Hkv + c.g;
    const int64_t pair_start = Hkv * row_tiles[c.r] + (int64_t)c.g * c.nt;
    st.write_partial(p.part.o, p.part.ml, pair_start >= t0 ? W + pair : w, p.G, lane, true);
    if (lane == 0)
      for (int64_t kk = k; kk < issued; ++kk) mbar_wait_bounded(&full[kk % NS], (uint32_t)((kk / NS) & 1), nullptr);
    __syncwarp();
  }
}

template <typename KT, int D, int NH>
cudaError_t launch_stream_t(const DecodePlan& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                            cudaStream_t stream, cudaEvent_t after_main) {
  auto kern = decode_stream_kernel<KT, D, NH>;
  using Ring = StreamRing<D, StreamTraits<KT, D, NH>::ES>;
  static std::atomic<unsigned long long> smem_set{0ull};
  cudaError_t e = set_smem_limit_once(smem_set, kern, Ring::TOTAL);
  if (e != cudaSuccess) return e;
  if (!p.plan_inline) {
    decode_plan_kernel<<<1, 1024, 0, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.W);
  cfg.blockDim = dim3(32);
  cfg.dynamicSmemBytes = Ring::TOTAL;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tmK, tmV, p);
  if (e != cudaSuccess) return e;
  if (after_main) cudaEventRecord(after_main, stream);
  return cudaSuccess;
}

template <typename KT>
cudaError_t launch_stream_k(const DecodePlan& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                            cudaStream_t stream, cudaEvent_t ev) {
  const bool h16 = p.G > 8;
  switch (p.D) {
    case 64: return h16 ? launch_stream_t<KT, 64, 16>(p, tmK, tmV, stream, ev)
                        : launch_stream_t<KT, 64, 8>(p, tmK, tmV, stream, ev);
    case 128: return h16 ? launch_stream_t<KT, 128, 16>(p, tmK, tmV, stream, ev)
                         : launch_stream_t<KT, 128, 8>(p, tmK, tmV, stream, ev);
    default: return h16 ? launch_stream_t<KT, 256, 16>(p, tmK, tmV, stream, ev)
                        : launch_stream_t<KT, 256, 8>(p, tmK, tmV, stream, ev);
  }
}

template <typename KT, int D, int NH>
int stream_blocks_per_sm() {
  int n = 0;
  using Ring = StreamRing<D, StreamTraits<KT, D, NH>::ES>;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_stream_kernel<KT, D, NH>, 32, Ring::TOTAL) !=
          cudaSuccess ||
      n <= 0) {
    cudaGetLastError();
    // no device: the shared-memory bound of a 228 KB SM with 1 KB reserved per CTA
    n = (228 * 1024) / (Ring::TOTAL + 1024);
  }
  return n;
}

// ---------------------------------------------------------------------------
// cluster decode: one thread-block cluster per (row, KV head)
// ---------------------------------------------------------------------------
// A latency variant for few, long rows (TensorFold PR #985, change list: a
// cluster of CTAs shares a head over distributed shared memory).  The row's
// 16-cell tiles of one KV head are cut into kClWarps * kClCtas equal runs
// (16 CTAs of 8 warps: one long row's 8 KV heads then cover 128 SMs);
// each warp of each CTA of the cluster folds its run with the tensor-core
// tile step (its own TMA ring, as in the stream kernel) and leaves its
// partial (m, l, O) in its CTA's shared memory; after a cluster barrier CTA
// rank 0 reads all partials over distributed shared memory and folds them in
// (rank, warp) order with the sink -- no workspace, no combine launch.  Both
// cluster barriers are reached on every path (a warp whose bounded wait runs
// out poisons its partial and drains its copies), so no CTA waits forever.
constexpr int kClCtas = 16;   // CTAs per cluster (above the portable 8: opted in at launch)
constexpr int kClWarps = 8;   // warps per CTA

template <int D, int NH>
struct ClusterSmem {
  using Ring = StreamRing<D, 2>;
  static constexpr int RING = Ring::NS * Ring::STAGE;           // one warp's stages
  static constexpr int BARS = kClWarps * RING;                  // [kClWarps][NS] mbarriers
  static constexpr int PART_O = BARS + kClWarps * Ring::NS * 8; // [kClWarps][NH][D] floats
  static constexpr int PART_ML = PART_O + kClWarps * NH * D * 4;  // [kClWarps][NH][2]
  static constexpr int TOTAL = PART_ML + kClWarps * NH * 2 * 4 + 1024;
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_cluster(const void* local, uint32_t rank) {
  uint32_t a = smem_u32(local), ra;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
  return v;
}

template <typename KT, int D, int NH>
__global__ void __launch_bounds__(32 * kClWarps)
decode_cluster_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const DecodePlan p) {
  using Sm = ClusterSmem<D, NH>;
  using Ring = typename Sm::Ring;
  constexpr int NS = Ring::NS;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = align1024(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int unit = blockIdx.x / kClCtas;
  const int r = unit / p.Hkv, g = unit % p.Hkv;
  unsigned char* ring = smem + warp * Sm::RING;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Sm::BARS) + warp * NS;
  float* part_o = reinterpret_cast<float*>(smem + Sm::PART_O);
  float* part_ml = reinterpret_cast<float*>(smem + Sm::PART_ML);
  if (lane == 0) {
    for (int i = 0; i < NS; ++i) mbar_init(&full[i], 1);
    fence_mbar_init();
  }
  __syncwarp();

  // this warp's run of the (row, KV head)'s tiles
  Cursor c;
  c.r = r;
  c.g = g;
  c.raw_b = p.f.row_begin ? __ldg(p.f.row_begin + r) : 0;
  c.raw_e = p.f.row_end ? __ldg(p.f.row_end + r) : p.N;
  c.begin = max(c.raw_b, 0);
  c.end = max(min(c.raw_e, p.N), c.begin);
  const int64_t nt = (c.end - c.begin + kWarpTile - 1) / kWarpTile;
  const int share = (int)rank * kClWarps + warp, n_share = kClCtas * kClWarps;
  const int64_t t0 = nt * share / n_share, t1 = nt * (share + 1) / n_share;
  const int64_t n = t1 - t0;
  uint64_t pol = 0;
  int64_t issued = 0;
  if (lane == 0) {
    pol = policy_evict_first();
    for (; issued < (n < NS ? n : (int64_t)NS); ++issued)
      issue_stream_tile<D, 2>(ring + issued * Ring::STAGE, &full[issued], &tmK, &tmV, g,
                              c.begin + (int)((t0 + issued) * kWarpTile), pol);
  }
  const bool has_filter = (p.f.cell_seq && p.f.row_seq) || p.f.causal || p.f.mask;
  RowCtx rc;
  rc.begin = c.begin;
  rc.end = c.end;
  rc.pos_base = c.raw_b;
  rc.s_begin = c.begin;
  rc.s_end = c.end;
  rc.row_seq = p.f.row_seq ? __ldg(p.f.row_seq + r) : 0;
  rc.row_pos = p.f.row_pos ? (int64_t)__ldg(p.f.row_pos + r) : (int64_t)c.raw_e - c.raw_b - 1;
  WarpTileState<KT, D, NH> st;
  st.reset();
  st.init_offsets(lane);
  st.load_q(p, r, g * p.G, lane);
  bool aborted = false;
  int64_t k = 0;
  for (; k < n; ++k) {
    const int stg = (int)(k % NS);
    if (!mbar_wait_bounded(&full[stg], (uint32_t)((k / NS) & 1), p.status)) {
      aborted = true;
      break;
    }
    unsigned char* stage = ring + stg * Ring::STAGE;
    st.load_tile(stage);
    auto refill = [&]() {
      __syncwarp();
      if (lane == 0 && issued < n) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        issue_stream_tile<D, 2>(stage, &full[stg], &tmK, &tmV, g, c.begin + (int)((t0 + issued) * kWarpTile), pol);
        ++issued;
      }
    };
    if (decltype(st)::kEarlyRelease) refill();
    st.compute(p, rc, r, c.begin + (int)((t0 + k) * kWarpTile), has_filter, lane, stage);
    if (!decltype(st)::kEarlyRelease) refill();
  }
  if (aborted && lane == 0)   // leave no copy in flight
    for (int64_t kk = k; kk < issued; ++kk) mbar_wait_bounded(&full[kk % NS], (uint32_t)((kk / NS) & 1), nullptr);
  st.finish_sums();
  // this warp's partial: [NH][D] and [NH][2] in its slot of the CTA's shared memory
  st.write_partial(part_o + warp * NH * D, part_ml + warp * NH * 2, 0, NH, lane, aborted);
  cluster_sync_all();   // every CTA's partials are in place
  if (rank == 0) {
    // fold the kClCtas x kClWarps partials in (rank, warp) order with the sink:
    // thread t takes head t / 32 (t < 32 G), dims lane, lane + 32, ...
    const int hh = threadIdx.x >> 5;
    for (int h = hh; h < p.G; h += kClWarps) {
      const int hq = g * p.G + h;
      const float sigma = p.lg.sinks ? __ldg(p.lg.sinks + hq) : neg_inf();
      float M = sigma;
      for (int q = 0; q < n_share; ++q) {
        const float mq = ld_cluster(part_ml + ((q % kClWarps) * NH + h) * 2, (uint32_t)(q / kClWarps));
        M = fmax_nan(M, mq);
      }
      const bool is_nan = isnan(M), is_zero = (M == neg_inf());
      float L = (is_nan || is_zero) ? 1.f : ex2((sigma - M) * kLog2e);
      for (int q = 0; q < n_share; ++q) {
        const uint32_t rk = (uint32_t)(q / kClWarps);
        const float* ml = part_ml + ((q % kClWarps) * NH + h) * 2;
        const float mq = ld_cluster(ml, rk);
        const float wq = (is_nan || is_zero) ? 0.f : ex2((mq - M) * kLog2e);
        L = fmaf(ld_cluster(ml + 1, rk), wq, L);
      }
      const int64_t ob = (int64_t)r * p.out.sr + (int64_t)hq * p.out.sh;
      for (int d = lane; d < D; d += 32) {
        float o = 0.f;
        for (int q = 0; q < n_share; ++q) {
          const uint32_t rk = (uint32_t)(q / kClWarps);
          const float mq = ld_cluster(part_ml + ((q % kClWarps) * NH + h) * 2, rk);
          const float wq = (is_nan || is_zero) ? 0.f : ex2((mq - M) * kLog2e);
          o = fmaf(ld_cluster(part_o + ((q % kClWarps) * NH + h) * D + d, rk), wq, o);
        }
        const float v = is_nan ? qnan() : is_zero ? 0.f : o / L;
        store_from_float(p.out.out, ob + d, p.out.type, v);
      }
    }
  }
  cluster_sync_all();   // no CTA leaves while rank 0 may still read its shared memory
}

template <typename KT, int D, int NH>
cudaError_t launch_cluster_t(const DecodePlan& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                             cudaStream_t stream) {
  using Sm = ClusterSmem<D, NH>;
  auto kern = decode_cluster_kernel<KT, D, NH>;
  static std::atomic<unsigned long long> smem_set{0ull};
  cudaError_t e = set_smem_limit_once(smem_set, kern, Sm::TOTAL);
  if (e != cudaSuccess) return e;
  static std::atomic<unsigned long long> np_set{0ull};
  {
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(np_set.load() & bit)) {
      if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1)) != cudaSuccess) return e;
      np_set.fetch_or(bit);
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((int64_t)p.R * p.Hkv * kClCtas));
  cfg.blockDim = dim3(32 * kClWarps);
  cfg.dynamicSmemBytes = Sm::TOTAL;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kClCtas;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tmK, tmV, p);
}

}  // namespace

cudaError_t launch_decode_cluster(const DecodePlan& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                                  cudaStream_t stream) {
  const bool bf = p.kv_type == ATTN_BF16, h16 = p.G > 8;
  switch (p.D) {
    case 64:
      return bf ? (h16 ? launch_cluster_t<__nv_bfloat16, 64, 16>(p, tmK, tmV, stream)
                       : launch_cluster_t<__nv_bfloat16, 64, 8>(p, tmK, tmV, stream))
                : (h16 ? launch_cluster_t<__half, 64, 16>(p, tmK, tmV, stream)
                       : launch_cluster_t<__half, 64, 8>(p, tmK, tmV, stream));
    default:
      return bf ? (h16 ? launch_cluster_t<__nv_bfloat16, 128, 16>(p, tmK, tmV, stream)
                       : launch_cluster_t<__nv_bfloat16, 128, 8>(p, tmK, tmV, stream))
                : (h16 ? launch_cluster_t<__half, 128, 16>(p, tmK, tmV, stream)
                       : launch_cluster_t<__half, 128, 8>(p, tmK, tmV, stream));
  }
}

int decode_stream_warps(int kv_type, int D, int G, int sms) {
  int per_sm;
  const bool h16 = G > 8;
  if (kv_type == ATTN_FP8_E4M3 || kv_type == ATTN_I8) {
    const bool e4 = kv_type == ATTN_FP8_E4M3;
    per_sm = D == 128 ? (e4 ? stream_blocks_per_sm<e4m3_code, 128, 8>() : stream_blocks_per_sm<i8_code, 128, 8>())
                      : (e4 ? stream_blocks_per_sm<e4m3_code, 256, 8>() : stream_blocks_per_sm<i8_code, 256, 8>());
  } else if (kv_type == ATTN_F16) {
    per_sm = D == 64 ? (h16 ? stream_blocks_per_sm<__half, 64, 16>() : stream_blocks_per_sm<__half, 64, 8>())
           : D == 128 ? (h16 ? stream_blocks_per_sm<__half, 128, 16>() : stream_blocks_per_sm<__half, 128, 8>())
                      : (h16 ? stream_blocks_per_sm<__half, 256, 16>() : stream_blocks_per_sm<__half, 256, 8>());
  } else {
    per_sm = D == 64 ? (h16 ? stream_blocks_per_sm<__nv_bfloat16, 64, 16>() : stream_blocks_per_sm<__nv_bfloat16, 64, 8>())
           : D == 128 ? (h16 ? stream_blocks_per_sm<__nv_bfloat16, 128, 16>() : stream_blocks_per_sm<__nv_bfloat16, 128, 8>())
                      : (h16 ? stream_blocks_per_sm<__nv_bfloat16, 256, 16>() : stream_blocks_per_sm<__nv_bfloat16, 256, 8>());
  }
  return std::max(1, per_sm) * std::max(1, sms);
}

bool decode_stream8_supported(int kv_type, int q_type, const void* q, int64_t q_sr, int64_t q_sh, int D, int G) {
  // one-byte caches on the tensor cores: head dim 128 or 256, up to 8 q heads
  // per KV head, Q in bf16 or f16 with 16-byte-aligned rows
  return (kv_type == ATTN_FP8_E4M3 || kv_type == ATTN_I8) && (q_type == ATTN_BF16 || q_type == ATTN_F16) &&
         (D == 128 || D == 256) && G >= 1 && G <= 8 && (reinterpret_cast<uintptr_t>(q) & 15u) == 0 &&
         q_sr % 8 == 0 && q_sh % 8 == 0;
}

cudaError_t launch_decode_stream(const DecodePlan& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                                 cudaStream_t stream, cudaEvent_t after_main) {
  if (p.kv_type == ATTN_FP8_E4M3 || p.kv_type == ATTN_I8) {
    const bool e4 = p.kv_type == ATTN_FP8_E4M3;
    if (p.D == 128)
      return e4 ? launch_stream_t<e4m3_code, 128, 8>(p, tmK, tmV, stream, after_main)
                : launch_stream_t<i8_code, 128, 8>(p, tmK, tmV, stream, after_main);
    return e4 ? launch_stream_t<e4m3_code, 256, 8>(p, tmK, tmV, stream, after_main)
              : launch_stream_t<i8_code, 256, 8>(p, tmK, tmV, stream, after_main);
  }
  if (p.kv_type == ATTN_F16) return launch_stream_k<__half>(p, tmK, tmV, stream, after_main);
  return launch_stream_k<__nv_bfloat16>(p, tmK, tmV, stream, after_main);
}

}  // namespace attn
