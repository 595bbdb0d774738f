"""Seeded synthetic inputs for attention over a KV cache.

This module only draws numbers and lays them out (shapes, dtypes, lengths,
sequence ids, selection lists, masks, poison cells).  It holds none of the
attention arithmetic, so both the CUDA path and the FP64 oracle consume the
same stored values without sharing any computation.

Every tensor is a CPU torch tensor in its storage dtype.  Floating values are
drawn as float32 N(0, 1) from ``numpy.random.default_rng(seed)`` and then cast
to the storage dtype with round-to-nearest-even (torch's cast).

The five named workloads follow the shapes of the pages' workloads:
  * decode at depth over a bf16 cache and split-K slices -- TensorFold PR #2595
    (attn_decode on a (rows, heads, slices) grid, "Receipt" and "Kernel
    contract" sections);
  * maskless selected-key prefill, GQA 12 at head size 256, top-k blocks of
    4 cells -- strix-llama.cpp PR #115/#119 (flash_attn_sel.comp commit
    message, llama-bench pp2048 at depth);
  * causal prefill with softcap, ALiBi, sinks and an F32 mask -- HartsyInference
    PR #910 "attention semantic correctness";
  * a unified cache with interleaved sequences -- strix-llama.cpp PR #115,
    "Isolation" measurements (-np 4 -kvu).
No dataset, model or text is involved.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

F32, F16, BF16 = torch.float32, torch.float16, torch.bfloat16


@dataclasses.dataclass
class Problem:
    """One attention call's inputs (host tensors, storage dtypes)."""
    name: str
    q: torch.Tensor                      # [R, Hq, D]
    k: torch.Tensor                      # [N, Hkv, D]
    v: torch.Tensor                      # [N, Hkv, D]
    out_dtype: torch.dtype = F32
    scale: float = 1.0
    softcap: float = 0.0
    row_begin: Optional[torch.Tensor] = None   # int32 [R]
    row_end: Optional[torch.Tensor] = None     # int32 [R]
    cell_seq: Optional[torch.Tensor] = None    # int32 [N]
    row_seq: Optional[torch.Tensor] = None     # int32 [R]
    cell_pos: Optional[torch.Tensor] = None    # int32 [N]
    row_pos: Optional[torch.Tensor] = None     # int32 [R]
    causal: bool = False
    mask: Optional[torch.Tensor] = None        # float32 [R, N]
    alibi_slopes: Optional[torch.Tensor] = None  # float32 [Hq]
    sinks: Optional[torch.Tensor] = None       # float32 [Hq]
    sel: Optional[torch.Tensor] = None         # int32 [R, n_sel]
    n_slices: int = 0                          # 0: chosen by the planner
    max_row_len: int = 0                       # 0: unknown (bounded by N)
    k_scale: Optional[torch.Tensor] = None     # float32 [N, Hkv] (e4m3 / int8 caches)
    v_scale: Optional[torch.Tensor] = None     # float32 [N, Hkv]

    @property
    def n_rows(self) -> int: return self.q.shape[0]
    @property
    def n_head_q(self) -> int: return self.q.shape[1]
    @property
    def head_dim(self) -> int: return self.q.shape[2]
    @property
    def n_cells(self) -> int: return self.k.shape[0]
    @property
    def n_head_kv(self) -> int: return self.k.shape[1]

    def row_subset(self, rows) -> "Problem":
        """The same problem restricted to some query rows (for sampled checks)."""
        idx = torch.as_tensor(rows, dtype=torch.long)
        pick = lambda t: None if t is None else t.index_select(0, idx).contiguous()
        return dataclasses.replace(
            self, q=pick(self.q), row_begin=pick(self.row_begin), row_end=pick(self.row_end),
            row_seq=pick(self.row_seq), row_pos=pick(self.row_pos), mask=pick(self.mask),
            sel=pick(self.sel))


def _normal(rng: np.random.Generator, shape, dtype: torch.dtype) -> torch.Tensor:
    x = torch.from_numpy(rng.standard_normal(size=shape, dtype=np.float32))
    return x if dtype == F32 else x.to(dtype)


def _i32(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.int32)))


def alibi_slopes_textbook(n_head: int) -> torch.Tensor:
    """Slopes 2^(-8h/n_head) for h = 1..n_head (the textbook geometric set)."""
    h = np.arange(1, n_head + 1, dtype=np.float64)
    return torch.from_numpy((2.0 ** (-8.0 * h / n_head)).astype(np.float32))


# ----------------------------------------------------------------------------
# The five named workloads
# ----------------------------------------------------------------------------

def tiny_decode(seed: int = 1001) -> Problem:
    """1 row, 4 q heads over 1 KV head, D 64, 128 cells, FP32, 4 slices."""
    rng = np.random.default_rng(seed)
    R, Hq, Hkv, D, N = 1, 4, 1, 64, 128
    q = _normal(rng, (R, Hq, D), F32)
    k = _normal(rng, (N, Hkv, D), F32)
    v = _normal(rng, (N, Hkv, D), F32)
    return Problem("tiny_decode", q, k, v, out_dtype=F32, scale=1.0 / math.sqrt(D), n_slices=4)


def gqa_decode(seed: int = 1002, n_seq: int = 16, cap: int = 8192, Hq: int = 32,
               Hkv: int = 8, D: int = 128, poison_unused: bool = True) -> Problem:
    """16 sequences x 1 row, 32/8 heads, D 128, bf16 cache [16*8192, 8, 128];
    sequence s occupies cells [8192 s, 8192 s + len_s), len_s ~ U{1024..8192}.
    Cells past a sequence's length hold NaN (they must never be read)."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(1024, cap + 1, size=n_seq)
    N = n_seq * cap
    q = _normal(rng, (n_seq, Hq, D), BF16)
    k = torch.full((N, Hkv, D), float("nan") if poison_unused else 0.0, dtype=BF16)
    v = torch.full((N, Hkv, D), float("nan") if poison_unused else 0.0, dtype=BF16)
    for s in range(n_seq):
        b, n = s * cap, int(lens[s])
        k[b:b + n] = _normal(rng, (n, Hkv, D), BF16)
        v[b:b + n] = _normal(rng, (n, Hkv, D), BF16)
    begin = np.arange(n_seq, dtype=np.int64) * cap
    return Problem("gqa_decode", q, k, v, out_dtype=BF16, scale=1.0 / math.sqrt(D),
                   row_begin=_i32(begin), row_end=_i32(begin + lens), max_row_len=cap)


def quantize_kv(x: torch.Tensor, fmt: str):
    """Codes and float32 [N, Hkv] scales of a float [N, Hkv, D] cache: one scale
    per (cell, KV head) = amax / 448 for e4m3 (TensorFold PR #911), amax / 127
    for int8; an all-zero row gets scale 1."""
    amax = x.abs().amax(dim=2).to(torch.float32)
    top = 448.0 if fmt == "e4m3" else 127.0
    scale = torch.where(amax > 0, amax / top, torch.ones_like(amax))
    y = x.to(torch.float32) / scale[:, :, None]
    if fmt == "e4m3":
        return y.to(torch.float8_e4m3fn), scale
    return torch.round(y).clamp(-127, 127).to(torch.int8), scale


def quantized_decode(seed: int = 1007, fmt: str = "e4m3", n_seq: int = 16, cap: int = 8192, Hq: int = 32,
                     Hkv: int = 8, D: int = 128) -> Problem:
    """The GQA decode batch (16 sequences x 1 row, 32/8 heads, D 128, len_s ~
    U{1024..8192} in a [16*8192, 8, 128] cache) over an e4m3 or int8 cache
    quantized from N(0,1) rows with per (cell, KV head) scales; bf16 Q and out."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(min(1024, cap), cap + 1, size=n_seq)
    N = n_seq * cap
    q = _normal(rng, (n_seq, Hq, D), BF16)
    k, ks = quantize_kv(_normal(rng, (N, Hkv, D), F32), fmt)
    v, vs = quantize_kv(_normal(rng, (N, Hkv, D), F32), fmt)
    begin = np.arange(n_seq, dtype=np.int64) * cap
    return Problem(f"quantized_decode_{fmt}", q, k, v, out_dtype=BF16, scale=1.0 / math.sqrt(D),
                   row_begin=_i32(begin), row_end=_i32(begin + lens), max_row_len=cap, k_scale=ks, v_scale=vs)


def selected_prefill(seed: int = 1003, R: int = 2048, N: int = 32768, Hq: int = 48,
                     Hkv: int = 4, D: int = 256, n_blocks: int = 512, block: int = 4,
                     dup_frac: float = 0.05, inv_frac: float = 0.03) -> Problem:
    """2048 rows at positions N-R..N-1 over N = 32768 fp16 cells, GQA 12, D 256.
    Each row's list: 512 distinct fully causal blocks of 4 cells chosen
    uniformly (a stand-in for an indexer's top-k blocks), then 5% of the
    entries overwritten by copies of other entries and 3% by -1, then shuffled."""
    rng = np.random.default_rng(seed)
    q = _normal(rng, (R, Hq, D), F16)
    k = _normal(rng, (N, Hkv, D), F16)
    v = _normal(rng, (N, Hkv, D), F16)
    pos = (N - R) + np.arange(R, dtype=np.int64)
    sel = _block_lists(rng, pos, n_blocks, block, dup_frac, inv_frac)
    return Problem("selected_prefill", q, k, v, out_dtype=F32, scale=1.0 / math.sqrt(D),
                   row_pos=_i32(pos), sel=_i32(sel))


def _block_lists(rng, pos, n_blocks, block, dup_frac, inv_frac):
    R = len(pos)
    n_sel = n_blocks * block
    n_avail = (pos + 1) // block                     # blocks entirely at or before pos
    maxb = int(n_avail.max())
    keys = rng.random((R, maxb))
    keys[np.arange(maxb)[None, :] >= n_avail[:, None]] = np.inf
    blocks = np.argpartition(keys, n_blocks - 1, axis=1)[:, :n_blocks]
    cells = (block * blocks[:, :, None] + np.arange(block)[None, None, :]).reshape(R, n_sel)
    n_dup = int(round(dup_frac * n_sel))
    n_inv = int(round(inv_frac * n_sel))
    perm = np.argsort(rng.random((R, n_sel)), axis=1)
    rows = np.arange(R)[:, None]
    dup_at = perm[:, :n_dup]
    inv_at = perm[:, n_dup:n_dup + n_inv]
    rest = perm[:, n_dup + n_inv:]
    src = rest[rows, rng.integers(0, rest.shape[1], size=(R, n_dup))]
    cells[rows, dup_at] = cells[rows, src]
    cells[rows, inv_at] = -1
    shuffle = np.argsort(rng.random((R, n_sel)), axis=1)
    return cells[rows, shuffle]


def causal_prefill(seed: int = 1004, R: int = 2048, depth: int = 12000, Hq: int = 64,
                   Hkv: int = 8, D: int = 128, softcap: float = 50.0) -> Problem:
    """2048 new rows at positions depth..depth+R-1 over depth+R bf16 cells;
    softcap 50, ALiBi slopes 2^(-8h/64), per-head sinks N(0,1), causality
    carried by an F32 mask (0 visible, -inf hidden); causal flag off."""
    rng = np.random.default_rng(seed)
    N = depth + R
    q = _normal(rng, (R, Hq, D), BF16)
    k = _normal(rng, (N, Hkv, D), BF16)
    v = _normal(rng, (N, Hkv, D), BF16)
    sinks = torch.from_numpy(rng.standard_normal(Hq).astype(np.float32))
    rpos = depth + np.arange(R, dtype=np.int64)
    cols = np.arange(N, dtype=np.int64)
    mask = np.where(cols[None, :] <= rpos[:, None], np.float32(0.0), np.float32(-np.inf))
    return Problem("causal_prefill", q, k, v, out_dtype=BF16, scale=1.0 / math.sqrt(D),
                   softcap=softcap, row_pos=_i32(rpos), mask=torch.from_numpy(mask),
                   alibi_slopes=alibi_slopes_textbook(Hq), sinks=sinks)


def semantics_sweep(seed: int = 1005, R: int = 256, n_seq: int = 8, max_len: int = 65536,
                    Hq: int = 16, Hkv: int = 4, D: int = 128) -> Problem:
    """Unified fp16 cache of 8 interleaved sequences (per-cell seq id and pos),
    256 rows with visible lengths log-uniform in [1, 65536], causal, F32 mask
    with -inf/+inf entries, 2% of rows fully excluded, NaN in 1% of visible
    cells' V, NaN K in one cell of two sequences, NaN-filled cells that no row
    may read (a ninth, row-less sequence, and cells masked for all rows of
    their sequence), sinks on heads 0..7."""
    rng = np.random.default_rng(seed)
    row_seq = rng.integers(0, n_seq, size=R)
    ell = np.floor(np.exp(rng.uniform(0.0, math.log(max_len), size=R))).astype(np.int64)
    ell = np.clip(ell, 1, max_len)
    L = np.zeros(n_seq, dtype=np.int64)
    for s in range(n_seq):
        if np.any(row_seq == s):
            L[s] = ell[row_seq == s].max()
    N0 = int(L.sum())
    n_dead = max(1, N0 // 100)                      # row-less poison cells
    N = N0 + n_dead
    seq_of = np.concatenate([np.repeat(np.arange(n_seq), L), np.full(n_dead, n_seq)])
    pos_of = np.concatenate([np.concatenate([np.arange(l) for l in L]),
                             rng.integers(0, max_len, size=n_dead)])
    perm = rng.permutation(N)
    cell_seq = np.empty(N, dtype=np.int64); cell_seq[perm] = seq_of
    cell_pos = np.empty(N, dtype=np.int64); cell_pos[perm] = pos_of
    row_pos = ell - 1

    q = _normal(rng, (R, Hq, D), F16)
    k = _normal(rng, (N, Hkv, D), F16)
    v = _normal(rng, (N, Hkv, D), F16)

    mask = np.zeros((R, N), dtype=np.float32)
    mask[rng.random((R, N)) < 0.05] = -np.inf
    visible = lambda r: np.nonzero((cell_seq == row_seq[r]) & (cell_pos <= row_pos[r]))[0]
    for r in rng.choice(R, size=max(1, round(0.001 * R)), replace=False):
        cand = visible(r)
        mask[r, cand[rng.integers(len(cand))]] = np.inf
    for r in rng.choice(R, size=max(1, round(0.02 * R)), replace=False):
        mask[r, visible(r)] = -np.inf

    real = np.nonzero(cell_seq < n_seq)[0]
    nan_v = rng.choice(real, size=max(1, len(real) // 100), replace=False)
    for g in range(Hkv):
        v[nan_v, g, rng.integers(0, D, size=len(nan_v))] = float("nan")
    for s in rng.choice(n_seq, size=2, replace=False):
        c = rng.choice(np.nonzero(cell_seq == s)[0])
        k[c, rng.integers(Hkv), rng.integers(D)] = float("nan")
    hidden = rng.choice(real, size=max(1, len(real) // 200), replace=False)
    for c in hidden:                                 # masked for every row of its sequence
        mask[row_seq == cell_seq[c], c] = -np.inf
    dead = np.concatenate([hidden, np.nonzero(cell_seq == n_seq)[0]])
    k[dead] = float("nan")
    v[dead] = float("nan")

    sinks = np.full(Hq, -np.inf, dtype=np.float32)
    sinks[: Hq // 2] = rng.standard_normal(Hq // 2).astype(np.float32)
    return Problem("semantics_sweep", q, k, v, out_dtype=F32, scale=1.0 / math.sqrt(D),
                   cell_seq=_i32(cell_seq), row_seq=_i32(row_seq), cell_pos=_i32(cell_pos),
                   row_pos=_i32(row_pos), causal=True, mask=torch.from_numpy(mask),
                   sinks=torch.from_numpy(sinks), max_row_len=N)


def tree_decode(seed: int = 1006, width: int = 16, visible: int = 32770, Hq: int = 32, Hkv: int = 8,
                D: int = 128) -> Problem:
    """Draft-tree decode rows (TensorFold PR #2595: tree table with heap-order
    parents, widths 1..16, visible keys such as 33, 34, 8193, 32768..32770):
    `width` rows, node i's parent (i - 1) // 2 (a binary heap; -1 for the
    root), node i's token in cell prefix + i with prefix = visible - 1, so the
    root sees `visible` cells.  Bf16 Q/K/V ~ N(0, 1), bf16 out.  The visibility
    mask (0 for the prefix and the row's ancestors-or-self, -inf elsewhere) is
    built here on the host for the oracle; the CUDA path builds its own."""
    rng = np.random.default_rng(seed)
    prefix = visible - 1
    N = prefix + width
    q = _normal(rng, (width, Hq, D), BF16)
    k = _normal(rng, (N, Hkv, D), BF16)
    v = _normal(rng, (N, Hkv, D), BF16)
    parent = np.array([-1] + [(i - 1) // 2 for i in range(1, width)], dtype=np.int64)
    mask = np.full((width, N), -np.inf, dtype=np.float32)
    mask[:, :prefix] = 0.0
    for r in range(width):
        node = r
        while node >= 0:
            mask[r, prefix + node] = 0.0
            node = parent[node]
    p = Problem("tree_decode", q, k, v, out_dtype=BF16, scale=1.0 / math.sqrt(D), mask=torch.from_numpy(mask))
    p.tree_parent = _i32(parent)
    p.tree_prefix = prefix
    return p


WORKLOADS = {
    "tiny_decode": tiny_decode,
    "gqa_decode": gqa_decode,
    "selected_prefill": selected_prefill,
    "causal_prefill": causal_prefill,
    "semantics_sweep": semantics_sweep,
}


# ----------------------------------------------------------------------------
# Small randomised problems for the test suite
# ----------------------------------------------------------------------------

def random_problem(seed: int, R: int = 3, Hq: int = 4, Hkv: int = 2, D: int = 64,
                   N: int = 100, kv_dtype=F32, q_dtype=None, out_dtype=F32,
                   lengths: Optional[list] = None, ranges: bool = True,
                   seqs: int = 0, causal: bool = False, mask_frac: float = 0.0,
                   softcap: float = 0.0, alibi: bool = False, sinks: bool = False,
                   n_slices: int = 0, scale: Optional[float] = None,
                   value_scale: float = 1.0, positions: str = "given",
                   overhang: int = 0) -> Problem:
    """A small dense-visibility problem.  Each row r gets a range
    [begin_r, begin_r + len_r) inside [0, N) (or the whole cache when
    ranges=False); optional sequence ids, positions, mask, softcap, ALiBi
    and sinks.  positions (used when causal or alibi): "given" (a random
    permutation of cell positions and random row positions), "none" (both
    left unset, so the defaults from the range apply), "row" (row positions
    only), "cell" (cell positions only).  overhang > 0 moves each range's ends
    by up to that many cells past 0 and N (a range partly outside the cache)."""
    rng = np.random.default_rng(seed)
    q_dtype = q_dtype or kv_dtype
    q = _normal(rng, (R, Hq, D), F32) * value_scale
    q = q.to(q_dtype)
    k = (_normal(rng, (N, Hkv, D), F32) * value_scale).to(kv_dtype)
    v = _normal(rng, (N, Hkv, D), kv_dtype)
    p = Problem("random", q, k, v, out_dtype=out_dtype,
                scale=(1.0 / math.sqrt(D)) if scale is None else scale,
                softcap=softcap, causal=causal, n_slices=n_slices)
    if ranges:
        if lengths is None:
            lengths = [int(x) for x in rng.integers(0, N + 1, size=R)]
        begins = [int(rng.integers(0, N - l + 1)) for l in lengths]
        ends = [b + l for b, l in zip(begins, lengths)]
        if overhang > 0:
            begins = [b - int(rng.integers(0, overhang + 1)) if b == 0 or rng.random() < 0.5 else b
                      for b in begins]
            ends = [e + int(rng.integers(0, overhang + 1)) if e == N or rng.random() < 0.5 else e
                    for e in ends]
        p.row_begin = _i32(begins)
        p.row_end = _i32(ends)
    if seqs:
        p.cell_seq = _i32(rng.integers(0, seqs, size=N))
        p.row_seq = _i32(rng.integers(0, seqs, size=R))
    if causal or alibi:
        cpos, rpos = rng.permutation(N), rng.integers(0, N, size=R)
        if positions in ("given", "cell"):
            p.cell_pos = _i32(cpos)
        if positions in ("given", "row"):
            p.row_pos = _i32(rpos)
    if mask_frac > 0:
        m = rng.standard_normal((R, N)).astype(np.float32)
        m[rng.random((R, N)) < mask_frac] = -np.inf
        p.mask = torch.from_numpy(m)
    if alibi:
        p.alibi_slopes = torch.from_numpy(rng.uniform(0.01, 0.5, size=Hq).astype(np.float32))
    if sinks:
        p.sinks = torch.from_numpy(rng.standard_normal(Hq).astype(np.float32))
    return p


def random_prefill(seed: int, R: int = 130, Hq: int = 4, Hkv: int = 2, D: int = 128,
                   depth: int = 300, kv_dtype=BF16, out_dtype=F32, causal_by: str = "flag",
                   softcap: float = 0.0, alibi: bool = False, sinks: bool = False,
                   bias_frac: float = 0.0, nan_v: int = 0, extra_cells: int = 0,
                   value_scale: float = 1.0, scale: Optional[float] = None) -> Problem:
    """R new query rows at positions depth .. depth+R-1 over a cache of
    depth + R cells (plus `extra_cells` later cells no row may see).
    causal_by: "flag" (causal flag, row positions, affine cell positions),
    "pos" (causal flag with explicit cell positions), "mask" (an F32 mask of
    0 / -inf carries causality, causal flag off).  bias_frac: that fraction of
    mask entries on visible cells get a finite N(0,1) bias (mask mode only).
    nan_v: that many cells of the last R (each visible to some rows only) get a
    NaN in one V element of every KV head."""
    rng = np.random.default_rng(seed)
    N = depth + R + extra_cells
    q = (_normal(rng, (R, Hq, D), F32) * value_scale).to(kv_dtype)
    k = (_normal(rng, (N, Hkv, D), F32) * value_scale).to(kv_dtype)
    v = _normal(rng, (N, Hkv, D), kv_dtype)
    rpos = depth + np.arange(R, dtype=np.int64)
    p = Problem("random_prefill", q, k, v, out_dtype=out_dtype,
                scale=(1.0 / math.sqrt(D)) if scale is None else scale, softcap=softcap,
                row_pos=_i32(rpos))
    if causal_by in ("flag", "pos"):
        p.causal = True
        if causal_by == "pos":
            p.cell_pos = _i32(np.arange(N))
    elif causal_by == "mask":
        cols = np.arange(N, dtype=np.int64)
        m = np.where(cols[None, :] <= rpos[:, None], np.float32(0.0), np.float32(-np.inf))
        if bias_frac > 0:
            hit = (rng.random((R, N)) < bias_frac) & (m == 0)
            m[hit] = rng.standard_normal(int(hit.sum())).astype(np.float32)
        p.mask = torch.from_numpy(m)
    else:
        raise ValueError(causal_by)
    if nan_v:
        cells = rng.choice(np.arange(depth, depth + R), size=min(nan_v, R), replace=False)
        vv = p.v.clone()
        for c in cells:
            vv[int(c), :, int(rng.integers(D))] = float("nan")
        p.v = vv
    if alibi:
        p.alibi_slopes = alibi_slopes_textbook(Hq)
    if sinks:
        p.sinks = torch.from_numpy(rng.standard_normal(Hq).astype(np.float32))
    return p


def random_selected(seed: int, R: int = 4, Hq: int = 8, Hkv: int = 2, D: int = 64,
                    N: int = 200, n_sel: int = 96, kv_dtype=F16, out_dtype=F32,
                    inv_frac: float = 0.05, dup_frac: float = 0.1, softcap: float = 0.0,
                    alibi: bool = False, sinks: bool = False) -> Problem:
    """A small selected-key problem: random lists with duplicates and invalid
    entries (both -1 and >= N)."""
    rng = np.random.default_rng(seed)
    q = _normal(rng, (R, Hq, D), kv_dtype)
    k = _normal(rng, (N, Hkv, D), kv_dtype)
    v = _normal(rng, (N, Hkv, D), kv_dtype)
    sel = rng.integers(0, N, size=(R, n_sel))
    dup = rng.random((R, n_sel)) < dup_frac
    sel[dup] = sel[:, :1].repeat(n_sel, axis=1)[dup]
    inv = rng.random((R, n_sel)) < inv_frac
    sel[inv] = rng.choice(np.array([-1, -7, N, N + 5]), size=int(inv.sum()))
    p = Problem("random_selected", q, k, v, out_dtype=out_dtype, scale=1.0 / math.sqrt(D),
                softcap=softcap, sel=_i32(sel))
    if alibi:
        p.row_pos = _i32(rng.integers(0, N, size=R))
        p.alibi_slopes = torch.from_numpy(rng.uniform(0.01, 0.5, size=Hq).astype(np.float32))
    if sinks:
        p.sinks = torch.from_numpy(rng.standard_normal(Hq).astype(np.float32))
    return p
