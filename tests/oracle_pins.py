"""Pins of the FP64 oracle to things other than itself.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with
what the pages or the mathematics fix.  The pins use:
  * values the pages print for worked examples (tests/golden/*.json);
  * a library routine: torch's scaled_dot_product_attention in float64, to
    which dense visibility, masks, textbook causal ALiBi and sinks reduce
    (a sink is one extra key whose K and V are zero and whose bias is the
    sink logit);
  * closed forms (one key, zero query, two keys, softcap/ALiBi order);
  * brute-force enumeration of visibility subsets and special values on tiny
    inputs;
  * invariants (selection duplicates and order, unified-cache isolation, the
    split form, full selection == dense causal);
  * numpy.unique for the selection compaction;
  * torch's float8_e4m3fn conversion for the e4m3 codes of a quantized cache.
test_oracle_pins.py runs each one; test_oracle_mutations.py plants each known
kind of mistake in the oracle and checks that some pin catches it.
"""
from __future__ import annotations

import dataclasses
import itertools
import json
import math
import os

import numpy as np
import torch
import torch.nn.functional as F

import oracle
from attention_split_attn_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
INF = float("inf")
NAN = float("nan")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _num(x):
    return float(x) if not isinstance(x, str) else float(x.replace("inf", "inf"))


def _problem_from_golden(g):
    q = torch.tensor(g["q"], dtype=torch.float32)
    k = torch.tensor(g["k"], dtype=torch.float32)
    v = torch.tensor(g["v"], dtype=torch.float32)
    mask = torch.tensor([[_num(x) for x in row] for row in g["mask"]], dtype=torch.float32)
    return W.Problem("golden", q, k, v, scale=float(g["scale"]), mask=mask)


def _close(a, b, rtol=1e-13, atol=1e-300):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    na, nb = np.isnan(a), np.isnan(b)
    assert np.array_equal(na, nb), f"NaN pattern differs: {np.argwhere(na != nb)[:5]}"
    fa, fb = a[~na], b[~nb]
    err = np.abs(fa - fb)
    tol = atol + rtol * np.maximum(np.abs(fa), np.abs(fb))
    bad = err > tol
    assert not bad.any(), f"max err {err.max():.3e} at {np.argwhere(bad)[:3]}, {fa[bad][:3]} vs {fb[bad][:3]}"


# ----------------------------------------------------------------------------
# Library reference: torch SDPA in float64
# ----------------------------------------------------------------------------

def _positions(p):
    """Cell positions per row [R, N] and row positions [R] (int64).  Where the
    problem gives none, the boundary's defaults (the C ABI's "Positions"
    rule): cell c of row r sits at c - row_begin[r] and row r at
    row_end[r] - row_begin[r] - 1, from the range as given, even where it
    reaches outside [0, N)."""
    R, N = p.n_rows, p.n_cells
    b = p.row_begin.numpy().astype(np.int64) if p.row_begin is not None else np.zeros(R, np.int64)
    e = p.row_end.numpy().astype(np.int64) if p.row_end is not None else np.full(R, N, np.int64)
    if p.cell_pos is not None:
        cpos = np.broadcast_to(p.cell_pos.numpy().astype(np.int64)[None, :], (R, N))
    else:
        cpos = np.arange(N, dtype=np.int64)[None, :] - b[:, None]
    rpos = p.row_pos.numpy().astype(np.int64) if p.row_pos is not None else e - b - 1
    return cpos, rpos


def _visibility_bias(p):
    """[Hq, R, N] float64 bias: -inf where invisible, mask + textbook ALiBi where visible."""
    R, Hq, N = p.n_rows, p.n_head_q, p.n_cells
    vis = np.ones((R, N), dtype=bool)
    cols = np.arange(N)
    if p.row_begin is not None:
        b = p.row_begin.numpy()[:, None]
        e = p.row_end.numpy()[:, None]
        vis &= (cols[None, :] >= b) & (cols[None, :] < e)
    if p.cell_seq is not None and p.row_seq is not None:
        vis &= p.cell_seq.numpy()[None, :] == p.row_seq.numpy()[:, None]
    cpos, rpos = _positions(p)
    if p.causal:
        vis &= cpos <= rpos[:, None]
    bias = np.zeros((Hq, R, N), dtype=np.float64)
    if p.mask is not None:
        m = p.mask.numpy().astype(np.float64)
        vis &= ~(np.isneginf(m))
        bias += np.where(vis, m, 0.0)[None]
    if p.alibi_slopes is not None:
        # textbook causal ALiBi (Press et al.): bias = slope * (j - i) for key j <= query i
        assert p.causal, "the library pin covers causal ALiBi only"
        rel = (cpos - rpos[:, None]).astype(np.float64)                # <= 0 where visible
        slopes = p.alibi_slopes.numpy().astype(np.float64)
        bias += slopes[:, None, None] * np.where(vis, rel, 0.0)[None]
    bias[:, ~vis] = -INF
    return bias, vis


def sdpa_reference(p):
    """[R, Hq, D] via torch SDPA (float64), sinks as an extra zero key.  Rows
    with neither a visible key nor a sink come out NaN from SDPA; callers
    compare those separately."""
    assert p.softcap == 0 and p.sel is None
    R, Hq, D, N, Hkv = p.n_rows, p.n_head_q, p.head_dim, p.n_cells, p.n_head_kv
    G = Hq // Hkv
    q = p.q.to(torch.float64).permute(1, 0, 2)[None]                      # [1, Hq, R, D]
    k = p.k.to(torch.float64).repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    v = p.v.to(torch.float64).repeat_interleave(G, dim=1).permute(1, 0, 2)[None]
    bias, vis = _visibility_bias(p)
    bias = torch.from_numpy(bias)[None]                                   # [1, Hq, R, N]
    if p.sinks is not None:
        z = torch.zeros((1, Hq, 1, D), dtype=torch.float64)
        k = torch.cat([k, z], dim=2)
        v = torch.cat([v, z], dim=2)
        s = p.sinks.to(torch.float64)[None, :, None, None].expand(1, Hq, R, 1)
        bias = torch.cat([bias, s], dim=3)
    out = F.scaled_dot_product_attention(q, k, v, attn_mask=bias, scale=p.scale)
    return out[0].permute(1, 0, 2).numpy(), vis


def _compare_with_sdpa(p):
    ref, vis = sdpa_reference(p)
    got = oracle.attn(p)
    has_key = vis.any(axis=1)
    sig = p.sinks.numpy() if p.sinks is not None else np.full(p.n_head_q, -INF)
    for r in range(p.n_rows):
        for h in range(p.n_head_q):
            if has_key[r] or not np.isneginf(sig[h]):
                _close(got[r, h], ref[r, h], rtol=1e-12, atol=1e-14)
            else:   # fully excluded, no sink: exactly +0.0 (SDPA gives NaN here)
                assert np.all(got[r, h] == 0) and not np.signbit(got[r, h]).any()


def pin_sdpa_dense_ranges():
    for seed in range(6):
        _compare_with_sdpa(W.random_problem(seed, R=5, Hq=6, Hkv=3, D=16, N=70))


def pin_sdpa_mask_seq_causal():
    for seed in range(6):
        _compare_with_sdpa(W.random_problem(100 + seed, R=6, Hq=4, Hkv=2, D=8, N=60,
                                            ranges=(seed % 2 == 0), seqs=3, causal=True,
                                            mask_frac=0.3))


def pin_sdpa_alibi_textbook():
    for seed in range(4):
        _compare_with_sdpa(W.random_problem(200 + seed, R=5, Hq=4, Hkv=1, D=8, N=50,
                                            ranges=False, causal=True, alibi=True))


def pin_sdpa_default_positions():
    """No cell and/or row positions given: the defaults come from each row's
    range as given (nonzero and negative begins, ends past N), under causality,
    ALiBi and sinks."""
    for seed in range(4):
        for mode in ("none", "row", "cell"):
            _compare_with_sdpa(W.random_problem(400 + seed, R=7, Hq=4, Hkv=2, D=8, N=40,
                                                causal=True, alibi=True, sinks=True,
                                                positions=mode, overhang=6 * (seed % 2)))


def pin_sdpa_sinks():
    for seed in range(4):
        _compare_with_sdpa(W.random_problem(300 + seed, R=6, Hq=4, Hkv=2, D=8, N=40,
                                            sinks=True, mask_frac=0.2,
                                            lengths=[0, 1, 5, 40, 17, 2]))


def pin_gqa_mapping():
    """q heads 2g and 2g+1 read KV head g: with KV head 1 all zero, heads 2,3
    equal mean(V[:,1]) for Q = 0 and heads 0,1 follow KV head 0."""
    p = W.random_problem(7, R=2, Hq=4, Hkv=2, D=8, N=20, ranges=False)
    _compare_with_sdpa(p)
    p.q = torch.zeros_like(p.q)
    out = oracle.attn(p)
    mean_v = p.v.to(torch.float64).mean(dim=0).numpy()                    # [Hkv, D]
    for h in range(4):
        _close(out[0, h], mean_v[h // 2])


# ----------------------------------------------------------------------------
# Worked examples printed on the pages
# ----------------------------------------------------------------------------

def pin_golden_m03():
    g = _golden("m03_excluded_row.json")
    out = oracle.attn(_problem_from_golden(g))
    assert np.array_equal(out, np.array(g["expected"])), out
    assert not np.signbit(out).any(), "excluded row must be +0.0"


def pin_golden_finite_sentinel():
    g = _golden("finite_sentinel.json")
    _close(oracle.attn(_problem_from_golden(g)), np.array(g["expected"]))


def pin_golden_bias_range():
    g = _golden("bias_range.json")
    out = oracle.attn(_problem_from_golden(g))
    v0, v1 = g["v"][0][0][0], g["v"][1][0][0]
    _close(out[0, 0, 0], (v0 + math.e * v1) / (1 + math.e))


def pin_golden_sink_edges():
    g = _golden("sink_edge_cases.json")
    for case in g["cases"]:
        p = W.random_problem(11, R=1, Hq=1, Hkv=1, D=4, N=8, lengths=[0])
        p.sinks = torch.tensor([_num(case["sink"])], dtype=torch.float32)
        out = oracle.attn(p)
        if case["expected"] == "zero":
            assert np.all(out == 0) and not np.signbit(out).any(), (case, out)
        else:
            assert np.all(np.isnan(out)), (case, out)


def pin_golden_softcap_then_alibi():
    g = _golden("softcap_then_alibi.json")
    cap = g["softcap"]
    # two keys, D = 1: q = 10, k = (10, 0) -> raw scores (100, 0); slope 50 at
    # distances (1, 0) -> ALiBi biases (-50, 0)
    p = W.Problem("order", q=torch.tensor([[[10.0]]]), k=torch.tensor([[[10.0]], [[0.0]]]),
                  v=torch.tensor(g["v"], dtype=torch.float32).reshape(2, 1, 1),
                  scale=1.0, softcap=cap, row_pos=torch.tensor([1], dtype=torch.int32),
                  cell_pos=torch.tensor([0, 1], dtype=torch.int32),
                  alibi_slopes=torch.tensor([50.0]))
    x0 = cap * math.tanh(100.0 / cap) - 50.0
    expect = 1.0 / (1.0 + math.exp(0.0 - x0))
    out = oracle.attn(p)[0, 0, 0]
    _close(out, expect)
    wrong = 1.0 / (1.0 + math.exp(-cap * math.tanh(50.0 / cap)))
    assert abs(out - wrong) > 0.5


# ----------------------------------------------------------------------------
# Closed forms
# ----------------------------------------------------------------------------

def pin_closed_one_key():
    p = W.random_problem(21, R=3, Hq=2, Hkv=1, D=8, N=30, lengths=[1, 1, 1], softcap=3.0)
    out = oracle.attn(p)
    for r in range(3):
        c = int(p.row_begin[r])
        _close(out[r, 0], p.v[c, 0].double().numpy())
    # with a sink sigma: v / (1 + exp(sigma - x))
    p.sinks = torch.tensor([0.3, -1.2], dtype=torch.float32)
    p.softcap = 0.0
    out = oracle.attn(p)
    for r in range(3):
        c = int(p.row_begin[r])
        for h in range(2):
            x = p.scale * float((p.q[r, h].double() * p.k[c, 0].double()).sum())
            w = 1.0 / (1.0 + math.exp(float(p.sinks[h]) - x))
            _close(out[r, h], w * p.v[c, 0].double().numpy())


def pin_closed_zero_query_mean():
    p = W.random_problem(22, R=2, Hq=2, Hkv=2, D=8, N=40, lengths=[13, 40])
    p.q = torch.zeros_like(p.q)
    out = oracle.attn(p)
    for r in range(2):
        b, e = int(p.row_begin[r]), int(p.row_end[r])
        for h in range(2):
            _close(out[r, h], p.v[b:e, h].double().mean(dim=0).numpy())


def pin_closed_two_keys_logistic():
    p = W.random_problem(23, R=1, Hq=1, Hkv=1, D=4, N=2, ranges=False, softcap=2.0)
    out = oracle.attn(p)[0, 0]
    x = [p.softcap * math.tanh(p.scale * float((p.q[0, 0].double() * p.k[c, 0].double()).sum())
                               / p.softcap) for c in range(2)]
    w0 = 1.0 / (1.0 + math.exp(x[1] - x[0]))
    _close(out, w0 * p.v[0, 0].double().numpy() + (1 - w0) * p.v[1, 0].double().numpy())


def pin_softcap_limit():
    """softcap c -> infinity leaves the logits unchanged (tanh(y) ~ y)."""
    p = W.random_problem(24, R=3, Hq=2, Hkv=1, D=8, N=30)
    ref = oracle.attn(p)
    p.softcap = 1e7
    _close(oracle.attn(p), ref, rtol=1e-9, atol=1e-12)


def pin_scale_applies_inside_softcap():
    """softcap(scale * qk): doubling the scale with halved q is the identity."""
    p = W.random_problem(25, R=2, Hq=2, Hkv=1, D=8, N=30, softcap=1.5, scale=0.8)
    ref = oracle.attn(p)
    p2 = dataclasses.replace(p, q=(p.q * 4.0), scale=0.2)
    _close(oracle.attn(p2), ref, rtol=1e-12)
    p3 = dataclasses.replace(p, scale=1.6)
    p3 = dataclasses.replace(p3, q=p.q * 0.5)
    _close(oracle.attn(p3), ref, rtol=1e-12)
    # and the cap really bites at this scale
    p4 = dataclasses.replace(p, softcap=0.0)
    assert np.abs(oracle.attn(p4) - ref).max() > 1e-3


# ----------------------------------------------------------------------------
# Brute force on tiny inputs: every visibility subset x special values
# ----------------------------------------------------------------------------

def pin_brute_force_subsets():
    rng = np.random.default_rng(31)
    N, D = 4, 3
    q = torch.from_numpy(rng.standard_normal((1, 2, D)).astype(np.float32))
    k = torch.from_numpy(rng.standard_normal((N, 1, D)).astype(np.float32))
    v = torch.from_numpy(rng.standard_normal((N, 1, D)).astype(np.float32))
    specials = [0.0, 1e5, INF, NAN]
    sinks = [None, 0.5, -INF, INF, NAN]
    for bits in range(1 << N):
        for special, at in itertools.product(specials, range(N)):
            m = np.where([(bits >> c) & 1 for c in range(N)], 0.0, -INF).astype(np.float32)
            m = m.copy()
            if (bits >> at) & 1:
                m[at] = special
            for s in sinks:
                p = W.Problem("bf", q, k, v, scale=0.7, mask=torch.from_numpy(m[None]),
                              sinks=None if s is None else torch.tensor([s, s], dtype=torch.float32))
                ref, vis = sdpa_reference(p)
                got = oracle.attn(p)
                if not vis.any() and (s is None or s == -INF):
                    assert np.all(got == 0) and not np.signbit(got).any(), (bits, special, s, got)
                else:
                    _close(got, ref, rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------------------
# NaN semantics (HartsyInference #910: NaN carried through the max and sum)
# ----------------------------------------------------------------------------

def pin_nan_in_visible_v_poisons_one_dim():
    p = W.random_problem(41, R=2, Hq=2, Hkv=1, D=6, N=10, ranges=False)
    p.v = p.v.clone()
    p.v[3, 0, 2] = NAN
    out = oracle.attn(p)
    assert np.isnan(out[:, :, 2]).all() and not np.isnan(np.delete(out, 2, axis=2)).any()


def pin_nan_v_with_underflowing_weight():
    """A visible key whose weight underflows to 0 still poisons its dim (0*NaN)."""
    p = W.random_problem(42, R=1, Hq=1, Hkv=1, D=4, N=3, ranges=False)
    p.mask = torch.tensor([[0.0, -2000.0, 0.0]])
    p.v = p.v.clone()
    p.v[1, 0, 1] = NAN
    out = oracle.attn(p)
    assert np.isnan(out[0, 0, 1]) and not np.isnan(out[0, 0, [0, 2, 3]]).any()


def pin_nan_in_visible_k_poisons_row_head():
    p = W.random_problem(43, R=1, Hq=2, Hkv=2, D=4, N=6, ranges=False)
    p.k = p.k.clone()
    p.k[4, 1, 0] = NAN
    out = oracle.attn(p)
    assert np.isnan(out[0, 1]).all() and not np.isnan(out[0, 0]).any()


def pin_plus_inf_score_gives_nan():
    p = W.random_problem(44, R=1, Hq=1, Hkv=1, D=4, N=6, ranges=False)
    p.mask = torch.zeros((1, 6))
    p.mask[0, 2] = INF
    assert np.isnan(oracle.attn(p)).all()


def pin_masked_nan_cell_not_read():
    p = W.random_problem(45, R=1, Hq=1, Hkv=1, D=4, N=6, ranges=False)
    p.k = p.k.clone(); p.v = p.v.clone()
    p.k[1] = NAN; p.v[1] = NAN
    p.mask = torch.zeros((1, 6)); p.mask[0, 1] = -INF
    out = oracle.attn(p)
    assert not np.isnan(out).any()
    p2 = dataclasses.replace(p, k=torch.cat([p.k[:1], p.k[2:]]), v=torch.cat([p.v[:1], p.v[2:]]),
                             mask=torch.zeros((1, 5)))
    _close(out, oracle.attn(p2))


# ----------------------------------------------------------------------------
# Invariants
# ----------------------------------------------------------------------------

def pin_select_compact_numpy_unique():
    rng = np.random.default_rng(51)
    N = 300
    sel = rng.integers(-20, N + 20, size=(12, 80)).astype(np.int32)
    sel[3, :] = 7                                 # all duplicates
    sel[4, :] = -1                                # all invalid
    srt, cnt = oracle.select_compact(torch.from_numpy(sel), N)
    for r in range(12):
        u = np.unique(sel[r][(sel[r] >= 0) & (sel[r] < N)])
        assert cnt[r] == len(u) and np.array_equal(srt[r, :cnt[r]], u)
        assert np.all(srt[r, cnt[r]:] == -1)


def pin_selected_duplicates_and_order_irrelevant():
    p = W.random_selected(52, R=3, Hq=4, Hkv=2, D=8, N=80, n_sel=40, kv_dtype=torch.float32)
    ref = oracle.attn(p)
    srt, cnt = oracle.select_compact(p.sel, p.n_cells)
    for r in range(3):
        clean = dataclasses.replace(p.row_subset([r]),
                                    sel=torch.from_numpy(srt[r:r + 1, :cnt[r]].copy()))
        assert np.array_equal(oracle.attn(clean)[0], ref[r])
    rng = np.random.default_rng(3)
    shuf = torch.from_numpy(rng.permuted(p.sel.numpy(), axis=1).copy())
    assert np.array_equal(oracle.attn(dataclasses.replace(p, sel=shuf)), ref)


def pin_selected_full_list_equals_dense_causal():
    rng = np.random.default_rng(53)
    p = W.random_problem(53, R=4, Hq=4, Hkv=2, D=8, N=50, ranges=False, alibi=False,
                         softcap=2.5, sinks=True)
    rpos = rng.integers(0, 50, size=4)
    p.row_pos = torch.from_numpy(rpos.astype(np.int32))
    p.cell_pos = torch.arange(50, dtype=torch.int32)
    p.causal = True
    dense = oracle.attn(p)
    sel = np.full((4, 60), -1, dtype=np.int32)
    for r in range(4):
        sel[r, :rpos[r] + 1] = rng.permutation(rpos[r] + 1)
    ps = dataclasses.replace(p, causal=False, sel=torch.from_numpy(sel))
    _close(oracle.attn(ps), dense, rtol=1e-14)


def pin_unified_cache_isolation():
    p = W.random_problem(54, R=6, Hq=4, Hkv=2, D=8, N=90, ranges=False, seqs=3, causal=True,
                         sinks=True)
    ref = oracle.attn(p)
    other = p.cell_seq.numpy()[None, :] != p.row_seq.numpy()[:, None]    # [R, N]
    for r in range(6):
        k, v = p.k.clone(), p.v.clone()
        cells = torch.from_numpy(np.nonzero(other[r])[0])
        k[cells] = NAN
        v[cells] = torch.randn_like(v[cells])
        out = oracle.attn(dataclasses.replace(p, k=k, v=v))
        assert np.array_equal(out[r], ref[r], equal_nan=True)


def pin_split_form_equals_plain():
    cases = [W.random_problem(55, R=4, Hq=4, Hkv=2, D=8, N=300, seqs=2, causal=True,
                              mask_frac=0.2, sinks=True, softcap=4.0, alibi=True),
             W.random_problem(56, R=5, Hq=2, Hkv=1, D=8, N=129, lengths=[0, 1, 31, 33, 129],
                              sinks=True)]
    c = W.random_problem(57, R=3, Hq=2, Hkv=1, D=4, N=100, ranges=False, mask_frac=0.1)
    c.v = c.v.clone(); c.v[50, 0, 1] = NAN
    c.mask[1, :] = -INF
    cases.append(c)
    for p in cases:
        ref = oracle.attn(p)
        for S in (1, 2, 3, 7, 16, 33, 64):
            got = oracle.attn_split(p, S)
            _close(got, ref, rtol=1e-14, atol=1e-15)
            z = (ref == 0)
            assert np.array_equal(got[z], ref[z]) and not np.signbit(got[z]).any()


# ----------------------------------------------------------------------------
# Quantized caches (e4m3 / int8 codes with per (cell, KV head) scales)
# ----------------------------------------------------------------------------

def pin_e4m3_codes_match_torch():
    """The oracle's E4M3 decoding, written from the format's definition, against
    torch's float8_e4m3fn conversion for all 256 codes (NaN codes included)."""
    codes = np.arange(256, dtype=np.uint8)
    mine = oracle.e4m3_value(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(mine[ok], ref[ok])
    assert np.signbit(mine[0x80]) and mine[0x80] == 0 and mine[0x7E] == 448.0 and mine[0x01] == 2.0 ** -9


def pin_quantized_cache_equals_dequantized_sdpa():
    """An e4m3 or int8 cache with scales that differ across cells and KV heads
    (a scale applied to the wrong cell, head or tensor changes the result) is
    SDPA over the cache dequantized by torch (code * scale) in float64."""
    for fmt in ("e4m3", "i8"):
        for seed in range(3):
            rng = np.random.default_rng(700 + seed)
            R, Hq, Hkv, D, N = 3, 4, 2, 16, 40
            q = torch.from_numpy(rng.standard_normal((R, Hq, D)).astype(np.float32))
            raw_k = torch.from_numpy((rng.standard_normal((N, Hkv, D)) *
                                      rng.uniform(0.1, 8.0, (N, Hkv, 1))).astype(np.float32))
            raw_v = torch.from_numpy((rng.standard_normal((N, Hkv, D)) *
                                      rng.uniform(0.1, 8.0, (N, Hkv, 1))).astype(np.float32))
            k, ks = W.quantize_kv(raw_k, fmt)
            v, vs = W.quantize_kv(raw_v, fmt)
            pq = W.Problem("quant_pin", q, k, v, scale=0.3, k_scale=ks, v_scale=vs,
                           row_begin=torch.tensor([0, 5, 11], dtype=torch.int32),
                           row_end=torch.tensor([40, 33, 12], dtype=torch.int32),
                           sinks=torch.tensor([0.5, -1.0, -INF, 2.0], dtype=torch.float32))
            deq = lambda c, sc: c.to(torch.float64) * sc.to(torch.float64)[:, :, None]
            pd = dataclasses.replace(pq, k=deq(k, ks), v=deq(v, vs), k_scale=None, v_scale=None)
            ref, _ = sdpa_reference(pd)
            _close(oracle.attn(pq), ref, rtol=1e-12, atol=1e-14)


PINS = {name: fn for name, fn in globals().items() if name.startswith("pin_") and callable(fn)}
