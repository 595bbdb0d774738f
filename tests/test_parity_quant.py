"""attn_decode and attn_prefill over e4m3 and int8 caches against the FP64
oracle on a B200.

The cache holds one-byte codes with one F32 scale per (cell, KV head) for K
and for V (TensorFold PR #911's e4m3 rows with scale amax / 448; TensorFold
PR #2595's int8 cache with K and V scales); the oracle dequantizes the codes
from the format's definition.  Covers head sizes, GQA groups and forced or
automatic slices, the semantics features (ranges, sequences, causal, mask,
softcap, ALiBi, sinks), e4m3 NaN codes in visible and in excluded cells, and
the quantized GQA decode batch at full size.  attn_prefill widens the codes
(times their scales, rounded once to the Q dtype) into its workspace and runs
the tensor-core prefill on them: the same oracle, over head sizes, the
causality routes, softcap + ALiBi + sinks, sequence ids, packed rows, the e4m3
NaN code in cells some rows see, and the causal prefill workload's shape.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import attention_split_attn_b200 as A
from attention_split_attn_b200 import workloads as W
from parity import check, run_decode, run_prefill

pytestmark = pytest.mark.gpu

FMTS = ["e4m3", "i8"]


def quantized(p, fmt):
    k, ks = W.quantize_kv(p.k.to(torch.float32), fmt)
    v, vs = W.quantize_kv(p.v.to(torch.float32), fmt)
    return dataclasses.replace(p, k=k, v=v, k_scale=ks, v_scale=vs)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("G", [1, 4, 8, 16])
def test_dim_group_sweep(cuda_lib, fmt, D, G):
    Hkv = 2
    p = quantized(W.random_problem(9000 + D * 10 + G, R=3, Hq=G * Hkv, Hkv=Hkv, D=D, N=300,
                                   q_dtype=torch.bfloat16, out_dtype=torch.float32, lengths=[300, 45, 0]), fmt)
    ref = oracle.attn(p)
    for S in (0, 1, 3):
        check(p, run_decode(p, n_slices=S), f"{fmt} D={D} G={G} S={S}", ref=ref)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("feat", ["seqs", "causal", "mask", "softcap_alibi_sinks"])
def test_semantics_features(cuda_lib, fmt, feat):
    kw = dict(seqs=dict(seqs=3), causal=dict(causal=True), mask=dict(mask_frac=0.3),
              softcap_alibi_sinks=dict(softcap=20.0, alibi=True, sinks=True, causal=True))[feat]
    p = quantized(W.random_problem(9500 + len(feat), R=5, Hq=8, Hkv=2, D=128, N=700, q_dtype=torch.float16,
                                   out_dtype=torch.bfloat16, **kw), fmt)
    ref = oracle.attn(p)
    for S in (0, 4):
        check(p, run_decode(p, n_slices=S), f"{fmt} {feat} S={S}", ref=ref)


def test_e4m3_nan_code_visible_and_excluded(cuda_lib):
    """The e4m3 NaN code in a visible cell's V reaches that element of the
    output (also across the split combine); in a cell outside every row's range
    it is never read."""
    p = quantized(W.random_problem(9700, R=2, Hq=4, Hkv=2, D=64, N=200, q_dtype=torch.bfloat16,
                                   lengths=[150, 60]), "e4m3")
    b0, b1 = int(p.row_begin[0]), int(p.row_begin[1])
    v = p.v.view(torch.uint8).clone()
    c0 = next(c for c in range(b0, b0 + 150) if not b1 <= c < b1 + 60)
    v[c0, 1, 5] = 0x7F                                 # visible to row 0 only, KV head 1
    outside = [c for c in range(200) if not (b0 <= c < b0 + 150 or b1 <= c < b1 + 60)]
    if outside:
        v[outside[0], :, :] = 0x7F                     # seen by no row
    p = dataclasses.replace(p, v=v.view(torch.float8_e4m3fn))
    ref = oracle.attn(p)
    assert np.isnan(ref[0, 2:, 5]).all() and not np.isnan(ref[1]).any()
    for S in (0, 1, 3):
        check(p, run_decode(p, n_slices=S), f"nan S={S}", ref=ref)


@pytest.mark.parametrize("fmt", FMTS)
def test_quantized_gqa_decode_full(cuda_lib, fmt):
    """The GQA decode batch over a quantized cache at full size (16 rows, up to
    8192 cells each), every output element against the oracle."""
    p = W.quantized_decode(fmt=fmt)
    check(p, run_decode(p), f"{fmt} full")


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("q_dtype", [torch.bfloat16, torch.float16])
def test_prefill_dims_and_q_dtypes(cuda_lib, fmt, D, q_dtype):
    p = W.random_prefill(9800 + D, R=150, Hq=8, Hkv=2, D=D, depth=300, kv_dtype=torch.float32,
                         causal_by="mask", softcap=30.0, alibi=True, sinks=True)
    p = quantized(dataclasses.replace(p, q=p.q.to(q_dtype)), fmt)
    check(p, run_prefill(p), f"prefill {fmt} D={D} q={q_dtype}")


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("causal_by", ["flag", "pos", "mask"])
def test_prefill_causality_routes(cuda_lib, fmt, causal_by):
    p = W.random_prefill(9850 + len(causal_by), R=200, Hq=8, Hkv=2, D=128, depth=500, kv_dtype=torch.float32,
                         causal_by=causal_by, alibi=True)
    p = quantized(dataclasses.replace(p, q=p.q.to(torch.bfloat16)), fmt)
    check(p, run_prefill(p), f"prefill {fmt} causal by {causal_by}")


@pytest.mark.parametrize("fmt", FMTS)
def test_prefill_sequences_and_packed_rows(cuda_lib, fmt):
    """Sequence ids (the dense path's filter) and few rows (packed rows)."""
    p = quantized(W.random_problem(9900, R=5, Hq=16, Hkv=4, D=128, N=900, q_dtype=torch.bfloat16,
                                   out_dtype=torch.float32, seqs=3, causal=True, sinks=True), fmt)
    check(p, run_prefill(p), f"prefill {fmt} seqs + packed")
    p = quantized(W.random_problem(9901, R=40, Hq=8, Hkv=2, D=64, N=3000, q_dtype=torch.float16,
                                   out_dtype=torch.bfloat16, mask_frac=0.2), fmt)
    check(p, run_prefill(p), f"prefill {fmt} mask + packed")


def test_prefill_e4m3_nan_code_in_some_rows(cuda_lib):
    """The e4m3 NaN code in V of cells only the later rows see: NaN in that
    element for those rows, never for the rows that cannot see the cell."""
    p = W.random_prefill(9950, R=130, Hq=4, Hkv=2, D=128, depth=200, kv_dtype=torch.float32, causal_by="mask")
    p = quantized(dataclasses.replace(p, q=p.q.to(torch.bfloat16)), "e4m3")
    v = p.v.view(torch.uint8).clone()
    v[p.n_cells - 20, 0, 7] = 0x7F          # the row at position n_cells - 20 and later see it
    p = dataclasses.replace(p, v=v.view(torch.float8_e4m3fn))
    ref = oracle.attn(p)
    assert np.isnan(ref).any() and not np.isnan(ref).all()
    check(p, run_prefill(p), "prefill e4m3 NaN code", ref=ref)


@pytest.mark.parametrize("fmt", FMTS)
def test_prefill_causal_workload_shape_sampled(cuda_lib, fmt):
    """The causal prefill workload (2048 rows over 14048 cells, 64 q / 8 KV
    heads, softcap 50, ALiBi, sinks, F32 causal mask) over a quantized cache;
    one row of every 128-row tile against the oracle."""
    p = W.causal_prefill()
    p = quantized(p, fmt)
    out = run_prefill(p)
    rng = np.random.default_rng(11)
    rows = np.array([t * 128 + int(rng.integers(128)) for t in range(p.n_rows // 128)])
    sub = p.row_subset(rows)
    check(sub, out[torch.from_numpy(rows).cuda()], f"causal prefill {fmt} sample")
