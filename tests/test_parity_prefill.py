"""attn_prefill against the FP64 oracle on a B200.

Causal prefill with the semantics of HartsyInference PR #910 ("attention
semantic correctness": softcap before ALiBi, F32 mask bias unnarrowed,
per-head sinks, +0 for rows that see nothing, NaN propagation), on the
tensor-core path (tiles of 128 rows x 128 cells).  Covers dtypes / head sizes
/ GQA groups (odd ones leave a head slot idle), ragged row and cell counts,
the three ways causality reaches the kernel (flag with affine positions, flag
with explicit positions, an F32 mask), finite mask biases (mixed tiles), the
softcap polynomial and its large-logit branch, NaN V in cells only some rows
of a tile see (the CUDA-core P V route), empty caches and sink edge cases,
determinism, the unified-cache semantics sweep and the full-size causal
prefill workload (sampled rows).
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import attention_split_attn_b200 as A
from attention_split_attn_b200 import workloads as W
from parity import check, poisoned_workspace, run_prefill

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kv", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("G", [1, 2, 3, 8])
def test_dtype_dim_group_sweep(cuda_lib, kv, D, G):
    p = W.random_prefill(100 + D + G + (0 if kv == torch.float16 else 7), R=130, Hq=2 * G, Hkv=2, D=D,
                         depth=300, kv_dtype=kv)
    check(p, run_prefill(p), f"{kv} D={D} G={G}")


@pytest.mark.parametrize("R,depth,extra", [(1, 0, 0), (1, 5000, 0), (127, 1, 3), (128, 128, 0),
                                           (129, 0, 200), (300, 700, 129), (64, 0, 0)])
def test_ragged_rows_and_cells(cuda_lib, R, depth, extra):
    p = W.random_prefill(200 + R + depth, R=R, Hq=8, Hkv=2, D=128, depth=depth, extra_cells=extra,
                         out_dtype=torch.bfloat16, sinks=True)
    check(p, run_prefill(p), f"R={R} depth={depth} extra={extra}")


@pytest.mark.parametrize("causal_by", ["flag", "pos", "mask"])
def test_causality_routes(cuda_lib, causal_by):
    p = W.random_prefill(300, R=200, Hq=4, Hkv=1, D=128, depth=333, causal_by=causal_by, alibi=True,
                         sinks=True, softcap=30.0)
    check(p, run_prefill(p), causal_by)


@pytest.mark.parametrize("feature", ["softcap", "softcap_large", "alibi", "sinks", "bias", "all"])
def test_feature_sweep(cuda_lib, feature):
    big = feature == "softcap_large"
    p = W.random_prefill(400, R=160, Hq=6, Hkv=2, D=128, depth=250, causal_by="mask",
                         softcap=2.0 if big else (30.0 if feature in ("softcap", "all") else 0.0),
                         alibi=feature in ("alibi", "all"), sinks=feature in ("sinks", "all"),
                         bias_frac=0.2 if feature in ("bias", "all") else 0.0,
                         value_scale=2.0 if big else 1.0, out_dtype=torch.float32)
    check(p, run_prefill(p), feature)


def test_nan_v_in_cells_some_rows_cannot_see(cuda_lib):
    """A NaN in the V of cell c reaches exactly the rows that see c (rows at
    positions >= c); the rows of the same tile that do not see it stay finite."""
    p = W.random_prefill(500, R=256, Hq=4, Hkv=2, D=128, depth=64, causal_by="flag", nan_v=5, sinks=True)
    out = run_prefill(p)
    ref = oracle.attn(p)
    assert np.isnan(ref).any() and np.isfinite(ref).any()
    check(p, out, "nan v", ref=ref)


def test_nan_k_and_inf_mask(cuda_lib):
    p = W.random_prefill(501, R=140, Hq=4, Hkv=2, D=64, depth=200, causal_by="mask", kv_dtype=torch.float16)
    k = p.k.clone()
    k[10, 1, 3] = float("nan")               # visible to every row: KV head 1's rows all NaN
    k[250, 0, 0] = float("nan")              # visible to rows at positions >= 250
    mask = p.mask.clone()
    mask[7, 3] = float("inf")                # one +inf bias: row 7 NaN
    mask[9, :] = float("-inf")               # row 9 sees nothing: +0
    p = dataclasses.replace(p, k=k, mask=mask)
    check(p, run_prefill(p), "nan k / inf mask")


def test_empty_cache_and_sink_edges(cuda_lib):
    p = W.random_prefill(502, R=5, Hq=8, Hkv=2, D=128, depth=0, causal_by="flag", sinks=True)
    p = dataclasses.replace(p, k=p.k[:0].contiguous(), v=p.v[:0].contiguous())
    p.sinks = torch.tensor([0.5, -1.0, float("inf"), float("nan"), float("-inf"), 2.0, 0.0, 1.0])
    check(p, run_prefill(p), "empty cache")


def test_rows_seeing_nothing_are_zero(cuda_lib):
    p = W.random_prefill(503, R=130, Hq=4, Hkv=2, D=128, depth=100, causal_by="mask", sinks=False)
    mask = p.mask.clone()
    mask[::3] = float("-inf")
    p = dataclasses.replace(p, mask=mask)
    out = run_prefill(p)
    check(p, out, "excluded rows")
    assert torch.all(out[::3] == 0) and not torch.signbit(out[::3].float()).any()


def test_generic_visibility(cuda_lib):
    """Row ranges, sequence ids, explicit positions and a random mask: every
    tile is mixed."""
    p = W.random_problem(504, R=150, Hq=8, Hkv=2, D=128, N=500, kv_dtype=torch.bfloat16,
                         out_dtype=torch.float32, seqs=3, causal=True, mask_frac=0.1, alibi=True,
                         sinks=True, softcap=20.0)
    check(p, run_prefill(p), "generic")


def test_deterministic(cuda_lib):
    p = W.random_prefill(505, R=300, Hq=8, Hkv=2, D=128, depth=900, causal_by="mask", bias_frac=0.05,
                         nan_v=3, alibi=True, sinks=True, softcap=40.0)
    a = run_prefill(p)
    b = run_prefill(p)
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))
    check(p, a, "bias + NaN V + ALiBi + softcap")


def test_mask_bits_tiles(cuda_lib):
    """A 0 / -inf causal mask with ALiBi, softcap and NaN V: the diagonal tiles
    take the packed path with the classifier's visibility bits, and those
    holding a NaN V run P V on the CUDA cores over the visible cells only."""
    p = W.random_prefill(506, R=300, Hq=8, Hkv=2, D=128, depth=500, causal_by="mask", nan_v=4,
                         alibi=True, sinks=True, softcap=40.0)
    out = run_prefill(p)
    ref = oracle.attn(p)
    assert np.isnan(ref).any() and np.isfinite(ref).any()
    check(p, out, "mask bits", ref=ref)


@pytest.mark.parametrize("alibi", [False, True])
def test_noncausal_zero_mask(cuda_lib, alibi):
    """A 0 / -inf mask that lets rows see cells after their own position: with
    ALiBi those tiles carry |row_pos - cell_pos| on both sides of the row."""
    p = W.random_prefill(507, R=200, Hq=4, Hkv=1, D=128, depth=300, causal_by="mask", alibi=alibi,
                         softcap=30.0)
    rng = np.random.default_rng(7)
    m = np.zeros(tuple(p.mask.shape), dtype=np.float32)
    m[rng.random(m.shape) < 0.1] = -np.inf
    p = dataclasses.replace(p, mask=torch.from_numpy(m))
    check(p, run_prefill(p), f"non-causal mask alibi={alibi}")


@pytest.fixture(scope="module")
def semantics_problem():
    p = W.semantics_sweep()
    return p, oracle.attn(p)


def test_semantics_sweep_prefill(cuda_lib, semantics_problem):
    p, ref = semantics_problem
    check(p, run_prefill(p), "semantics sweep", ref=ref)


def test_causal_prefill_workload_sampled(cuda_lib):
    """The full-size causal prefill workload against the oracle on sampled
    rows (all heads): one random row in every 128-row tile (so every unit of
    the launch, split units included, is checked), both edges of the first
    tile boundary, and the first and last rows."""
    p = W.causal_prefill()
    out = run_prefill(p)
    rng = np.random.default_rng(4)
    n_tiles = (p.n_rows + 127) // 128
    per_tile = [t * 128 + int(rng.integers(min(128, p.n_rows - t * 128))) for t in range(n_tiles)]
    rows = np.unique(np.concatenate([[0, 127, 128, p.n_rows - 1], per_tile,
                                     rng.choice(p.n_rows, size=8, replace=False)]))
    assert len(np.unique(rows // 128)) == n_tiles
    sub = p.row_subset(rows)
    check(sub, out[torch.from_numpy(rows).cuda()], "causal_prefill sample")
