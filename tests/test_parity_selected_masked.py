"""The masked per-cell route of selected-key attention against the FP64 oracle
and against attn_selected, on a B200.

strix-llama.cpp PR #115 ("Measurements") compares the selected-key kernel with
the route a backend without it takes: the selection as a dense per-cell mask
over the cache and the ordinary masked attention on it.  attn_selected_masked
builds that mask (-inf, 0 at every valid listed cell) and runs the tensor-core
prefill kernel on it.  The visible set is the same as attn_selected's, so both
must match the oracle within the same tolerances (and each other), with
duplicate and invalid entries and the list order irrelevant, and unselected
cells (NaN-poisoned here) never read.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import attention_split_attn_b200 as A
from attention_split_attn_b200 import workloads as W
from parity import check, compare, poisoned_workspace, tolerance

pytestmark = pytest.mark.gpu


def run_masked(p, **over):
    (q, k, v, out), kw = A.problem_kwargs(p)
    kw.update(over)
    sel = kw.pop("sel")
    out.fill_(float("nan"))
    args = A.make_selected_args(q, k, v, out, sel, **kw)
    ws = poisoned_workspace(A.selected_masked_workspace_size(args))
    A.attn_selected_masked_args(args, ws=ws)
    torch.cuda.synchronize()
    A.check_device_status()
    return out


def run_selected(p):
    (q, k, v, out), kw = A.problem_kwargs(p)
    sel = kw.pop("sel")
    out.fill_(float("nan"))
    args = A.make_selected_args(q, k, v, out, sel, **kw)
    ws = poisoned_workspace(A.selected_workspace_size(args))
    A.attn_selected_args(args, ws=ws)
    torch.cuda.synchronize()
    return out


def test_reduced_selected_prefill_shape(cuda_lib):
    """The selected-key workload's structure (GQA 12, head dim 256, FP16,
    lists of 4-cell causal blocks with 5% duplicates and 3% invalid entries)
    on 200 rows over 4096 cells."""
    p = W.selected_prefill(seed=71, R=200, N=4096, n_blocks=96)
    ref = oracle.attn(p)
    masked = run_masked(p)
    check(p, masked, "masked route", ref=ref)
    sel = run_selected(p)
    check(p, sel, "selected kernel", ref=ref)
    tol, max_abs = tolerance(p)
    compare(masked, sel.double().cpu().numpy(), tol, max_abs, "masked route vs selected kernel")


@pytest.mark.parametrize("feature", ["softcap", "alibi", "sinks", "all"])
@pytest.mark.parametrize("D", [128, 256])
def test_feature_sweep(cuda_lib, feature, D):
    p = W.random_selected(300 + D, R=130, Hq=8, Hkv=2, D=D, N=700, n_sel=300,
                          softcap=30.0 if feature in ("softcap", "all") else 0.0,
                          alibi=feature in ("alibi", "all"), sinks=feature in ("sinks", "all"),
                          out_dtype=torch.bfloat16)
    check(p, run_masked(p), f"{feature} D={D}")


def test_empty_lists_and_order(cuda_lib):
    """Rows whose lists hold no valid entry are +0 (or the sink's NaN); a
    permuted list gives the same bits; cells no row selected are never read."""
    p = W.random_selected(320, R=70, Hq=8, Hkv=2, D=128, N=500, n_sel=64, sinks=True)
    sel = p.sel.clone()
    sel[0] = -1
    sel[1] = 1000
    p.sel = sel
    base = run_masked(p)
    check(p, base, "empty lists")
    rng = np.random.default_rng(9)
    shuf = dataclasses.replace(p, sel=torch.from_numpy(rng.permuted(p.sel.numpy(), axis=1).copy()))
    assert torch.equal(base.view(torch.int32), run_masked(shuf).view(torch.int32))
    chosen = np.zeros(p.n_cells, dtype=bool)
    s = p.sel.numpy()
    chosen[s[(s >= 0) & (s < p.n_cells)]] = True
    k, v = p.k.clone(), p.v.clone()
    k[torch.from_numpy(~chosen)] = float("nan")
    v[torch.from_numpy(~chosen)] = float("nan")
    out = run_masked(dataclasses.replace(p, k=k, v=v))
    check(p, out, "unselected NaN cells")
