"""attn_selected against the FP64 oracle on a B200.

Maskless selected-key attention (strix-llama.cpp PR #115/#119): visibility is
the row's list alone, sorted, with invalid and duplicate entries skipped.
Covers the compaction (bit-exact against the oracle's sort + unique), parity
over dtypes / head sizes / GQA groups / softcap / ALiBi / sinks / forced row
splits, the full-size workload (sampled rows), invariance of the result --
bit for bit -- under permutation of the list and under added duplicates and
invalid entries, empty lists, NaN in unselected cells, and a full causal
list against the dense path.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import attention_split_attn_b200 as A
from attention_split_attn_b200 import workloads as W
from parity import check, poisoned_workspace, run_decode

pytestmark = pytest.mark.gpu


def run_selected(p, want_compact=False, **over):
    (q, k, v, out), kw = A.problem_kwargs(p)
    kw.update(over)
    sel = kw.pop("sel")
    out.fill_(float("nan"))
    sorted_out = count_out = None
    if want_compact:
        sorted_out = torch.full(sel.shape, 12345, dtype=torch.int32, device="cuda")
        count_out = torch.full((sel.shape[0],), -9, dtype=torch.int32, device="cuda")
    args = A.make_selected_args(q, k, v, out, sel, sorted_out=sorted_out, count_out=count_out, **kw)
    ws = poisoned_workspace(A.selected_workspace_size(args))
    A.attn_selected_args(args, ws=ws)
    torch.cuda.synchronize()
    A.check_device_status()
    return (out, sorted_out, count_out) if want_compact else out


def test_compaction_bit_exact(cuda_lib):
    rng = np.random.default_rng(8)
    N = 500
    sel = rng.integers(-30, N + 30, size=(9, 300)).astype(np.int32)
    sel[2, :] = 17                   # one value repeated
    sel[3, :] = -1                   # nothing valid
    sel[4, :] = N                    # nothing valid (past the end)
    sel[5, :] = np.arange(300)[::-1]  # already distinct, reversed
    p = W.random_selected(1, R=9, Hq=4, Hkv=1, D=64, N=N, n_sel=300)
    p.sel = torch.from_numpy(sel)
    _, srt, cnt = run_selected(p, want_compact=True)
    ref_srt, ref_cnt = oracle.select_compact(p.sel, N)
    assert np.array_equal(cnt.cpu().numpy(), ref_cnt)
    assert np.array_equal(srt.cpu().numpy(), ref_srt)


@pytest.mark.parametrize("n_sel", [1, 31, 32, 33, 1000, 4096])
def test_compaction_sizes(cuda_lib, n_sel):
    p = W.random_selected(n_sel, R=5, Hq=8, Hkv=2, D=128, N=6000, n_sel=n_sel)
    out, srt, cnt = run_selected(p, want_compact=True)
    ref_srt, ref_cnt = oracle.select_compact(p.sel, p.n_cells)
    assert np.array_equal(cnt.cpu().numpy(), ref_cnt)
    assert np.array_equal(srt.cpu().numpy(), ref_srt)
    check(p, out, f"n_sel={n_sel}")


@pytest.mark.parametrize("kv", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("G", [1, 4, 12, 16])
def test_dtype_dim_group_sweep(cuda_lib, kv, D, G):
    seed = (1 if kv == torch.float16 else 2) * 1000 + D + G
    p = W.random_selected(seed, R=5, Hq=2 * G, Hkv=2, D=D, N=700, n_sel=150, kv_dtype=kv,
                          out_dtype=torch.float32)
    ref = oracle.attn(p)
    for S in (0, 1, 3):
        check(p, run_selected(p, n_slices=S), f"{kv} D={D} G={G} S={S}", ref=ref)


@pytest.mark.parametrize("feature", ["softcap", "alibi", "sinks", "all"])
def test_feature_sweep(cuda_lib, feature):
    p = W.random_selected(21, R=6, Hq=12, Hkv=1, D=256, N=900, n_sel=400,
                          softcap=30.0 if feature in ("softcap", "all") else 0.0,
                          alibi=feature in ("alibi", "all"), sinks=feature in ("sinks", "all"),
                          out_dtype=torch.bfloat16)
    ref = oracle.attn(p)
    for S in (1, 2, 7):
        check(p, run_selected(p, n_slices=S), f"{feature} S={S}", ref=ref)


def test_empty_lists_and_sinks(cuda_lib):
    p = W.random_selected(22, R=4, Hq=8, Hkv=2, D=128, N=100, n_sel=64, sinks=True)
    sel = p.sel.clone()
    sel[0] = -1                       # empty list: sink only -> 0
    sel[1] = 1000                     # empty list
    p.sel = sel
    p.sinks = torch.tensor([0.5, -1.0, float("inf"), float("nan"), float("-inf"), 2.0, 0.0, 1.0])
    check(p, run_selected(p), "empty lists")


def test_permutation_and_duplicates_bit_identical(cuda_lib):
    p = W.random_selected(23, R=6, Hq=12, Hkv=1, D=256, N=2000, n_sel=512, dup_frac=0.2,
                          inv_frac=0.1, sinks=True)
    base = run_selected(p)
    rng = np.random.default_rng(5)
    shuf = dataclasses.replace(p, sel=torch.from_numpy(rng.permuted(p.sel.numpy(), axis=1).copy()))
    assert torch.equal(base.view(torch.int32), run_selected(shuf).view(torch.int32))
    srt, cnt = oracle.select_compact(p.sel, p.n_cells)
    clean = dataclasses.replace(p, sel=torch.from_numpy(srt))     # -1 padding is invalid
    assert torch.equal(base.view(torch.int32), run_selected(clean).view(torch.int32))
    check(p, base, "dup/perm")


def test_unselected_nan_cells_are_not_read(cuda_lib):
    p = W.random_selected(24, R=4, Hq=8, Hkv=2, D=128, N=600, n_sel=100)
    base = run_selected(p)
    chosen = np.zeros(p.n_cells, dtype=bool)
    s = p.sel.numpy()
    chosen[s[(s >= 0) & (s < p.n_cells)]] = True
    k, v = p.k.clone(), p.v.clone()
    k[torch.from_numpy(~chosen)] = float("nan")
    v[torch.from_numpy(~chosen)] = float("nan")
    out = run_selected(dataclasses.replace(p, k=k, v=v))
    assert torch.equal(base.view(torch.int32), out.view(torch.int32))


def test_full_causal_list_equals_dense(cuda_lib):
    """The full causal list gives the dense causal result (selected-key
    attention reduces to decode)."""
    rng = np.random.default_rng(25)
    N, R = 300, 4
    p = W.random_problem(25, R=R, Hq=8, Hkv=2, D=128, N=N, kv_dtype=torch.float16,
                         out_dtype=torch.float32, ranges=False, sinks=True, softcap=20.0)
    rpos = rng.integers(0, N, size=R).astype(np.int32)
    p.row_pos = torch.from_numpy(rpos)
    p.cell_pos = torch.arange(N, dtype=torch.int32)
    p.causal = True
    dense = run_decode(p, n_slices=2)
    sel = np.full((R, N), -1, dtype=np.int32)
    for r in range(R):
        sel[r, :rpos[r] + 1] = rng.permutation(rpos[r] + 1)
    ps = dataclasses.replace(p, causal=False, sel=torch.from_numpy(sel), cell_pos=None)
    sel_out = run_selected(ps)
    ref = oracle.attn(p)
    check(p, dense, "dense", ref=ref)
    check(ps, sel_out, "selected", ref=ref)


def test_selected_prefill_workload_sampled(cuda_lib):
    """The full-size selected-key workload; 48 sampled rows against the oracle,
    and the compaction of every row bit-exact."""
    p = W.selected_prefill()
    out, srt, cnt = run_selected(p, want_compact=True)
    ref_srt, ref_cnt = oracle.select_compact(p.sel, p.n_cells)
    assert np.array_equal(cnt.cpu().numpy(), ref_cnt)
    assert np.array_equal(srt.cpu().numpy(), ref_srt)
    rows = np.random.default_rng(3).choice(p.n_rows, size=48, replace=False)
    sub = p.row_subset(rows)
    check(sub, out[torch.from_numpy(rows).cuda()], "selected_prefill sample")


def test_compaction_large_cache_sort_path(cuda_lib):
    """Caches above 256K cells take the sort-and-unique compaction instead of
    the bitmap one; both must give the oracle's list bit for bit."""
    p = W.random_selected(26, R=3, Hq=4, Hkv=1, D=64, N=300000, n_sel=600, dup_frac=0.2)
    out, srt, cnt = run_selected(p, want_compact=True)
    ref_srt, ref_cnt = oracle.select_compact(p.sel, p.n_cells)
    assert np.array_equal(cnt.cpu().numpy(), ref_cnt)
    assert np.array_equal(srt.cpu().numpy(), ref_srt)
    check(p, out, "large cache")
