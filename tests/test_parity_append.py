"""attn_decode_append (the step's K/V cache append fused into the decode
launch, TensorFold PR #985's change list) on a B200: the new K/V rows land in
cell row_end - 1 and the same launch attends over them.  The output and the
cache must equal, bit for bit, a separate append followed by attn_decode, and
the output must match the FP64 oracle over the updated cache.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import attention_split_attn_b200 as A
from attention_split_attn_b200 import workloads as W
from parity import check, poisoned_workspace

pytestmark = pytest.mark.gpu


def _new_rows(p, seed):
    rng = np.random.default_rng(seed)
    shape = (p.n_rows, p.n_head_kv, p.head_dim)
    mk = lambda: torch.from_numpy(rng.standard_normal(shape, dtype=np.float32)).to(p.k.dtype)
    return mk(), mk()


def _run(p, k_new, v_new, fused):
    (q, k, v, out), kw = A.problem_kwargs(p)
    out.fill_(float("nan"))
    args = A.make_args(q, k, v, out, **kw)
    ws = poisoned_workspace(A.workspace_size(args, A.OP_DECODE))
    kn, vn = k_new.cuda(), v_new.cuda()
    if fused:
        A.attn_decode_append_args(args, kn, vn, ws=ws)
    else:
        ends = (p.row_end.tolist() if p.row_end is not None else [p.n_cells] * p.n_rows)
        for r, e in enumerate(ends):
            k[e - 1] = kn[r]
            v[e - 1] = vn[r]
        A.attn_decode_args(args, ws=ws)
    torch.cuda.synchronize()
    A.check_device_status()
    return out, k, v


@pytest.mark.parametrize("D,G", [(128, 4), (64, 8), (256, 2), (128, 16)])
def test_fused_append_equals_append_then_decode(cuda_lib, D, G):
    p = W.random_problem(900 + D + G, R=6, Hq=2 * G, Hkv=2, D=D, N=3000, kv_dtype=torch.bfloat16,
                         out_dtype=torch.bfloat16, lengths=[3000, 1200, 977, 64, 17, 1], sinks=True)
    # rows of separate sequences: give each row its own stretch of the cache
    begins, ends, b = [], [], 0
    for r in range(p.n_rows):
        n = [1500, 600, 500, 250, 100, 50][r]
        begins.append(b)
        ends.append(b + n)
        b += n
    p.row_begin = torch.tensor(begins, dtype=torch.int32)
    p.row_end = torch.tensor(ends, dtype=torch.int32)
    k_new, v_new = _new_rows(p, D + G)
    o_ref, k_ref, v_ref = _run(p, k_new, v_new, fused=False)
    o_fus, k_fus, v_fus = _run(p, k_new, v_new, fused=True)
    assert torch.equal(k_fus.view(torch.int16), k_ref.view(torch.int16))
    assert torch.equal(v_fus.view(torch.int16), v_ref.view(torch.int16))
    assert torch.equal(o_fus.view(torch.int16), o_ref.view(torch.int16))
    upd = dataclasses.replace(p, k=k_ref.cpu(), v=v_ref.cpu())
    check(upd, o_fus, f"append D={D} G={G}")


def test_single_row_whole_cache(cuda_lib):
    """One row, no ranges: the new token goes to the last cell."""
    p = W.random_problem(950, R=1, Hq=8, Hkv=1, D=128, N=4097, kv_dtype=torch.float16,
                         out_dtype=torch.float32, ranges=False, causal=True, alibi=True, positions="none")
    k_new, v_new = _new_rows(p, 5)
    o_ref, k_ref, v_ref = _run(p, k_new, v_new, fused=False)
    o_fus, k_fus, v_fus = _run(p, k_new, v_new, fused=True)
    assert torch.equal(k_fus.view(torch.int16), k_ref.view(torch.int16))
    assert torch.equal(v_fus.view(torch.int16), v_ref.view(torch.int16))
    assert torch.equal(o_fus.view(torch.int32), o_ref.view(torch.int32))
    check(dataclasses.replace(p, k=k_ref.cpu(), v=v_ref.cpu()), o_fus, "single row")


# ---- cluster decode (the other half of the same change list) ----------------

def _run_cluster(p):
    (q, k, v, out), kw = A.problem_kwargs(p)
    out.fill_(float("nan"))
    args = A.make_args(q, k, v, out, **kw)
    A.attn_decode_cluster_args(args)
    torch.cuda.synchronize()
    A.check_device_status()
    return out


@pytest.mark.parametrize("D,G,kv", [(128, 4, torch.bfloat16), (64, 8, torch.float16), (128, 16, torch.bfloat16)])
def test_cluster_decode_long_row(cuda_lib, D, G, kv):
    """One long row and a few short ones (fewer cells than the cluster's 64
    warps included), with causality, ALiBi, softcap and sinks."""
    p = W.random_problem(1200 + D + G, R=3, Hq=2 * G, Hkv=2, D=D, N=20000, kv_dtype=kv, out_dtype=torch.float32,
                         lengths=[20000, 300, 5], causal=True, alibi=True, softcap=20.0, sinks=True,
                         positions="none")
    out = _run_cluster(p)
    check(p, out, f"cluster D={D} G={G}")
    assert torch.equal(out.view(torch.int32), _run_cluster(p).view(torch.int32))   # deterministic


def test_cluster_decode_semantics(cuda_lib):
    """Masked cells, a NaN in a visible V element, an empty row and a +inf
    sink on the cluster path."""
    p = W.random_problem(1300, R=3, Hq=8, Hkv=2, D=128, N=5000, kv_dtype=torch.bfloat16,
                         out_dtype=torch.float32, lengths=[5000, 0, 2000], mask_frac=0.3, sinks=True)
    v = p.v.clone()
    v[int(p.row_begin[0]) + 17, 1, 5] = float("nan")
    p = dataclasses.replace(p, v=v)
    check(p, _run_cluster(p), "cluster semantics")
