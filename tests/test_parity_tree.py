"""Draft-tree decode rows on a B200 (attn_tree_mask + attn_decode, and
attn_tree_mask + attn_prefill).

TensorFold PR #2595 decodes the nodes of a draft tree as the rows of one
attn_decode call (tree table with heap-order parents; its kernel contract
checks tree widths 1, 2, 4, 8, 12, 16 at 33, 34, 8193, 32768, 32769 and 32770
visible keys).  Here the visibility mask comes from the library's tree-mask
kernel; it must equal the mask the workload generator builds on the host, and
the decoded rows must match the FP64 oracle under the host mask.  The same
rows through attn_prefill take its packed-rows tiles (fewer rows than a tile:
each tile holds the rows x the q heads of one KV group), which must match the
oracle as well, at every contract shape and with several KV groups.
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

WIDTHS = [1, 2, 4, 8, 12, 16]
KEYS = [33, 34, 8193, 32768, 32769, 32770]


def decode_tree(p, n_slices=0, grid_order=0):
    (q, k, v, out), kw = A.problem_kwargs(p)
    kw.pop("mask")
    parent = p.tree_parent.cuda()
    mask = A.tree_mask(parent, p.tree_prefix, p.n_cells)
    out.fill_(float("nan"))
    args = A.make_args(q, k, v, out, mask=mask, **{**kw, "n_slices": n_slices, "grid_order": grid_order})
    ws = poisoned_workspace(A.workspace_size(args, A.OP_DECODE))
    A.attn_decode_args(args, ws=ws)
    torch.cuda.synchronize()
    A.check_device_status()
    return out, mask


@pytest.mark.parametrize("width", WIDTHS)
@pytest.mark.parametrize("visible", [33, 34, 8193])
def test_tree_mask_equals_host_mask(cuda_lib, width, visible):
    p = W.tree_decode(width=width, visible=visible, Hq=4, Hkv=1, D=64)
    mask = A.tree_mask(p.tree_parent.cuda(), p.tree_prefix, p.n_cells)
    torch.cuda.synchronize()
    assert torch.equal(mask.cpu(), p.mask)


@pytest.mark.parametrize("visible", KEYS)
@pytest.mark.parametrize("width", WIDTHS)
def test_tree_decode_contract_shapes(cuda_lib, width, visible):
    p = W.tree_decode(seed=2000 + width * 7 + visible % 97, width=width, visible=visible, Hq=8, Hkv=2, D=128)
    ref = oracle.attn(p)
    for S in (0, 7):
        out, _ = decode_tree(p, n_slices=S)
        check(p, out, f"width={width} keys={visible} S={S}", ref=ref)


def prefill_tree(p):
    (q, k, v, out), kw = A.problem_kwargs(p)
    kw.pop("mask")
    mask = A.tree_mask(p.tree_parent.cuda(), p.tree_prefix, p.n_cells)
    out.fill_(float("nan"))
    args = A.make_args(q, k, v, out, mask=mask, **kw)
    ws = poisoned_workspace(A.workspace_size(args, A.OP_PREFILL))
    A.attn_prefill_args(args, ws=ws)
    torch.cuda.synchronize()
    A.check_device_status()
    return out


@pytest.mark.parametrize("visible", KEYS)
@pytest.mark.parametrize("width", WIDTHS)
def test_tree_prefill_packed_contract_shapes(cuda_lib, width, visible):
    p = W.tree_decode(seed=2100 + width * 7 + visible % 97, width=width, visible=visible, Hq=8, Hkv=2, D=128)
    check(p, prefill_tree(p), f"prefill width={width} keys={visible}")


@pytest.mark.parametrize("D", [64, 256])
def test_tree_prefill_packed_heads_and_dims(cuda_lib, D):
    """GQA 4 and 8 groups, head dims 64 and 256, with softcap, ALiBi and
    sinks; two runs give the same bits."""
    p = W.tree_decode(seed=2200 + D, width=12, visible=5000, Hq=32, Hkv=8 if D == 64 else 4, D=D)
    p.softcap = 30.0
    p.alibi_slopes = torch.linspace(0.01, 0.2, p.n_head_q)
    p.sinks = torch.linspace(-1.0, 1.0, p.n_head_q)
    a = prefill_tree(p)
    check(p, a, f"prefill packed D={D}")
    assert torch.equal(a.view(torch.int16), prefill_tree(p).view(torch.int16))


def test_tree_prefill_full_heads_matches_decode(cuda_lib):
    """The bench's heads (32 q / 8 KV, D 128) at width 16 over 32770 keys:
    packed prefill against the oracle and against the decode route."""
    p = W.tree_decode(width=16, visible=32770)
    ref = oracle.attn(p)
    pre = prefill_tree(p)
    check(p, pre, "tree packed prefill", ref=ref)
    dec, _ = decode_tree(p)
    check(p, dec, "tree decode", ref=ref)


def test_tree_decode_full_heads_orders_bit_identical(cuda_lib):
    """The GQA decode heads (32 q / 8 KV, D 128) at width 16 over 32770 keys;
    every grid order and repeated run gives the same bits."""
    p = W.tree_decode(width=16, visible=32770)
    ref = oracle.attn(p)
    base, _ = decode_tree(p, n_slices=16)
    check(p, base, "tree full heads", ref=ref)
    for order in (0, 1):
        again, _ = decode_tree(p, n_slices=16, grid_order=order)
        assert torch.equal(base.view(torch.int16), again.view(torch.int16))
    auto, _ = decode_tree(p)
    check(p, auto, "tree full heads, balanced", ref=ref)


def test_tree_mask_rejects_a_parent_that_is_not_smaller(cuda_lib):
    """A parent index >= its child is not heap order: the kernel's own check
    stops the walk and the device status word reports it.  The nodes walked
    up to the bad link (the row itself included) stay visible; the ancestors
    above it are hidden."""
    p = W.tree_decode(width=8, visible=100, Hq=4, Hkv=1, D=64)
    parent = p.tree_parent.clone()
    parent[5] = 6
    mask = A.tree_mask(parent.cuda(), p.tree_prefix, p.n_cells)
    with pytest.raises(A.AttnError) as e:
        A.check_device_status()
    assert e.value.status == -1
    A.check_device_status()   # the status word was cleared
    row5 = mask[5].cpu()
    assert torch.all(row5[:p.tree_prefix] == 0)
    tree = row5[p.tree_prefix:p.tree_prefix + p.n_rows]
    expect = torch.full_like(tree, float("-inf"))
    expect[5] = 0.0
    assert torch.equal(tree, expect)
