"""attn_decode against the FP64 oracle on a B200.

Covers the tiny FP32 decode (NMSE <= 1e-10), the GQA split-K decode at full
size, the unified-cache semantics sweep at every forced slice count, a sweep
over dtypes / head sizes / GQA groups / filters / softcap / ALiBi / sinks,
the boundary key counts of TensorFold PR #2595's kernel contract (33, 34,
8193, 32768, 32769, 32770 and the 32-cell edges), NaN-poisoned workspace and
output, strided layouts, and bit-identical results across repeated runs and
both grid orders (the contract's byte-equality gate).
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import attention_split_attn_b200 as A
from attention_split_attn_b200 import workloads as W
from parity import check, run_decode, tolerance, compare, poisoned_workspace

pytestmark = pytest.mark.gpu


def test_tiny_decode_fp32(cuda_lib):
    p = W.tiny_decode()
    ref = oracle.attn(p)
    for S in (4, 1, 2, 3):
        nmse = check(p, run_decode(p, n_slices=S), f"tiny S={S}", ref=ref)
        assert nmse <= 1e-10


@pytest.mark.parametrize("kv", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("G", [1, 3, 4, 8, 12, 16])
def test_dtype_dim_group_sweep(cuda_lib, kv, D, G):
    Hkv = 2
    seed = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}[kv] * 1000 + D * 10 + G
    p = W.random_problem(seed, R=3, Hq=G * Hkv, Hkv=Hkv, D=D, N=300,
                         kv_dtype=kv, out_dtype=kv, lengths=[300, 45, 0])
    for S in (0, 1, 5):
        check(p, run_decode(p, n_slices=S), f"{kv} D={D} G={G} S={S}")


@pytest.mark.parametrize("q_dtype,out_dtype", [(torch.float32, torch.bfloat16),
                                               (torch.bfloat16, torch.float32),
                                               (torch.float16, torch.float16)])
def test_mixed_q_out_dtypes(cuda_lib, q_dtype, out_dtype):
    p = W.random_problem(7, R=4, Hq=8, Hkv=2, D=128, N=200, kv_dtype=torch.bfloat16,
                         q_dtype=q_dtype, out_dtype=out_dtype)
    check(p, run_decode(p, n_slices=3), "mixed")


@pytest.mark.parametrize("feature", ["seq", "causal", "mask", "softcap", "alibi", "sinks", "all"])
@pytest.mark.parametrize("kv", [torch.float32, torch.bfloat16])
def test_feature_sweep(cuda_lib, feature, kv):
    f = dict(seqs=3 if feature in ("seq", "all") else 0,
             causal=feature in ("causal", "all", "alibi"),
             mask_frac=0.2 if feature in ("mask", "all") else 0.0,
             softcap=5.0 if feature in ("softcap", "all") else 0.0,
             alibi=feature in ("alibi", "all"),
             sinks=feature in ("sinks", "all"))
    p = W.random_problem(11, R=6, Hq=8, Hkv=2, D=128, N=700, kv_dtype=kv, out_dtype=torch.float32,
                         ranges=feature != "all", **f)
    ref = oracle.attn(p)
    for S in (1, 2, 7, 33):
        check(p, run_decode(p, n_slices=S), f"{feature} S={S}", ref=ref)


@pytest.mark.parametrize("length", [0, 1, 31, 32, 33, 34, 127, 128, 129, 8193, 32768, 32769, 32770])
def test_boundary_lengths(cuda_lib, length):
    N = max(length, 1) + 40
    p = W.random_problem(length, R=2, Hq=8, Hkv=2, D=128, N=N, kv_dtype=torch.bfloat16,
                         out_dtype=torch.bfloat16, lengths=[length, min(length, 16)], sinks=True)
    ref = oracle.attn(p)
    for S in (0, 1, 3, 16, 64):
        check(p, run_decode(p, n_slices=S, max_row_len=length), f"len={length} S={S}", ref=ref)


@pytest.mark.parametrize("kv", [torch.float32, torch.bfloat16])
def test_max_row_len_below_real_length(cuda_lib, kv):
    """max_row_len only sizes the slices: rows longer than it are still
    computed in full, the last slice taking the excess."""
    p = W.random_problem(77 + (kv == torch.bfloat16), R=5, Hq=8, Hkv=2, D=128, N=2000, kv_dtype=kv,
                         out_dtype=torch.float32, lengths=[2000, 1500, 700, 90, 0], sinks=True)
    ref = oracle.attn(p)
    for S in (0, 2, 5, 17, 64):
        for mrl in (1, 33, 100, 999):
            check(p, run_decode(p, n_slices=S, max_row_len=mrl), f"S={S} max_row_len={mrl}", ref=ref)


def test_launch_guard_16_rows_over_33_keys(cuda_lib):
    """TensorFold PR #2595's planted control went red at 16 rows over 33 keys
    with more slices than rows; here every slice count must stay inside the
    buffers and correct at that shape."""
    p = W.random_problem(33, R=16, Hq=8, Hkv=2, D=128, N=33, kv_dtype=torch.bfloat16,
                         out_dtype=torch.float32, ranges=False)
    ref = oracle.attn(p)
    for S in (1, 2, 17, 33, 64):
        for order in (0, 1):
            check(p, run_decode(p, n_slices=S, grid_order=order), f"S={S} order={order}", ref=ref)


def test_gqa_decode_full_size(cuda_lib):
    p = W.gqa_decode()
    ref = oracle.attn(p)
    out = run_decode(p)
    check(p, out, "gqa_decode auto S", ref=ref)
    for S in (1, 8, 32):
        check(p, run_decode(p, n_slices=S), f"gqa_decode S={S}", ref=ref)


def test_determinism_and_grid_order(cuda_lib):
    p = W.gqa_decode(n_seq=8, cap=4096)
    for S in (5, 32):
        base = run_decode(p, n_slices=S)
        again = run_decode(p, n_slices=S)
        other = run_decode(p, n_slices=S, grid_order=1)
        assert torch.equal(base.view(torch.int16), again.view(torch.int16))
        assert torch.equal(base.view(torch.int16), other.view(torch.int16))


@pytest.mark.parametrize("S", [1, 2, 3, 7, 16, 33, 64])
def test_semantics_sweep_decode(cuda_lib, S, semantics_problem):
    p, ref = semantics_problem
    check(p, run_decode(p, n_slices=S), f"semantics S={S}", ref=ref)


@pytest.fixture(scope="module")
def semantics_problem():
    p = W.semantics_sweep()
    return p, oracle.attn(p)


def test_semantics_grid_orders_bit_identical(cuda_lib, semantics_problem):
    p, _ = semantics_problem
    a = run_decode(p, n_slices=7)
    b = run_decode(p, n_slices=7, grid_order=1)
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_isolation_other_sequences(cuda_lib):
    """A sequence's output does not change, bit for bit, when every cell of
    the other sequences changes, NaN included (strix-llama.cpp PR #115,
    isolation: one conversation's output must not depend on another's)."""
    p = W.random_problem(5, R=8, Hq=8, Hkv=2, D=128, N=2000, kv_dtype=torch.float16,
                         out_dtype=torch.float32, ranges=False, seqs=4, causal=True, sinks=True)
    base = run_decode(p, n_slices=4)
    other = (p.cell_seq != 0)
    k, v = p.k.clone(), p.v.clone()
    k[other] = float("nan")
    v[other] = torch.randn_like(v[other].float()).to(v.dtype)
    q = dataclasses.replace(p, k=k, v=v)
    changed = run_decode(q, n_slices=4)
    rows0 = (p.row_seq == 0).nonzero().flatten().cuda()
    assert rows0.numel() > 0
    assert torch.equal(base[rows0].view(torch.int32), changed[rows0].view(torch.int32))


def test_strided_layouts(cuda_lib):
    """Non-contiguous Q/out rows and a head-major K/V cache."""
    p = W.random_problem(9, R=5, Hq=8, Hkv=2, D=128, N=400, kv_dtype=torch.bfloat16,
                         out_dtype=torch.float32)
    (q, k, v, out), kw = A.problem_kwargs(p)
    qpad = torch.zeros((5, 8, 256), dtype=q.dtype, device="cuda")[:, :, :128]
    qpad.copy_(q)
    kh = k.transpose(0, 1).contiguous().transpose(0, 1)     # strides (128, N*128, 1)
    vh = v.transpose(0, 1).contiguous().transpose(0, 1)
    opad = torch.full((5, 10, 128), float("nan"), dtype=out.dtype, device="cuda")[:, 1:9, :]
    A.decode(qpad, kh, vh, opad, **{**kw, "n_slices": 3})
    torch.cuda.synchronize()
    check(p, opad, "strided")


def test_workspace_too_small_is_refused(cuda_lib):
    p = W.random_problem(3, R=2, Hq=4, Hkv=1, D=64, N=300, kv_dtype=torch.float16)
    (q, k, v, out), kw = A.problem_kwargs(p)
    args = A.make_args(q, k, v, out, **{**kw, "n_slices": 4})
    need = A.workspace_size(args, A.OP_DECODE)
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    lib = A.load_library()
    import ctypes
    st = lib.attn_decode(ctypes.byref(args), ws.data_ptr(), ws.numel(),
                         torch.cuda.current_stream().cuda_stream)
    assert st == -3


# ---- the balanced persistent scheme (n_slices = 0, 16-bit cache) -----------

def test_balanced_semantics_sweep(cuda_lib, semantics_problem):
    p, ref = semantics_problem
    check(p, run_decode(p, n_slices=0), "semantics balanced", ref=ref)


def test_balanced_order_bit_identical(cuda_lib):
    """Reversing which warp takes which run changes nothing, bit for bit."""
    p = W.gqa_decode(n_seq=8, cap=4096)
    a = run_decode(p, n_slices=0)
    b = run_decode(p, n_slices=0, grid_order=1)
    c = run_decode(p, n_slices=0)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(a.view(torch.int16), c.view(torch.int16))
    check(p, a, "gqa_decode balanced")


def test_balanced_one_long_row(cuda_lib):
    """One row whose cells are spread over every resident warp (hundreds of
    records per row in the combine)."""
    p = W.random_problem(77, R=1, Hq=4, Hkv=1, D=128, N=120000, kv_dtype=torch.bfloat16,
                         out_dtype=torch.float32, ranges=False, sinks=True)
    check(p, run_decode(p, n_slices=0), "one long row")


def test_balanced_more_warps_than_tiles(cuda_lib):
    """Fewer tiles than warps: most warp runs are empty."""
    p = W.random_problem(78, R=3, Hq=8, Hkv=2, D=64, N=40, kv_dtype=torch.float16,
                         out_dtype=torch.float16, lengths=[40, 17, 0], sinks=True)
    check(p, run_decode(p, n_slices=0), "tiny balanced")
    p = W.random_problem(79, R=70, Hq=16, Hkv=1, D=256, N=300, kv_dtype=torch.bfloat16,
                         out_dtype=torch.float32, softcap=3.0)
    check(p, run_decode(p, n_slices=0), "many short rows")


@pytest.mark.parametrize("R", [63, 64, 65, 200])
def test_balanced_row_counts_around_inline_prefix(cuda_lib, R):
    """Up to 64 rows every warp computes the row tile prefix itself; above
    that a planner kernel does.  Both, with empty rows among them, and the
    second call on the same workspace, give the oracle's result."""
    rng = np.random.default_rng(R)
    lengths = [int(x) for x in rng.integers(0, 700, size=R)]
    lengths[R // 2] = 0
    p = W.random_problem(900 + R, R=R, Hq=8, Hkv=2, D=128, N=800, kv_dtype=torch.bfloat16,
                         out_dtype=torch.float32, lengths=lengths, sinks=True, causal=True)
    ref = oracle.attn(p)
    (q, k, v, out), kw = A.problem_kwargs(p)
    args = A.make_args(q, k, v, out, **kw)
    ws = poisoned_workspace(A.workspace_size(args, A.OP_DECODE))
    for _ in range(2):
        out.fill_(float("nan"))
        A.attn_decode_args(args, ws=ws)
        torch.cuda.synchronize()
        check(p, out, f"R={R}", ref=ref)
