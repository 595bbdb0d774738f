"""attn_decode_noalloc through the C ABI.

Some callers cannot allocate device memory: a real-time decode loop that must
never block in an allocator, a plugin that owns no memory pool, or code that
only ever receives pointers to its inputs and outputs.  For them the library
keeps the split partials in one built-in device array instead of a caller
workspace.  These checks call that entry point directly and compare its
output with attn_decode's (same inputs, the parity tolerance), on two calls
in a row -- the second call finds the array as the first one left it -- and
check that a problem too large for the array is refused rather than launched.

This file sorts last so that a run stopping at the first failure has already
run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import pytest
import torch

import attention_split_attn_b200 as A
from attention_split_attn_b200 import workloads as W
from parity import compare, tolerance

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 << 20


def _stream():
    return torch.cuda.current_stream().cuda_stream


@pytest.mark.parametrize("case", ["gqa_decode", "unified_cache"])
def test_no_alloc_matches_decode_on_two_calls(cuda_lib, case):
    lib = A.load_library()
    if case == "gqa_decode":
        p = W.gqa_decode(n_seq=8, cap=2048)
    else:
        p = W.random_problem(5, R=6, Hq=8, Hkv=2, D=128, N=900, kv_dtype=torch.float16,
                             out_dtype=torch.float32, ranges=False, seqs=2, causal=True,
                             sinks=True)
    (q, k, v, out), kw = A.problem_kwargs(p)
    A.decode(q, k, v, out, **kw)                     # the workspace entry point
    torch.cuda.synchronize()
    ref = out.double().cpu().numpy()

    got = torch.empty_like(out)
    args = A.make_args(q, k, v, got, **kw)
    assert lib.attn_workspace_size(ctypes.byref(args), A.OP_DECODE, 0) <= SCRATCH_BYTES
    nmse_tol, max_abs = tolerance(p)
    for call in range(2):
        got.fill_(float("nan"))
        st = lib.attn_decode_noalloc(ctypes.byref(args), _stream())
        assert st == 0, lib.attn_last_error().decode()
        torch.cuda.synchronize()
        compare(got, ref, nmse_tol, max_abs, f"{case}, call {call + 1}")
    A.check_device_status()


def test_no_alloc_refuses_a_problem_larger_than_its_scratch(cuda_lib):
    lib = A.load_library()
    R, Hq, Hkv, D, N = 2048, 64, 8, 256, 64
    q = torch.zeros((R, Hq, D), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((N, Hkv, D), dtype=torch.bfloat16, device="cuda")
    v = torch.zeros_like(k)
    out = torch.full((R, Hq, D), 7.0, dtype=torch.bfloat16, device="cuda")
    args = A.make_args(q, k, v, out, scale=0.0625)
    assert lib.attn_workspace_size(ctypes.byref(args), A.OP_DECODE, 0) > SCRATCH_BYTES
    st = lib.attn_decode_noalloc(ctypes.byref(args), _stream())
    assert st == -3, st
    assert str(SCRATCH_BYTES) in lib.attn_last_error().decode()
    torch.cuda.synchronize()
    assert bool((out == 7.0).all()), "a refused call must not launch"
