"""Default positions on the GPU path, against the FP64 oracle on a B200.

When cell_pos / row_pos are not given, cell c of row r sits at c - row_begin[r]
and row r at row_end[r] - row_begin[r] - 1, computed from the range as the
caller gave it; a range reaching below 0 or past n_cells is clipped for
visibility only (the C ABI's "Positions" rule).  These cases drive causality
and the ALiBi distances (after the softcap, HartsyInference PR #910 "attention
semantic correctness") through those defaults on every kernel that derives
them: the balanced tensor-core decode, the (rows, heads, slices) grid at forced
slice counts (tensor-core and CUDA-core tiles), the unified-cache visible-list
route of decode and prefill, and the prefill tile classifier and tensor-core
kernel.  Rows start at nonzero and negative cells and end past the cache.
"""
import pytest
import torch

import oracle
from attention_split_attn_b200 import workloads as W
from parity import check, run_decode, run_prefill

pytestmark = pytest.mark.gpu

MODES = ["none", "row", "cell"]


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("kv", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("overhang", [0, 40])
def test_decode_default_positions(cuda_lib, mode, kv, overhang):
    seed = 5000 + MODES.index(mode) * 10 + (kv == torch.bfloat16) * 100 + overhang
    p = W.random_problem(seed, R=9, Hq=8, Hkv=2, D=128, N=600, kv_dtype=kv, out_dtype=torch.float32,
                         causal=True, alibi=True, sinks=True, softcap=8.0, positions=mode,
                         overhang=overhang, lengths=[600, 599, 377, 250, 129, 64, 33, 1, 0])
    ref = oracle.attn(p)
    for S in (0, 1, 3, 16):
        check(p, run_decode(p, n_slices=S), f"{mode} {kv} overhang={overhang} S={S}", ref=ref)


@pytest.mark.parametrize("mode", MODES)
def test_unified_route_default_positions(cuda_lib, mode):
    """Per-cell sequence ids, causal, no ALiBi: decode and prefill take the
    visible-list route, whose causal test uses the default positions."""
    p = W.random_problem(5300 + MODES.index(mode), R=12, Hq=8, Hkv=2, D=128, N=900,
                         kv_dtype=torch.float16, out_dtype=torch.float32, seqs=3, causal=True,
                         sinks=True, positions=mode, overhang=50)
    ref = oracle.attn(p)
    for S in (0, 1, 5):
        check(p, run_decode(p, n_slices=S), f"unified decode {mode} S={S}", ref=ref)
    check(p, run_prefill(p), f"unified prefill {mode}", ref=ref)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("kv", [torch.float16, torch.bfloat16])
def test_prefill_default_positions(cuda_lib, mode, kv):
    """Ranges over a 5-tile cache for 130 rows (two row tiles), so full, mixed
    and skipped tiles all meet rows whose positions come from their ranges."""
    seed = 5400 + MODES.index(mode) + (kv == torch.bfloat16) * 10
    R, N = 130, 600
    lengths = [N - (r * 7) % 300 for r in range(R)]
    p = W.random_problem(seed, R=R, Hq=4, Hkv=2, D=128, N=N, kv_dtype=kv, out_dtype=torch.float32,
                         causal=True, alibi=True, sinks=True, softcap=20.0, positions=mode,
                         overhang=30, lengths=lengths)
    check(p, run_prefill(p), f"prefill {mode} {kv}")


def test_prefill_default_positions_no_ranges(cuda_lib):
    """No row ranges at all: every row spans the cache, cell c sits at c and
    every row at n_cells - 1 (causal admits every cell; ALiBi counts back from
    the last cell)."""
    p = W.random_problem(5500, R=200, Hq=4, Hkv=1, D=64, N=333, kv_dtype=torch.bfloat16,
                         out_dtype=torch.bfloat16, ranges=False, causal=True, alibi=True,
                         positions="none")
    check(p, run_prefill(p), "prefill whole-cache defaults")
    check(p, run_decode(p, n_slices=0), "decode whole-cache defaults")
