"""The C-ABI library on a machine without a GPU: it loads, exports every symbol
include/attn.h declares, its argument blocks have the same layout as the
Python mirrors, and argument validation refuses bad input before any CUDA
call (no compute happens here)."""
import ctypes
import os
import re
import subprocess

import pytest

import attention_split_attn_b200 as A

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


@pytest.fixture(scope="module")
def lib():
    from attention_split_attn_b200 import build
    build.build()
    return A.load_library()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(attn_[a-z_0-9]+)\s*\(",
                                 text, flags=re.M)))


def test_every_declared_symbol_is_exported(lib):
    declared = _declared_functions()
    assert set(declared) == set(A.EXPORTS), declared
    out = subprocess.run(["nm", "-D", "--defined-only", A.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (attn_[a-z_0-9]+)$", out, flags=re.M))
    for name in declared:
        assert name in exported, name
        assert getattr(lib, name) is not None


def test_abi_version(lib):
    assert lib.attn_abi_version() == 2


def test_struct_layout_matches_header(tmp_path):
    fields = [f[0] for f in A.AttnArgs._fields_]
    sel_fields = [f[0] for f in A.AttnSelectedArgs._fields_]
    src = tmp_path / "layout.c"
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "attn.h"', "int main(void){",
             'printf("attn_args %zu\\n", sizeof(attn_args));',
             'printf("attn_selected_args %zu\\n", sizeof(attn_selected_args));']
    lines += [f'printf("a.{f} %zu\\n", offsetof(attn_args, {f}));' for f in fields]
    lines += [f'printf("s.{f} %zu\\n", offsetof(attn_selected_args, {f}));' for f in sel_fields]
    lines.append("return 0;}")
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)])
    got = dict(l.split() for l in subprocess.check_output([str(exe)], text=True).splitlines())
    assert int(got["attn_args"]) == ctypes.sizeof(A.AttnArgs)
    assert int(got["attn_selected_args"]) == ctypes.sizeof(A.AttnSelectedArgs)
    for f in fields:
        assert int(got[f"a.{f}"]) == getattr(A.AttnArgs, f).offset, f
    for f in sel_fields:
        assert int(got[f"s.{f}"]) == getattr(A.AttnSelectedArgs, f).offset, f


def _args(**over):
    a = A.AttnArgs()
    a.n_rows, a.n_head_q, a.n_head_kv, a.head_dim, a.n_cells = 2, 8, 2, 128, 1024
    a.q, a.k, a.v, a.out = 0x10000, 0x20000, 0x30000, 0x40000
    a.q_type = a.kv_type = a.out_type = A.ATTN_BF16
    a.q_stride_row, a.q_stride_head = 8 * 128, 128
    a.kv_stride_cell, a.kv_stride_head = 2 * 128, 128
    a.o_stride_row, a.o_stride_head = 8 * 128, 128
    a.scale = 0.088
    for k, v in over.items():
        setattr(a, k, v)
    return a


def test_validation_accepts_good_args(lib):
    assert lib.attn_supports(ctypes.byref(_args()), A.OP_DECODE) == 0


@pytest.mark.parametrize("over,status", [
    (dict(head_dim=96), -2),
    (dict(n_head_q=7), -1),
    (dict(n_head_q=34, n_head_kv=2), -2),      # group 17 > 16
    (dict(q_type=9), -1),
    (dict(n_slices=65), -1),
    (dict(grid_order=2), -1),
    (dict(causal=3), -1),
    (dict(k=0x20008), -2),                      # not 16-byte aligned
    (dict(kv_stride_cell=2 * 128 + 3), -2),     # stride not a multiple of 16 bytes
    (dict(q=None), -1),
    (dict(n_rows=-1), -1),
    (dict(max_row_len=-5), -1),
])
def test_validation_refuses(lib, over, status):
    a = _args(**over)
    assert lib.attn_supports(ctypes.byref(a), A.OP_DECODE) == status
    assert lib.attn_last_error()


def test_validation_pairs_and_reserved(lib):
    a = _args()
    a.row_begin = 0x50000
    assert lib.attn_supports(ctypes.byref(a), A.OP_DECODE) == -1
    a = _args()
    a.cell_seq = 0x50000
    assert lib.attn_supports(ctypes.byref(a), A.OP_DECODE) == -1
    a = _args()
    a.reserved[2] = 1
    assert lib.attn_supports(ctypes.byref(a), A.OP_DECODE) == -1


def test_bounded_wait_test_field(lib):
    """reserved[0] is the prefill kernel's bounded-wait test (microseconds,
    0..1000000); every other op and field still takes zero only."""
    a = _args(q_type=A.ATTN_BF16, kv_type=A.ATTN_BF16)
    a.reserved[0] = 1000
    assert lib.attn_supports(ctypes.byref(a), A.OP_PREFILL) == 0
    assert lib.attn_supports(ctypes.byref(a), A.OP_DECODE) == -1
    assert lib.attn_supports(ctypes.byref(a), A.OP_SELECTED) == -1
    for bad in (-1, 1000001):
        a.reserved[0] = bad
        assert lib.attn_supports(ctypes.byref(a), A.OP_PREFILL) == -1
    a.reserved[0] = 1000
    a.cell_seq, a.row_seq = 0x50000, 0x60000      # the unified-cache route has no such wait
    assert lib.attn_supports(ctypes.byref(a), A.OP_PREFILL) == -1


def test_quantized_cache_validation(lib):
    """e4m3/int8 caches: decode and prefill (with a 16-bit Q and 16-byte
    aligned codes), scales required, and only for such caches; the prefill
    workspace holds the K and V widened to the Q dtype."""
    for kv in (A.ATTN_FP8_E4M3, A.ATTN_I8):
        a = _args(kv_type=kv, kv_stride_cell=2 * 128, kv_stride_head=128)
        assert lib.attn_supports(ctypes.byref(a), A.OP_DECODE) == -1      # scales missing
        a.k_scale, a.v_scale, a.scale_stride_cell = 0x60000, 0x70000, a.n_head_kv
        assert lib.attn_supports(ctypes.byref(a), A.OP_DECODE) == 0
        assert lib.attn_supports(ctypes.byref(a), A.OP_PREFILL) == 0
        widened = 2 * a.n_cells * a.n_head_kv * a.head_dim * 2
        assert lib.attn_workspace_size(ctypes.byref(a), A.OP_PREFILL, 0) >= widened
        assert lib.attn_supports(ctypes.byref(a), A.OP_SELECTED) == -2
        b = _args(kv_type=kv, kv_stride_cell=2 * 128, kv_stride_head=128, k_scale=0x60000, v_scale=0x70000,
                  scale_stride_cell=2, q_type=A.ATTN_F32)
        assert lib.attn_supports(ctypes.byref(b), A.OP_PREFILL) == -2     # Q must be F16/BF16 here
        b = _args(kv_type=kv, kv_stride_cell=2 * 128 + 8, kv_stride_head=128, k_scale=0x60000, v_scale=0x70000,
                  scale_stride_cell=2)
        assert lib.attn_supports(ctypes.byref(b), A.OP_PREFILL) == -2     # codes not 16-byte aligned
        b = _args(kv_type=kv, kv_stride_cell=2 * 128, kv_stride_head=128, k_scale=0x60000, v_scale=0x70000,
                  scale_stride_cell=2, cell_seq=0x50000, row_seq=0x58000)
        assert lib.attn_supports(ctypes.byref(b), A.OP_PREFILL) == 0      # sequence ids: the dense path's filter
        a.scale_stride_cell = a.n_head_kv - 1
        assert lib.attn_supports(ctypes.byref(a), A.OP_DECODE) == -1
    a = _args()
    a.k_scale, a.v_scale, a.scale_stride_cell = 0x60000, 0x70000, 8
    assert lib.attn_supports(ctypes.byref(a), A.OP_DECODE) == -1          # 16/32-bit cache with scales
    a = _args(q_type=A.ATTN_FP8_E4M3)
    assert lib.attn_supports(ctypes.byref(a), A.OP_DECODE) == -2          # Q is never quantized


def test_empty_problem_is_ok(lib):
    a = _args(n_rows=0)
    assert lib.attn_decode(ctypes.byref(a), None, 0, None) == 0


def test_quantized_decode_slice_plan(lib):
    """e4m3/int8 caches on the CUDA-core grid kernel (here: an F32 query) take
    2048-cell slices: 8192-cell rows -> 4 slices, R * Hq * 4 partial records
    of D + 2 floats.  With a BF16 query the balanced tensor-core kernel takes
    them instead: the row tile prefix and one record per warp and per
    (row, KV head)."""
    a = _args(n_rows=16, n_head_q=32, n_head_kv=8, n_cells=131072, max_row_len=8192,
              kv_type=A.ATTN_FP8_E4M3, kv_stride_cell=8 * 128, kv_stride_head=128, q_type=A.ATTN_F32)
    a.k_scale, a.v_scale, a.scale_stride_cell = 0x60000, 0x70000, 8
    ws = lib.attn_workspace_size(ctypes.byref(a), A.OP_DECODE, 0)
    slots = 16 * 32 * 4
    assert ws == (slots * 128 * 4 + 255) // 256 * 256 + (slots * 2 * 4 + 255) // 256 * 256
    a.q_type = A.ATTN_BF16
    ws_tc = lib.attn_workspace_size(ctypes.byref(a), A.OP_DECODE, 0)
    tiles = (17 * 8 + 255) // 256 * 256
    records = (ws_tc - tiles) // ((128 + 2) * 4)   # (W + R * Hkv) * G, up to the 256-byte padding
    assert records >= 16 * 8 * 4 and ws_tc != ws
    a.n_slices = 3                 # a forced count still wins
    ws = lib.attn_workspace_size(ctypes.byref(a), A.OP_DECODE, 0)
    slots = 16 * 32 * 3
    assert ws == (slots * 128 * 4 + 255) // 256 * 256 + (slots * 2 * 4 + 255) // 256 * 256


def test_binding_quantized_scale_arguments(lib):
    """The binding marshals e4m3 caches with their scales and refuses malformed
    scale tensors before anything reaches the library (CPU tensors: only the
    argument block is built and validated, nothing is launched)."""
    import torch
    q = torch.zeros((2, 8, 128), dtype=torch.bfloat16)
    out = torch.zeros((2, 8, 128), dtype=torch.bfloat16)
    k = torch.zeros((64, 2, 128), dtype=torch.uint8).view(torch.float8_e4m3fn)
    v = torch.zeros((64, 2, 128), dtype=torch.uint8).view(torch.float8_e4m3fn)
    ks = torch.ones((64, 2), dtype=torch.float32)
    vs = torch.ones((64, 2), dtype=torch.float32)
    a = A.make_args(q, k, v, out, scale=0.1, k_scale=ks, v_scale=vs)
    assert a.kv_type == A.ATTN_FP8_E4M3 and a.scale_stride_cell == 2
    assert a.k_scale == ks.data_ptr() and a.v_scale == vs.data_ptr()
    assert lib.attn_supports(ctypes.byref(a), A.OP_DECODE) == 0
    assert lib.attn_supports(ctypes.byref(a), A.OP_SELECTED) == -2
    with pytest.raises(ValueError):
        A.make_args(q, k, v, out, scale=0.1, k_scale=ks)                      # v_scale missing
    with pytest.raises(ValueError):
        A.make_args(q, k, v, out, scale=0.1, k_scale=ks.double(), v_scale=vs)   # not float32
    with pytest.raises(ValueError):
        A.make_args(q, k, v, out, scale=0.1, k_scale=ks[:32], v_scale=vs[:32])  # wrong cell count
    i8 = torch.zeros((64, 2, 128), dtype=torch.int8)
    a = A.make_args(q, i8, i8.clone(), out, scale=0.1, k_scale=ks, v_scale=vs)
    assert a.kv_type == A.ATTN_I8
    a = A.make_args(q, i8, i8.clone(), out, scale=0.1)                          # scales missing
    assert lib.attn_supports(ctypes.byref(a), A.OP_DECODE) == -1


def test_strerror(lib):
    for code, name in A.STATUS.items():
        assert lib.attn_strerror(code).decode() == name


def test_decode_workspace_plan(lib):
    # split plan: R * Hq * S * (D + 2) floats, 256-byte aligned pieces
    a = _args(n_rows=16, n_head_q=32, n_head_kv=8, n_cells=131072, max_row_len=8192, n_slices=32)
    ws = lib.attn_workspace_size(ctypes.byref(a), A.OP_DECODE, 0)
    slots = 16 * 32 * 32
    expect = (slots * 128 * 4 + 255) // 256 * 256 + (slots * 2 * 4 + 255) // 256 * 256
    assert ws == expect
    a.n_slices = 1
    assert lib.attn_workspace_size(ctypes.byref(a), A.OP_DECODE, 0) == 0


def test_no_gpu_call_reports_cuda_error(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert lib.attn_decode(ctypes.byref(_args()), None, 0, None) == -4
