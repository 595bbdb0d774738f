"""FP64 CPU oracle for attention over a KV cache -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's
``cpu_baseline`` / ``--impl reference`` legs may import this package.  The
product (``attention_split_attn_b200``) never imports it and shares no code
with it: the only thing both sides use is the seeded input generator module
``attention_split_attn_b200.workloads``, which holds no attention arithmetic.

The C library (``oracle.c``) is compiled with gcc, without fast-math, the
first time it is needed (or by ``build()``).  Inputs are widened exactly to
float64 here (every f16/bf16/f32 value is exactly representable in f64); the
codes of an e4m3 or int8 cache are dequantized here as code times the cell's
and KV head's scale, in float64, before the C definition sees them.  The
result is returned in float64, before any rounding to an output dtype.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_HDR = os.path.join(_HERE, "oracle.h")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

# Planted mistakes (names as in oracle.c); only the mutation tests use them.
MUTATIONS = {
    "alibi_before_softcap": 1, "sink_not_in_sum": 2, "alibi_sign": 3, "nan_dropped": 4,
    "empty_row_nan": 5, "gqa_modulo": 6, "no_dedup": 7, "mask_narrowed": 8,
    "invalid_clamped": 9, "scale_after_cap": 10, "neg_inf_mask_added": 11,
    "causal_strict": 12, "seq_ignored": 13, "k_d_reversed": 14,
    "cell_pos_no_begin": 15, "row_pos_no_minus1": 16, "pos_from_clipped": 17,
    # planted in the dequantization of e4m3 / int8 caches below (Python side)
    "e4m3_bias_8": 101, "e4m3_nan_as_number": 102, "scale_cells_reversed": 103,
    "scale_heads_reversed": 104, "k_scale_for_v": 105, "int8_as_unsigned": 106,
}
_py_mutation = 0   # the planted dequantization mistake in force (0: none)


def build(force: bool = False) -> str:
    """Compile liboracle.so if it is missing or older than its sources."""
    stale = (not os.path.exists(_LIB) or
             os.path.getmtime(_LIB) < max(os.path.getmtime(_SRC), os.path.getmtime(_HDR)))
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-pthread",
                               "-Wall", "-Wextra", "-Wno-unused-parameter",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Problem(ctypes.Structure):
    _fields_ = [
        ("n_rows", ctypes.c_int32), ("n_head_q", ctypes.c_int32),
        ("n_head_kv", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("n_cells", ctypes.c_int32),
        ("q", ctypes.c_void_p), ("q_stride_row", ctypes.c_int64), ("q_stride_head", ctypes.c_int64),
        ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("kv_stride_cell", ctypes.c_int64), ("kv_stride_head", ctypes.c_int64),
        ("row_begin", ctypes.c_void_p), ("row_end", ctypes.c_void_p),
        ("cell_seq", ctypes.c_void_p), ("row_seq", ctypes.c_void_p),
        ("cell_pos", ctypes.c_void_p), ("row_pos", ctypes.c_void_p),
        ("causal", ctypes.c_int32),
        ("mask", ctypes.c_void_p), ("mask_stride_row", ctypes.c_int64),
        ("scale", ctypes.c_double), ("softcap", ctypes.c_double),
        ("alibi_slopes", ctypes.c_void_p), ("sinks", ctypes.c_void_p),
        ("sel", ctypes.c_void_p), ("sel_stride_row", ctypes.c_int64), ("n_sel", ctypes.c_int32),
    ]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_attn.argtypes = [ctypes.POINTER(_Problem), ctypes.c_void_p, ctypes.c_int]
            lib.oracle_attn_split.argtypes = [ctypes.POINTER(_Problem), ctypes.c_int,
                                              ctypes.c_void_p, ctypes.c_int]
            lib.oracle_select_compact.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                                                  ctypes.c_int32, ctypes.c_int32,
                                                  ctypes.c_void_p, ctypes.c_void_p]
            lib.oracle_set_mutation.argtypes = [ctypes.c_int]
            lib.oracle_get_mutation.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(t):
    return np.ascontiguousarray(t.to(torch.float64).numpy())


def _i32(t):
    return None if t is None else np.ascontiguousarray(t.numpy().astype(np.int32))


def e4m3_value(codes: np.ndarray) -> np.ndarray:
    """float64 value of OCP FP8 E4M3 codes (uint8), from the format's definition:
    1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent 0 is
    subnormal (m/8 * 2^-6); there are no infinities, and exponent 15 with
    mantissa 7 is NaN.  (The e4m3 KV cache of TensorFold PR #911.)"""
    c = codes.astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    bias = 8 if _py_mutation == MUTATIONS["e4m3_bias_8"] else 7
    val = np.where(e == 0, np.ldexp(m / 8.0, 1 - bias), np.ldexp(1.0 + m / 8.0, e - bias))
    if _py_mutation != MUTATIONS["e4m3_nan_as_number"]:
        val = np.where((e == 15) & (c & 0x7 == 7), np.nan, val)
    return sign * val


def _kv64(t, scale):
    """A K or V cache widened to float64; an e4m3 or int8 cache is dequantized
    as code times its (cell, KV head) scale (TensorFold PR #911: one fp32 scale
    per position and key head; TensorFold PR #2595: K and V scales per key)."""
    if t.dtype == torch.float8_e4m3fn:
        code = e4m3_value(t.view(torch.uint8).numpy())
    elif t.dtype == torch.int8:
        code = t.numpy().astype(np.float64)
        if _py_mutation == MUTATIONS["int8_as_unsigned"]:
            code = t.view(torch.uint8).numpy().astype(np.float64)
    else:
        return _f64(t)
    sc = scale.numpy().astype(np.float64)
    if _py_mutation == MUTATIONS["scale_cells_reversed"]:
        sc = sc[::-1]
    if _py_mutation == MUTATIONS["scale_heads_reversed"]:
        sc = sc[:, ::-1]
    return np.ascontiguousarray(code * sc[:, :, None])


def _f32(t):
    return None if t is None else np.ascontiguousarray(t.numpy().astype(np.float32))


def _ptr(a):
    return None if a is None else a.ctypes.data


def _marshal(p):
    keep = {
        "q": _f64(p.q), "k": _kv64(p.k, p.k_scale),
        "v": _kv64(p.v, p.k_scale if _py_mutation == MUTATIONS["k_scale_for_v"] else p.v_scale),
        "row_begin": _i32(p.row_begin), "row_end": _i32(p.row_end),
        "cell_seq": _i32(p.cell_seq), "row_seq": _i32(p.row_seq),
        "cell_pos": _i32(p.cell_pos), "row_pos": _i32(p.row_pos),
        "mask": _f32(p.mask), "alibi_slopes": _f32(p.alibi_slopes),
        "sinks": _f32(p.sinks), "sel": _i32(p.sel),
    }
    R, Hq, D = p.q.shape
    N, Hkv, _ = p.k.shape
    s = _Problem()
    s.n_rows, s.n_head_q, s.n_head_kv, s.head_dim, s.n_cells = R, Hq, Hkv, D, N
    s.q, s.q_stride_row, s.q_stride_head = _ptr(keep["q"]), Hq * D, D
    s.k, s.v = _ptr(keep["k"]), _ptr(keep["v"])
    s.kv_stride_cell, s.kv_stride_head = Hkv * D, D
    for name in ("row_begin", "row_end", "cell_seq", "row_seq", "cell_pos", "row_pos",
                 "alibi_slopes", "sinks"):
        setattr(s, name, _ptr(keep[name]))
    s.causal = 1 if p.causal else 0
    s.mask = _ptr(keep["mask"])
    s.mask_stride_row = N
    s.scale, s.softcap = float(p.scale), float(p.softcap)
    s.sel = _ptr(keep["sel"])
    s.sel_stride_row = 0 if p.sel is None else p.sel.shape[1]
    s.n_sel = 0 if p.sel is None else p.sel.shape[1]
    return s, keep


class Prepared:
    """A problem already widened to float64 and laid out for the C oracle, so
    repeated evaluations (the CPU-baseline timing) measure the oracle alone."""

    def __init__(self, p):
        self.shape = (p.n_rows, p.n_head_q, p.head_dim)
        self.struct, self.keep = _marshal(p)

    def run(self, n_threads: int = 0) -> np.ndarray:
        out = np.empty(self.shape, dtype=np.float64)
        if _load().oracle_attn(ctypes.byref(self.struct), out.ctypes.data, int(n_threads)) != 0:
            raise ValueError("oracle_attn rejected the problem")
        return out


def attn(p, n_threads: int = 0) -> np.ndarray:
    """Plain-definition FP64 output [R, Hq, D] for a workloads.Problem."""
    return Prepared(p).run(n_threads)


def attn_split(p, n_slices: int, n_threads: int = 0) -> np.ndarray:
    """The same output computed as per-slice partials folded with the sink."""
    lib = _load()
    s, keep = _marshal(p)
    out = np.empty((p.n_rows, p.n_head_q, p.head_dim), dtype=np.float64)
    if lib.oracle_attn_split(ctypes.byref(s), int(n_slices), out.ctypes.data, int(n_threads)) != 0:
        raise ValueError("oracle_attn_split rejected the problem")
    return out


def select_compact(sel: torch.Tensor, n_cells: int):
    """(sorted [R, n_sel] padded with -1, count [R]) of the valid distinct entries."""
    lib = _load()
    a = _i32(sel)
    R, n_sel = a.shape
    out = np.empty((R, n_sel), dtype=np.int32)
    cnt = np.empty((R,), dtype=np.int32)
    if lib.oracle_select_compact(a.ctypes.data, n_sel, R, n_sel, int(n_cells),
                                 out.ctypes.data, cnt.ctypes.data) != 0:
        raise ValueError("oracle_select_compact rejected the input")
    return out, cnt


class mutation:
    """Context manager that plants one named mistake in the oracle."""

    def __init__(self, name: str):
        self.code = MUTATIONS[name]

    def __enter__(self):
        global _py_mutation
        if self.code >= 100:
            _py_mutation = self.code
        else:
            _load().oracle_set_mutation(self.code)
        return self

    def __exit__(self, *exc):
        global _py_mutation
        _py_mutation = 0
        _load().oracle_set_mutation(0)
        return False
