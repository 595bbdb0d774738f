"""attention_split_attn_b200 -- attention over a KV cache on B200 (sm_100a).

A thin ctypes binding over libattn_b200.so (C ABI in include/attn.h).  It only
marshals arguments: tensor pointers, strides, dtypes and the current CUDA
stream.  Every step of the computation runs in the library's kernels; there is
no fallback path.  If the library is missing or a call is refused, the call
raises.

    import attention_split_attn_b200 as A
    ws = A.workspace(args_for=...)       # or let the wrappers allocate
    A.decode(q, k, v, out, row_begin=..., row_end=..., scale=...)
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn_b200.so")

ATTN_F32, ATTN_F16, ATTN_BF16, ATTN_FP8_E4M3, ATTN_I8 = 0, 1, 2, 3, 4
OP_DECODE, OP_SELECTED, OP_PREFILL, OP_SELECTED_MASKED = 0, 1, 2, 3
STATUS = {0: "ATTN_OK", -1: "ATTN_ERR_INVALID_ARG", -2: "ATTN_ERR_UNSUPPORTED",
          -3: "ATTN_ERR_WORKSPACE", -4: "ATTN_ERR_CUDA", -5: "ATTN_ERR_DEVICE_TIMEOUT"}

_DTYPE = {torch.float32: ATTN_F32, torch.float16: ATTN_F16, torch.bfloat16: ATTN_BF16,
          torch.float8_e4m3fn: ATTN_FP8_E4M3, torch.int8: ATTN_I8}

# Every symbol include/attn.h declares.
EXPORTS = ("attn_workspace_size", "attn_supports", "attn_decode", "attn_selected",
           "attn_prefill", "attn_decode_timed", "attn_selected_timed", "attn_prefill_timed",
           "attn_decode_noalloc", "attn_tree_mask", "attn_selected_masked", "attn_selected_masked_timed",
           "attn_decode_append", "attn_decode_cluster",
           "attn_check_device_status",
           "attn_strerror", "attn_last_error", "attn_abi_version")


class AttnArgs(ctypes.Structure):
    """Mirror of attn_args (include/attn.h)."""
    _fields_ = [
        ("n_rows", ctypes.c_int32), ("n_head_q", ctypes.c_int32), ("n_head_kv", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("n_cells", ctypes.c_int32),
        ("q", ctypes.c_void_p), ("q_type", ctypes.c_int32),
        ("q_stride_row", ctypes.c_int64), ("q_stride_head", ctypes.c_int64),
        ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("kv_type", ctypes.c_int32),
        ("kv_stride_cell", ctypes.c_int64), ("kv_stride_head", ctypes.c_int64),
        ("out", ctypes.c_void_p), ("out_type", ctypes.c_int32),
        ("o_stride_row", ctypes.c_int64), ("o_stride_head", ctypes.c_int64),
        ("row_begin", ctypes.c_void_p), ("row_end", ctypes.c_void_p),
        ("cell_seq", ctypes.c_void_p), ("row_seq", ctypes.c_void_p),
        ("cell_pos", ctypes.c_void_p), ("row_pos", ctypes.c_void_p),
        ("causal", ctypes.c_int32),
        ("mask", ctypes.c_void_p), ("mask_stride_row", ctypes.c_int64),
        ("scale", ctypes.c_float), ("softcap", ctypes.c_float),
        ("alibi_slopes", ctypes.c_void_p), ("sinks", ctypes.c_void_p),
        ("n_slices", ctypes.c_int32), ("max_row_len", ctypes.c_int32),
        ("grid_order", ctypes.c_int32), ("reserved", ctypes.c_int32 * 5),
        ("k_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p), ("scale_stride_cell", ctypes.c_int64),
    ]


class AttnSelectedArgs(ctypes.Structure):
    """Mirror of attn_selected_args (include/attn.h)."""
    _fields_ = [
        ("base", AttnArgs),
        ("sel", ctypes.c_void_p), ("sel_stride_row", ctypes.c_int64), ("n_sel", ctypes.c_int32),
        ("sel_sorted_out", ctypes.c_void_p), ("sel_count_out", ctypes.c_void_p),
    ]


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str, reason: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}: {reason}")
        self.status = status


_lock = threading.Lock()
_lib = None


def load_library():
    """Load libattn_b200.so; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing: build it with "
                                  "`python -m attention_split_attn_b200.build`")
            lib = ctypes.CDLL(LIB_PATH)
            lib.attn_workspace_size.restype = ctypes.c_size_t
            lib.attn_workspace_size.argtypes = [ctypes.POINTER(AttnArgs), ctypes.c_int32, ctypes.c_int32]
            lib.attn_supports.restype = ctypes.c_int32
            lib.attn_supports.argtypes = [ctypes.POINTER(AttnArgs), ctypes.c_int32]
            for name in ("attn_decode", "attn_prefill"):
                fn = getattr(lib, name)
                fn.restype = ctypes.c_int32
                fn.argtypes = [ctypes.POINTER(AttnArgs), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
            for name in ("attn_decode_timed", "attn_prefill_timed"):
                fn = getattr(lib, name)
                fn.restype = ctypes.c_int32
                fn.argtypes = [ctypes.POINTER(AttnArgs), ctypes.c_void_p, ctypes.c_size_t,
                               ctypes.c_void_p, ctypes.c_void_p * 3]
            lib.attn_decode_noalloc.restype = ctypes.c_int32
            lib.attn_decode_noalloc.argtypes = [ctypes.POINTER(AttnArgs), ctypes.c_void_p]
            lib.attn_selected.restype = ctypes.c_int32
            lib.attn_selected.argtypes = [ctypes.POINTER(AttnSelectedArgs), ctypes.c_void_p,
                                          ctypes.c_size_t, ctypes.c_void_p]
            lib.attn_selected_timed.restype = ctypes.c_int32
            lib.attn_selected_timed.argtypes = [ctypes.POINTER(AttnSelectedArgs), ctypes.c_void_p,
                                                ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p * 3]
            for name in ("attn_selected_masked",):
                fn = getattr(lib, name)
                fn.restype = ctypes.c_int32
                fn.argtypes = [ctypes.POINTER(AttnSelectedArgs), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
            lib.attn_decode_cluster.restype = ctypes.c_int32
            lib.attn_decode_cluster.argtypes = [ctypes.POINTER(AttnArgs), ctypes.c_void_p]
            lib.attn_decode_append.restype = ctypes.c_int32
            lib.attn_decode_append.argtypes = [ctypes.POINTER(AttnArgs), ctypes.c_void_p, ctypes.c_void_p,
                                               ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t,
                                               ctypes.c_void_p]
            lib.attn_selected_masked_timed.restype = ctypes.c_int32
            lib.attn_selected_masked_timed.argtypes = [ctypes.POINTER(AttnSelectedArgs), ctypes.c_void_p,
                                                       ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p * 3]
            lib.attn_tree_mask.restype = ctypes.c_int32
            lib.attn_tree_mask.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                           ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]
            lib.attn_check_device_status.restype = ctypes.c_int32
            lib.attn_check_device_status.argtypes = [ctypes.c_void_p]
            lib.attn_strerror.restype = ctypes.c_char_p
            lib.attn_strerror.argtypes = [ctypes.c_int32]
            lib.attn_last_error.restype = ctypes.c_char_p
            lib.attn_last_error.argtypes = []
            lib.attn_abi_version.restype = ctypes.c_int32
            _lib = lib
    return _lib


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _check_i32(name, t, n):
    if t is None:
        return
    if t.dtype != torch.int32 or not t.is_cuda or t.dim() != 1 or t.stride(0) != 1 or t.numel() < n:
        raise ValueError(f"{name} must be a contiguous int32 CUDA tensor of at least {n} entries")


def make_args(q, k, v, out, *, scale, softcap=0.0, row_begin=None, row_end=None, cell_seq=None,
              row_seq=None, cell_pos=None, row_pos=None, causal=False, mask=None, alibi_slopes=None,
              sinks=None, n_slices=0, max_row_len=0, grid_order=0, k_scale=None, v_scale=None):
    """Fill an AttnArgs from CUDA tensors (q/out [R, Hq, D], k/v [N, Hkv, D]; for
    an e4m3 or int8 cache, k_scale/v_scale are float32 [N, Hkv])."""
    if q.dim() != 3 or k.dim() != 3 or v.dim() != 3 or out.dim() != 3:
        raise ValueError("q, out must be [rows, heads, dim] and k, v [cells, heads, dim]")
    if k.shape != v.shape or k.stride() != v.stride() or k.dtype != v.dtype:
        raise ValueError("k and v must share shape, strides and dtype")
    for name, t in (("q", q), ("k", k), ("out", out)):
        if t.stride(2) != 1:
            raise ValueError(f"{name}: the head dimension must be contiguous")
    R, Hq, D = q.shape
    N, Hkv, _ = k.shape
    a = AttnArgs()
    a.n_rows, a.n_head_q, a.n_head_kv, a.head_dim, a.n_cells = R, Hq, Hkv, D, N
    a.q, a.q_type, a.q_stride_row, a.q_stride_head = q.data_ptr(), _DTYPE[q.dtype], q.stride(0), q.stride(1)
    a.k, a.v, a.kv_type = k.data_ptr(), v.data_ptr(), _DTYPE[k.dtype]
    a.kv_stride_cell, a.kv_stride_head = k.stride(0), k.stride(1)
    a.out, a.out_type = out.data_ptr(), _DTYPE[out.dtype]
    a.o_stride_row, a.o_stride_head = out.stride(0), out.stride(1)
    for name, t, n in (("row_begin", row_begin, R), ("row_end", row_end, R), ("cell_seq", cell_seq, N),
                       ("row_seq", row_seq, R), ("cell_pos", cell_pos, N), ("row_pos", row_pos, R)):
        _check_i32(name, t, n)
        setattr(a, name, _ptr(t))
    a.causal = 1 if causal else 0
    if mask is not None:
        if mask.dtype != torch.float32 or mask.stride(1) != 1:
            raise ValueError("mask must be float32 with contiguous cells")
        a.mask, a.mask_stride_row = mask.data_ptr(), mask.stride(0)
    a.scale, a.softcap = float(scale), float(softcap)
    for name, t in (("alibi_slopes", alibi_slopes), ("sinks", sinks)):
        if t is not None and (t.dtype != torch.float32 or t.numel() < Hq or t.stride(0) != 1):
            raise ValueError(f"{name} must be a contiguous float32 tensor of n_head_q entries")
        setattr(a, name, _ptr(t))
    a.n_slices, a.max_row_len, a.grid_order = int(n_slices), int(max_row_len), int(grid_order)
    if (k_scale is None) != (v_scale is None):
        raise ValueError("k_scale and v_scale must both be given or both be None")
    if k_scale is not None:
        for name, t in (("k_scale", k_scale), ("v_scale", v_scale)):
            if t.dtype != torch.float32 or t.dim() != 2 or t.shape[0] != N or t.shape[1] != Hkv or t.stride(1) != 1:
                raise ValueError(f"{name} must be float32 [n_cells, n_head_kv] with contiguous heads")
        if k_scale.stride(0) != v_scale.stride(0):
            raise ValueError("k_scale and v_scale must share their cell stride")
        a.k_scale, a.v_scale, a.scale_stride_cell = k_scale.data_ptr(), v_scale.data_ptr(), k_scale.stride(0)
    return a


def _raise_if(status: int, where: str):
    if status != 0:
        lib = load_library()
        raise AttnError(status, where, lib.attn_last_error().decode())


def workspace_size(args: AttnArgs, op: int, n_sel: int = 0) -> int:
    lib = load_library()
    _raise_if(lib.attn_supports(ctypes.byref(args), op), "attn_supports")
    return int(lib.attn_workspace_size(ctypes.byref(args), op, n_sel))


def supports(args: AttnArgs, op: int) -> int:
    return int(load_library().attn_supports(ctypes.byref(args), op))


def _workspace(nbytes: int, device, ws: Optional[torch.Tensor]) -> Optional[torch.Tensor]:
    if nbytes == 0:
        return ws
    if ws is not None and ws.numel() * ws.element_size() >= nbytes and ws.data_ptr() % 256 == 0:
        return ws
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def _stream_handle(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def attn_decode_args(args: AttnArgs, ws: Optional[torch.Tensor] = None, stream=None):
    """attn_decode on a prepared AttnArgs (workspace allocated if needed)."""
    lib = load_library()
    need = workspace_size(args, OP_DECODE)
    dev = torch.device("cuda", torch.cuda.current_device())
    ws = _workspace(need, dev, ws)
    st = lib.attn_decode(ctypes.byref(args), None if ws is None else ws.data_ptr(),
                         0 if ws is None else ws.numel() * ws.element_size(), _stream_handle(stream))
    _raise_if(st, "attn_decode")
    return ws


def attn_decode_append_args(args: AttnArgs, k_new: torch.Tensor, v_new: torch.Tensor,
                            ws: Optional[torch.Tensor] = None, stream=None):
    """attn_decode with the step's cache append fused in (see include/attn.h):
    k_new / v_new [rows, n_head_kv, head_dim] in the cache dtype go to cell
    row_end[r] - 1 of the cache the AttnArgs points at."""
    for name, t in (("k_new", k_new), ("v_new", v_new)):
        if t.dim() != 3 or t.stride(2) != 1 or t.dtype not in _DTYPE:
            raise ValueError(f"{name} must be [rows, n_head_kv, head_dim] with the head dimension contiguous")
    if k_new.stride() != v_new.stride():
        raise ValueError("k_new and v_new must share strides")
    lib = load_library()
    need = workspace_size(args, OP_DECODE)
    dev = torch.device("cuda", torch.cuda.current_device())
    ws = _workspace(need, dev, ws)
    st = lib.attn_decode_append(ctypes.byref(args), k_new.data_ptr(), v_new.data_ptr(), k_new.stride(0),
                                k_new.stride(1), None if ws is None else ws.data_ptr(),
                                0 if ws is None else ws.numel() * ws.element_size(), _stream_handle(stream))
    _raise_if(st, "attn_decode_append")
    return ws


def attn_decode_cluster_args(args: AttnArgs, stream=None):
    """attn_decode through one 16-CTA cluster per (row, KV head), partials folded
    over distributed shared memory (no workspace; see include/attn.h)."""
    lib = load_library()
    _raise_if(lib.attn_decode_cluster(ctypes.byref(args), _stream_handle(stream)), "attn_decode_cluster")


def attn_decode_timed_args(args: AttnArgs, ws: Optional[torch.Tensor], events, stream=None):
    """attn_decode that also records three torch.cuda.Events (before the slice
    kernel, after it, after split_k_reduce) on the launching stream."""
    lib = load_library()
    handles = [None if e is None else e.cuda_event for e in events]
    if any(h == 0 for h in handles):
        raise ValueError("record each torch.cuda.Event once before passing it (torch creates it lazily)")
    ev = (ctypes.c_void_p * 3)(*handles)
    st = lib.attn_decode_timed(ctypes.byref(args), None if ws is None else ws.data_ptr(),
                               0 if ws is None else ws.numel() * ws.element_size(),
                               _stream_handle(stream), ev)
    _raise_if(st, "attn_decode_timed")


def decode(q, k, v, out, *, ws=None, stream=None, **kw):
    """Split-K decode attention into `out` (see include/attn.h)."""
    return attn_decode_args(make_args(q, k, v, out, **kw), ws=ws, stream=stream)


def attn_prefill_args(args: AttnArgs, ws: Optional[torch.Tensor] = None, stream=None):
    """attn_prefill on a prepared AttnArgs (workspace allocated if needed)."""
    lib = load_library()
    need = workspace_size(args, OP_PREFILL)
    dev = torch.device("cuda", torch.cuda.current_device())
    ws = _workspace(need, dev, ws)
    st = lib.attn_prefill(ctypes.byref(args), None if ws is None else ws.data_ptr(),
                          0 if ws is None else ws.numel() * ws.element_size(), _stream_handle(stream))
    _raise_if(st, "attn_prefill")
    return ws


def attn_prefill_timed_args(args: AttnArgs, ws: Optional[torch.Tensor], events, stream=None):
    """attn_prefill that also records three torch.cuda.Events (before the tile
    classifier, after the tensor-core kernel, after the last kernel)."""
    lib = load_library()
    handles = [None if e is None else e.cuda_event for e in events]
    if any(h == 0 for h in handles):
        raise ValueError("record each torch.cuda.Event once before passing it (torch creates it lazily)")
    ev = (ctypes.c_void_p * 3)(*handles)
    st = lib.attn_prefill_timed(ctypes.byref(args), None if ws is None else ws.data_ptr(),
                                0 if ws is None else ws.numel() * ws.element_size(),
                                _stream_handle(stream), ev)
    _raise_if(st, "attn_prefill_timed")


def prefill(q, k, v, out, *, ws=None, stream=None, **kw):
    """Causal prefill attention into `out` (see include/attn.h)."""
    return attn_prefill_args(make_args(q, k, v, out, **kw), ws=ws, stream=stream)


def make_selected_args(q, k, v, out, sel, *, sorted_out=None, count_out=None, **kw):
    """Fill an AttnSelectedArgs: `sel` is an int32 CUDA tensor [rows, n_sel]
    (row stride may exceed n_sel); sorted_out [rows, n_sel] and count_out
    [rows] are optional int32 outputs of the compaction."""
    for key in ("row_begin", "row_end", "cell_seq", "row_seq", "mask"):
        if kw.get(key) is not None:
            raise ValueError(f"selected-key attention takes no {key}")
    if kw.get("causal"):
        raise ValueError("selected-key attention is maskless (causal must be False)")
    a = AttnSelectedArgs()
    a.base = make_args(q, k, v, out, **kw)
    if sel.dtype != torch.int32 or not sel.is_cuda or sel.dim() != 2 or sel.stride(1) != 1:
        raise ValueError("sel must be an int32 CUDA tensor [rows, n_sel] with contiguous entries")
    a.sel, a.sel_stride_row, a.n_sel = sel.data_ptr(), sel.stride(0), sel.shape[1]
    for name, t, shape in (("sorted_out", sorted_out, tuple(sel.shape)), ("count_out", count_out, (sel.shape[0],))):
        if t is not None and (t.dtype != torch.int32 or not t.is_cuda or tuple(t.shape) != shape
                              or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous int32 CUDA tensor of shape {shape}")
    a.sel_sorted_out = _ptr(sorted_out)
    a.sel_count_out = _ptr(count_out)
    return a


def attn_selected_args(args: AttnSelectedArgs, ws: Optional[torch.Tensor] = None, stream=None):
    """attn_selected on a prepared AttnSelectedArgs (workspace allocated if needed)."""
    lib = load_library()
    _raise_if(lib.attn_supports(ctypes.byref(args.base), OP_SELECTED), "attn_supports")
    need = int(lib.attn_workspace_size(ctypes.byref(args.base), OP_SELECTED, args.n_sel))
    dev = torch.device("cuda", torch.cuda.current_device())
    ws = _workspace(need, dev, ws)
    st = lib.attn_selected(ctypes.byref(args), None if ws is None else ws.data_ptr(),
                           0 if ws is None else ws.numel() * ws.element_size(), _stream_handle(stream))
    _raise_if(st, "attn_selected")
    return ws


def attn_selected_timed_args(args: AttnSelectedArgs, ws: Optional[torch.Tensor], events, stream=None):
    """attn_selected that also records three torch.cuda.Events (before the
    compaction, after the gather kernel, after the combine)."""
    lib = load_library()
    handles = [None if e is None else e.cuda_event for e in events]
    if any(h == 0 for h in handles):
        raise ValueError("record each torch.cuda.Event once before passing it (torch creates it lazily)")
    ev = (ctypes.c_void_p * 3)(*handles)
    st = lib.attn_selected_timed(ctypes.byref(args), None if ws is None else ws.data_ptr(),
                                 0 if ws is None else ws.numel() * ws.element_size(),
                                 _stream_handle(stream), ev)
    _raise_if(st, "attn_selected_timed")


def attn_selected_masked_args(args: AttnSelectedArgs, ws: Optional[torch.Tensor] = None, stream=None):
    """The masked per-cell route of selected-key attention (per-cell mask + the
    dense tensor-core pass; see include/attn.h) on a prepared AttnSelectedArgs."""
    lib = load_library()
    _raise_if(lib.attn_supports(ctypes.byref(args.base), OP_SELECTED_MASKED), "attn_supports")
    need = int(lib.attn_workspace_size(ctypes.byref(args.base), OP_SELECTED_MASKED, args.n_sel))
    dev = torch.device("cuda", torch.cuda.current_device())
    ws = _workspace(need, dev, ws)
    st = lib.attn_selected_masked(ctypes.byref(args), None if ws is None else ws.data_ptr(),
                                  0 if ws is None else ws.numel() * ws.element_size(), _stream_handle(stream))
    _raise_if(st, "attn_selected_masked")
    return ws


def attn_selected_masked_timed_args(args: AttnSelectedArgs, ws: Optional[torch.Tensor], events, stream=None):
    """attn_selected_masked that also records three torch.cuda.Events (before
    the mask kernel, after the tensor-core kernel, after the last kernel)."""
    lib = load_library()
    handles = [None if e is None else e.cuda_event for e in events]
    if any(h == 0 for h in handles):
        raise ValueError("record each torch.cuda.Event once before passing it (torch creates it lazily)")
    ev = (ctypes.c_void_p * 3)(*handles)
    st = lib.attn_selected_masked_timed(ctypes.byref(args), None if ws is None else ws.data_ptr(),
                                        0 if ws is None else ws.numel() * ws.element_size(),
                                        _stream_handle(stream), ev)
    _raise_if(st, "attn_selected_masked_timed")


def selected_masked_workspace_size(args: AttnSelectedArgs) -> int:
    lib = load_library()
    _raise_if(lib.attn_supports(ctypes.byref(args.base), OP_SELECTED_MASKED), "attn_supports")
    return int(lib.attn_workspace_size(ctypes.byref(args.base), OP_SELECTED_MASKED, args.n_sel))


def selected_workspace_size(args: AttnSelectedArgs) -> int:
    lib = load_library()
    _raise_if(lib.attn_supports(ctypes.byref(args.base), OP_SELECTED), "attn_supports")
    return int(lib.attn_workspace_size(ctypes.byref(args.base), OP_SELECTED, args.n_sel))


def selected(q, k, v, out, sel, *, ws=None, stream=None, **kw):
    """Maskless selected-key attention into `out` (see include/attn.h)."""
    return attn_selected_args(make_selected_args(q, k, v, out, sel, **kw), ws=ws, stream=stream)


def tree_mask(parent: torch.Tensor, prefix_cells: int, n_cells: int, mask: Optional[torch.Tensor] = None,
              stream=None) -> torch.Tensor:
    """The F32 mask [rows, n_cells] under which attn_decode computes draft-tree
    rows: row r is node r (token in cell prefix_cells + r, parent parent[r] <
    r or -1) and sees the prefix and its ancestors' cells (see include/attn.h)."""
    _check_i32("parent", parent, parent.numel())
    R = parent.numel()
    if mask is None:
        mask = torch.empty((R, n_cells), dtype=torch.float32, device=parent.device)
    if mask.dtype != torch.float32 or mask.stride(1) != 1 or tuple(mask.shape) != (R, n_cells):
        raise ValueError("mask must be float32 [rows, n_cells] with contiguous cells")
    lib = load_library()
    _raise_if(lib.attn_tree_mask(parent.data_ptr(), R, int(prefix_cells), int(n_cells), mask.data_ptr(),
                                 mask.stride(0), _stream_handle(stream)), "attn_tree_mask")
    return mask


def check_device_status(stream=None):
    lib = load_library()
    _raise_if(lib.attn_check_device_status(_stream_handle(stream)), "attn_check_device_status")


# ----------------------------------------------------------------------------
# Moving a workloads.Problem to the device (inputs for tests and the benchmark)
# ----------------------------------------------------------------------------

def problem_kwargs(p, device="cuda", out=None):
    """Device tensors and keyword arguments for a workloads.Problem."""
    dev = lambda t: None if t is None else t.to(device, non_blocking=True)
    q, k, v = dev(p.q), dev(p.k), dev(p.v)
    if out is None:
        out = torch.empty((p.n_rows, p.n_head_q, p.head_dim), dtype=p.out_dtype, device=device)
    kw = dict(scale=p.scale, softcap=p.softcap, row_begin=dev(p.row_begin), row_end=dev(p.row_end),
              cell_seq=dev(p.cell_seq), row_seq=dev(p.row_seq), cell_pos=dev(p.cell_pos),
              row_pos=dev(p.row_pos), causal=p.causal, mask=dev(p.mask),
              alibi_slopes=dev(p.alibi_slopes), sinks=dev(p.sinks), n_slices=p.n_slices,
              max_row_len=p.max_row_len)
    if p.k_scale is not None:
        kw["k_scale"], kw["v_scale"] = dev(p.k_scale), dev(p.v_scale)
    if p.sel is not None:
        for key in ("row_begin", "row_end", "cell_seq", "row_seq", "mask", "causal", "max_row_len"):
            kw.pop(key)
        kw["sel"] = dev(p.sel)
    return (q, k, v, out), kw
