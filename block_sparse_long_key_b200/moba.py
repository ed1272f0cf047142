"""Thin ctypes binding of libmoba.so (include/moba.h).

Argument marshalling only: tensors are checked for device, dtype and layout,
their device pointers and the current CUDA stream are handed to the C ABI,
and every step of the computation runs in the library's kernels.  There is
no CPU or PyTorch fallback: a missing library or a non-CUDA tensor raises.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoba.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "moba.h")

MOBA_OK, MOBA_EINVAL, MOBA_EALIGN, MOBA_EWORKSPACE, MOBA_ELAUNCH, MOBA_EDEVICE = 0, -1, -2, -3, -4, -5
STATUS_BAD_SEQLENS, STATUS_BAD_SEL_IDX, STATUS_INDEX_OVERFLOW, STATUS_TIMEOUT = 1, 2, 4, 8
PATH_ROUTE_TCGEN05, PATH_FWD_TCGEN05, PATH_BWD_TCGEN05, PATH_EXACT_ROWS = 1, 2, 4, 8


class Shape(ctypes.Structure):
    _fields_ = [
        ("total_tokens", ctypes.c_int32),
        ("batch", ctypes.c_int32),
        ("h_q", ctypes.c_int32),
        ("h_kv", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("block_size", ctypes.c_int32),
        ("topk", ctypes.c_int32),
    ]


class MobaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__("%s failed: %s (%d)" % (where, status_string(code), code))


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmoba.so (built in-tree by ``block_sparse_long_key_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libmoba.so is not built (%s); run python -m block_sparse_long_key_b200.build"
                               % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        P, S, I, F = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.POINTER(Shape)
        L.moba_fwd_workspace_size.argtypes = [F]
        L.moba_fwd_workspace_size.restype = S
        L.moba_bwd_workspace_size.argtypes = [F]
        L.moba_bwd_workspace_size.restype = S
        L.moba_key_conv_centroid.argtypes = [P, P, I, P, F, P, P, P, S, P]
        L.moba_key_conv_centroid.restype = I
        L.moba_forward.argtypes = [P, P, P, P, F, P, I, P, P, P, P, P, S, P]
        L.moba_forward.restype = I
        L.moba_build_index.argtypes = [P, P, F, P, P, P, S, P]
        L.moba_build_index.restype = I
        L.moba_backward.argtypes = [P, P, P, P, P, P, P, P, F, P, P, P, P, S, P, P]
        L.moba_backward.restype = I
        L.moba_key_conv_backward.argtypes = [P, P, I, P, F, P, P, P, P, S, P]
        L.moba_key_conv_backward.restype = I
        L.moba_set_stage_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), I]
        L.moba_set_stage_events.restype = I
        L.moba_check_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_int32)]
        L.moba_check_status.restype = I
        L.moba_selftest_bounded_wait.argtypes = [ctypes.c_ulonglong, P, S, P]
        L.moba_selftest_bounded_wait.restype = I
        L.moba_check_path.argtypes = [P, P, ctypes.POINTER(ctypes.c_int32)]
        L.moba_check_path.restype = I
        L.moba_status_string.argtypes = [I]
        L.moba_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def header_functions():
    """Names of the functions include/moba.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moba_[a-z_]+)\s*\(", text)))


def status_string(code: int) -> str:
    return lib().moba_status_string(int(code)).decode()


def make_shape(total_tokens, batch, h_q, h_kv, head_dim, block_size, topk) -> Shape:
    return Shape(int(total_tokens), int(batch), int(h_q), int(h_kv), int(head_dim), int(block_size), int(topk))


def fwd_workspace_size(shape: Shape) -> int:
    return int(lib().moba_fwd_workspace_size(ctypes.byref(shape)))


def bwd_workspace_size(shape: Shape) -> int:
    return int(lib().moba_bwd_workspace_size(ctypes.byref(shape)))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, name, ndim=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if ndim is not None and t.dim() != ndim:
        raise ValueError("%s must have %d dims" % (name, ndim))


def _check(rc: int, where: str):
    if rc != MOBA_OK:
        raise MobaError(rc, where)


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    # torch's allocator returns 512-byte aligned blocks; the ABI asks for 256.
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def shape_of(q: torch.Tensor, k: torch.Tensor, cu_seqlens: torch.Tensor, block_size: int, topk: int) -> Shape:
    T, hq, d = q.shape
    return make_shape(T, cu_seqlens.numel() - 1, hq, k.shape[1], d, block_size, topk)


def key_conv_centroid(k, cu_seqlens, block_size, conv_w=None, workspace=None, h_q=None):
    """Returns (k', centroid [h_kv, T//B + batch, d] fp32); k' is None without conv."""
    _need(k, torch.bfloat16, "k", 3)
    _need(cu_seqlens, torch.int32, "cu_seqlens", 1)
    T, hkv, d = k.shape
    shape = make_shape(T, cu_seqlens.numel() - 1, h_q or hkv, hkv, d, block_size, 1)
    width = 0
    k_out = None
    if conv_w is not None:
        _need(conv_w, torch.float32, "conv_w", 3)
        width = conv_w.shape[2]
        k_out = torch.empty_like(k)
    nb = T // block_size + shape.batch
    cent = torch.empty((hkv, nb, d), dtype=torch.float32, device=k.device)
    ws = workspace if workspace is not None else alloc_workspace(fwd_workspace_size(shape), k.device)
    rc = lib().moba_key_conv_centroid(_ptr(k), _ptr(conv_w), width, _ptr(cu_seqlens), ctypes.byref(shape),
                                      _ptr(k_out), _ptr(cent), _ptr(ws), ws.numel(), _stream())
    _check(rc, "moba_key_conv_centroid")
    return k_out, cent


def forward(q, k, v, cu_seqlens, block_size: int, topk: int, conv_w=None, workspace=None,
            out=None, lse=None, sel_idx=None, k_conv=None):
    """MoBA forward.  Returns (out, lse, sel_idx, k_used) where k_used is k'
    when ``conv_w`` is given (pass it to ``backward``), else k."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n, 3)
    _need(cu_seqlens, torch.int32, "cu_seqlens", 1)
    shape = shape_of(q, k, cu_seqlens, block_size, topk)
    T, hq, d = q.shape
    dev = q.device
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((T, hq), dtype=torch.float32, device=dev) if lse is None else lse
    sel_idx = torch.empty((T, hq, topk), dtype=torch.int32, device=dev) if sel_idx is None else sel_idx
    width = 0
    if conv_w is not None:
        _need(conv_w, torch.float32, "conv_w", 3)
        width = conv_w.shape[2]
        k_conv = torch.empty_like(k) if k_conv is None else k_conv
    else:
        k_conv = None
    ws = workspace if workspace is not None else alloc_workspace(fwd_workspace_size(shape), dev)
    rc = lib().moba_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), ctypes.byref(shape), _ptr(conv_w), width,
                            _ptr(k_conv), _ptr(out), _ptr(lse), _ptr(sel_idx), _ptr(ws), ws.numel(), _stream())
    _check(rc, "moba_forward")
    return out, lse, sel_idx, (k_conv if k_conv is not None else k)


def build_index(sel_idx, cu_seqlens, h_kv: int, block_size: int, workspace=None):
    """Returns (blk_ptr [h_kv * nblk + 1], blk_rows [T * h_q * topk]) int32."""
    _need(sel_idx, torch.int32, "sel_idx", 3)
    _need(cu_seqlens, torch.int32, "cu_seqlens", 1)
    T, hq, topk = sel_idx.shape
    shape = make_shape(T, cu_seqlens.numel() - 1, hq, h_kv, 64, block_size, topk)
    nb = T // block_size + shape.batch
    dev = sel_idx.device
    ptr = torch.empty(h_kv * nb + 1, dtype=torch.int32, device=dev)
    rows = torch.empty(max(T * hq * topk, 1), dtype=torch.int32, device=dev)
    ws = workspace if workspace is not None else alloc_workspace(bwd_workspace_size(shape), dev)
    rc = lib().moba_build_index(_ptr(sel_idx), _ptr(cu_seqlens), ctypes.byref(shape), _ptr(ptr), _ptr(rows),
                                _ptr(ws), ws.numel(), _stream())
    _check(rc, "moba_build_index")
    return ptr, rows


def backward(q, k, v, out, lse, dout, sel_idx, cu_seqlens, block_size: int, workspace=None,
             dq=None, dk=None, dv=None, fwd_workspace=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """MoBA backward with the selection fixed.  Returns (dq, dk, dv).

    ``fwd_workspace``: the workspace of the forward call that produced
    ``sel_idx`` (untouched since); its block index is reused."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _need(t, torch.bfloat16, n, 3)
    _need(lse, torch.float32, "lse", 2)
    _need(sel_idx, torch.int32, "sel_idx", 3)
    _need(cu_seqlens, torch.int32, "cu_seqlens", 1)
    topk = sel_idx.shape[2]
    shape = shape_of(q, k, cu_seqlens, block_size, topk)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    ws = workspace if workspace is not None else alloc_workspace(bwd_workspace_size(shape), q.device)
    rc = lib().moba_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(sel_idx),
                             _ptr(cu_seqlens), ctypes.byref(shape), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(),
                             _ptr(fwd_workspace), _stream())
    _check(rc, "moba_backward")
    return dq, dk, dv


STAGES = ["fwd_plan", "fwd_centroid", "fwd_route", "fwd_index", "fwd_attn", "fwd_finalize",
          "bwd_plan", "bwd_index", "bwd_pre", "bwd_attn", "bwd_dq", "conv_bwd"]


class StageEvents:
    """Installs a per-stage CUDA event table on this thread (see
    moba_set_stage_events); ``ms()`` returns {stage: milliseconds}."""

    def __init__(self):
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * len(STAGES))]
        for e in self.events:   # torch creates the CUDA event on its first record
            e.record()
        self._arr = (ctypes.c_void_p * len(self.events))(*[e.cuda_event for e in self.events])

    def __enter__(self):
        _check(lib().moba_set_stage_events(self._arr, len(self.events)), "moba_set_stage_events")
        return self

    def __exit__(self, *exc):
        lib().moba_set_stage_events(None, 0)

    def ms(self):
        return {n: self.events[2 * i].elapsed_time(self.events[2 * i + 1]) for i, n in enumerate(STAGES)}


def key_conv_backward(k, conv_w, cu_seqlens, block_size: int, dk_conv, workspace=None, dk=None, dw=None, h_q=None):
    """Gradients of the key conv: (dK of the original keys, dW [h_kv, d, W])."""
    _need(k, torch.bfloat16, "k", 3)
    _need(dk_conv, torch.bfloat16, "dk_conv", 3)
    _need(conv_w, torch.float32, "conv_w", 3)
    _need(cu_seqlens, torch.int32, "cu_seqlens", 1)
    T, hkv, d = k.shape
    shape = make_shape(T, cu_seqlens.numel() - 1, h_q or hkv, hkv, d, block_size, 1)
    dk = torch.empty_like(k) if dk is None else dk
    dw = torch.empty_like(conv_w) if dw is None else dw
    ws = workspace if workspace is not None else alloc_workspace(bwd_workspace_size(shape), k.device)
    rc = lib().moba_key_conv_backward(_ptr(k), _ptr(conv_w), conv_w.shape[2], _ptr(cu_seqlens), ctypes.byref(shape),
                                      _ptr(dk_conv), _ptr(dk), _ptr(dw), _ptr(ws), ws.numel(), _stream())
    _check(rc, "moba_key_conv_backward")
    return dk, dw


def check_status(workspace: torch.Tensor) -> int:
    """Synchronises the current stream and returns the device status bits."""
    st = ctypes.c_int32(0)
    rc = lib().moba_check_status(_ptr(workspace), _stream(), ctypes.byref(st))
    if rc not in (MOBA_OK, MOBA_EDEVICE):
        raise MobaError(rc, "moba_check_status")
    return int(st.value)


def check_path(workspace: torch.Tensor) -> int:
    """Synchronises the current stream and returns the kernel-path bits
    (PATH_*) the last call on ``workspace`` set."""
    st = ctypes.c_int32(0)
    _check(lib().moba_check_path(_ptr(workspace), _stream(), ctypes.byref(st)), "moba_check_path")
    return int(st.value)


def selftest_bounded_wait(limit_ns: int, workspace: torch.Tensor) -> None:
    """Runs the bounded-wait self-test kernel (see moba_selftest_bounded_wait)
    on the current stream; read the outcome with ``check_status``."""
    _check(lib().moba_selftest_bounded_wait(int(limit_ns), _ptr(workspace), workspace.numel(), _stream()),
           "moba_selftest_bounded_wait")
