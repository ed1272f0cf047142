"""ctypes front end of the fp64 C++ oracle (``oracle/moba_oracle.cpp``).

TEST INFRASTRUCTURE ONLY: only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It
imports nothing from the CUDA package and the package imports nothing from
here.

Same functions, arguments and results as the numpy oracle
(``oracle/moba_oracle.py``) where both exist, so that the pins in
``tests/test_oracle_pins.py`` run against both; the C++ one runs its loops
over rows and heads on every host core (OpenMP).  Extra here, for large
inputs: ``route_rows``, ``attention_rows`` and ``backward_rows`` (listed rows
only, compact [R, ...] results), ``block_grads`` (dK, dV of chosen key
blocks) and ``num_threads``.  Arrays are float64 / int64 numpy arrays in the
layouts of the numpy oracle.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence

import numpy as np

from oracle import build_oracle

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = build_oracle.build()
        L = ctypes.CDLL(path)
        P, I, L64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        sig = {
            "orc_num_threads": ([], I),
            "orc_round_bf16": ([P, P, L64], None),
            "orc_silu": ([P, P, L64], None),
            "orc_key_conv": ([P, P, I, P, I, I, I, I, I, P], None),
            "orc_block_centroids": ([P, P, I, I, I, I, I, P], None),
            "orc_route": ([P, P, P, I, I, I, I, I, I, I, P, L64, P, P], None),
            "orc_attention": ([P, P, P, P, P, I, I, I, I, I, I, I, P, L64, P, P], None),
            "orc_backward_rows": ([P, P, P, P, P, P, I, I, I, I, I, I, I, P, L64, P], None),
            "orc_attention_backward": ([P, P, P, P, P, P, I, I, I, I, I, I, I, P, P, P], None),
            "orc_block_grads": ([P, P, P, P, P, P, I, I, I, I, I, I, I, P, L64, P, P, P, P], None),
            "orc_key_conv_backward": ([P, P, I, P, I, I, I, I, P, P, P], None),
            "orc_block_index": ([P, P, I, I, I, I, I, I, P, P], L64),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def num_threads() -> int:
    """Host threads the oracle's parallel loops use."""
    return int(lib().orc_num_threads())


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i64(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.int64))


def _cu(cu_seqlens) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32).ravel())


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _rows(rows) -> Optional[np.ndarray]:
    if rows is None:
        return None
    r = _i64([(int(t), int(h)) for t, h in rows]).reshape(-1, 2)
    return r


def _nblocks(cu: np.ndarray, B: int) -> List[int]:
    return [int((b - a + B - 1) // B) for a, b in zip(cu[:-1], cu[1:])]


def round_bf16(x) -> np.ndarray:
    x = _f64(x)
    y = np.empty_like(x)
    lib().orc_round_bf16(_p(x), _p(y), x.size)
    return y


def silu(x) -> np.ndarray:
    x = _f64(x)
    y = np.empty_like(x)
    lib().orc_silu(_p(x), _p(y), x.size)
    return y


def key_conv(k, w, cu_seqlens, round_output: bool = True) -> np.ndarray:
    k, w, cu = _f64(k), _f64(w), _cu(cu_seqlens)
    T, H, d = k.shape
    out = np.empty_like(k)
    lib().orc_key_conv(_p(k), _p(w), w.shape[2], _p(cu), len(cu) - 1, T, H, d, int(round_output), _p(out))
    return out


def _centroid_table(k, cu, B) -> np.ndarray:
    T, H, d = k.shape
    nbt = sum(_nblocks(cu, B))
    cent = np.empty((H, nbt, d))
    lib().orc_block_centroids(_p(k), _p(cu), len(cu) - 1, T, H, d, B, _p(cent))
    return cent


def block_centroids(k, cu_seqlens, block_size: int) -> List[np.ndarray]:
    """One array [H_kv, n_s, d] per sequence, as the numpy oracle."""
    k, cu = _f64(k), _cu(cu_seqlens)
    cent = _centroid_table(k, cu, block_size)
    out, off = [], 0
    for n in _nblocks(cu, block_size):
        out.append(cent[:, off:off + n].copy())
        off += n
    return out


def _table_of(cents: Sequence[np.ndarray]) -> np.ndarray:
    return np.ascontiguousarray(np.concatenate([np.asarray(c, dtype=np.float64) for c in cents], axis=1))


def route_rows(q, cents, cu_seqlens, block_size: int, topk: int, rows):
    """Routing of the listed (token, head) rows only: (sel [R, topk] int64,
    gap [R]) in list order."""
    q, cu = _f64(q), _cu(cu_seqlens)
    T, hq, d = q.shape
    table = _table_of(cents)
    r = _rows(rows)
    sel = np.empty((len(r), topk), dtype=np.int64)
    gap = np.empty(len(r))
    lib().orc_route(_p(q), _p(table), _p(cu), len(cu) - 1, T, hq, table.shape[0], d, block_size, topk, _p(r),
                    len(r), _p(sel), _p(gap))
    return sel, gap


def route(q, cents, cu_seqlens, block_size: int, topk: int, rows=None):
    """(sel [T, H_q, topk] int64, gap [T, H_q]); with ``rows`` only those
    (token, head) rows are routed and other entries hold -2 / nan."""
    q, cu = _f64(q), _cu(cu_seqlens)
    T, hq, d = q.shape
    if rows is not None:
        sr, gr = route_rows(q, cents, cu, block_size, topk, rows)
        sel = np.full((T, hq, topk), -2, dtype=np.int64)
        gap = np.full((T, hq), np.nan)
        idx = tuple(_rows(rows).T)
        sel[idx], gap[idx] = sr, gr
        return sel, gap
    table = _table_of(cents)
    sel = np.empty((T, hq, topk), dtype=np.int64)
    gap = np.empty((T, hq))
    lib().orc_route(_p(q), _p(table), _p(cu), len(cu) - 1, T, hq, table.shape[0], d, block_size, topk, None, 0,
                    _p(sel), _p(gap))
    return sel, gap


def attention_rows(q, k, v, sel_rows, cu_seqlens, block_size: int, rows):
    """O [R, d] and LSE [R] of the listed (token, head) rows, each under its
    own selection ``sel_rows`` [R, topk] (list order)."""
    q, k, v, cu = _f64(q), _f64(k), _f64(v), _cu(cu_seqlens)
    s = _i64(sel_rows)
    T, hq, d = q.shape
    r = _rows(rows)
    o = np.empty((len(r), d))
    lse = np.empty(len(r))
    lib().orc_attention(_p(q), _p(k), _p(v), _p(s), _p(cu), len(cu) - 1, T, hq, k.shape[1], d, block_size,
                        s.shape[1], _p(r), len(r), _p(o), _p(lse))
    return o, lse


def attention(q, k, v, sel, cu_seqlens, block_size: int, rows=None):
    """O [T, H_q, d] and LSE [T, H_q] under ``sel`` [T, H_q, topk]; with
    ``rows`` other entries are nan."""
    q, k, v, cu = _f64(q), _f64(k), _f64(v), _cu(cu_seqlens)
    s = _i64(sel)
    T, hq, d = q.shape
    o = np.full((T, hq, d), np.nan)
    lse = np.full((T, hq), np.nan)
    if rows is not None:
        idx = tuple(_rows(rows).T)
        o[idx], lse[idx] = attention_rows(q, k, v, s[idx], cu, block_size, rows)
        return o, lse
    lib().orc_attention(_p(q), _p(k), _p(v), _p(s), _p(cu), len(cu) - 1, T, hq, k.shape[1], d, block_size,
                        s.shape[2], None, 0, _p(o), _p(lse))
    return o, lse


def attention_backward(q, k, v, dout, sel, cu_seqlens, block_size: int):
    """(dQ, dK, dV) of every row, selection fixed."""
    q, k, v, do, cu = _f64(q), _f64(k), _f64(v), _f64(dout), _cu(cu_seqlens)
    s = _i64(sel)
    T, hq, d = q.shape
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    lib().orc_attention_backward(_p(q), _p(k), _p(v), _p(do), _p(s), _p(cu), len(cu) - 1, T, hq, k.shape[1], d,
                                 block_size, s.shape[2], _p(dq), _p(dk), _p(dv))
    return dq, dk, dv


def backward_rows(q, k, v, dout, sel_rows, cu_seqlens, block_size: int, rows):
    """dQ [R, d] of the listed (token, head) rows, each under its own
    selection ``sel_rows`` [R, topk] (the numpy oracle's function of this
    name takes the full sel and also returns per-row dK/dV contributions;
    ``block_grads`` gives dK/dV here)."""
    q, k, v, do, cu = _f64(q), _f64(k), _f64(v), _f64(dout), _cu(cu_seqlens)
    s = _i64(sel_rows)
    T, hq, d = q.shape
    r = _rows(rows)
    dq = np.empty((len(r), d))
    lib().orc_backward_rows(_p(q), _p(k), _p(v), _p(do), _p(s), _p(cu), len(cu) - 1, T, hq, k.shape[1], d,
                            block_size, s.shape[1], _p(r), len(r), _p(dq))
    return dq


def block_grads(q, k, v, dout, sel, cu_seqlens, block_size: int, blocks, magnitudes: bool = False):
    """dK, dV [len(blocks), B, d] of the listed (kv_head, global block) key
    blocks under the full selection ``sel`` [T, H_q, topk]: every query row
    of the group that selected the block adds its contribution to the
    block's tokens (rows past a partial block's end are 0).  With
    ``magnitudes`` also (dk_abs, dv_abs): the magnitude sums the GPU tests
    scale their rounding tolerance by (see orc_block_grads)."""
    q, k, v, do, cu = _f64(q), _f64(k), _f64(v), _f64(dout), _cu(cu_seqlens)
    s = _i64(sel)
    T, hq, d = q.shape
    b = _i64(blocks).reshape(-1, 2)
    dk = np.empty((len(b), block_size, d))
    dv = np.empty((len(b), block_size, d))
    dka = np.empty_like(dk) if magnitudes else None
    dva = np.empty_like(dv) if magnitudes else None
    lib().orc_block_grads(_p(q), _p(k), _p(v), _p(do), _p(s), _p(cu), len(cu) - 1, T, hq, k.shape[1], d,
                          block_size, s.shape[2], _p(b), len(b), _p(dk), _p(dv), _p(dka), _p(dva))
    return (dk, dv, dka, dva) if magnitudes else (dk, dv)


def key_conv_backward(k, w, cu_seqlens, dk_conv):
    """(dK [T, H, d], dW [H, d, W]) of the key convolution."""
    k, w, cu, g = _f64(k), _f64(w), _cu(cu_seqlens), _f64(dk_conv)
    T, H, d = k.shape
    dk = np.empty_like(k)
    dw = np.empty_like(w)
    lib().orc_key_conv_backward(_p(k), _p(w), w.shape[2], _p(cu), len(cu) - 1, T, H, d, _p(g), _p(dk), _p(dw))
    return dk, dw


def block_index(sel, cu_seqlens, block_size: int, h_kv: int):
    """{(kv_head, global block): sorted list of row ids t * H_q + h}."""
    s, cu = _i64(sel), _cu(cu_seqlens)
    T, hq, topk = s.shape
    nbt = sum(_nblocks(cu, block_size))
    ptr = np.empty(h_kv * nbt + 1, dtype=np.int64)
    rows = np.empty(max(int((s >= 0).sum()), 1), dtype=np.int64)
    lib().orc_block_index(_p(s), _p(cu), len(cu) - 1, T, hq, h_kv, block_size, topk, _p(ptr), _p(rows))
    out = {}
    for b in range(h_kv * nbt):
        if ptr[b + 1] > ptr[b]:
            out[(b // nbt, b % nbt)] = rows[ptr[b]:ptr[b + 1]].tolist()
    return out
