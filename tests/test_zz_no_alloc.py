"""moba_build_index_noalloc: the block index for callers that cannot give the
library device scratch memory (a host framework that owns every byte of
device memory, or a latency-critical path that must not call cudaMalloc).

It must return what the workspace version, moba_build_index, returns (the
same bucket offsets and, per bucket, the same row ids; their order inside a
bucket is unspecified), call after call, although every call reuses the same
static scratch array.  This file is collected last on purpose; it also passes when run on
its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_long_key_b200 import moba, synth


def _noalloc_fn():
    f = moba.lib().moba_build_index_noalloc
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(moba.Shape), ctypes.c_void_p, ctypes.c_void_p,
                  ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f


def _buckets(ptr, rows):
    ptr = ptr.cpu().numpy()
    rows = rows.cpu().numpy()
    return {b: sorted(rows[ptr[b]:ptr[b + 1]].tolist()) for b in range(len(ptr) - 1) if ptr[b + 1] > ptr[b]}


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # 2^20 blocks x 16 KV heads need far more than the built-in scratch; the
    # size check comes before any device work.
    s = moba.make_shape(1 << 24, 1, 1, 1, 64, 16, 4)
    s16 = moba.make_shape(1 << 20, 1, 16, 16, 64, 16, 4)
    fake = ctypes.c_void_p(1 << 20)
    f = _noalloc_fn()
    assert f(fake, fake, ctypes.byref(s16), fake, fake, None) == moba.MOBA_EWORKSPACE
    assert f(fake, fake, ctypes.byref(s), fake, fake, None) == moba.MOBA_EWORKSPACE


@pytest.mark.gpu
def test_noalloc_index_matches_workspace_version_on_consecutive_calls():
    assert torch.cuda.is_available()
    dev = torch.device("cuda:0")
    f = _noalloc_fn()
    cases = [((3000, 17, 900), 4, 2, 64, 32, 8, 1),     # varlen, GQA, a sequence shorter than B
             ((4096,), 2, 2, 128, 64, 16, 2)]
    for seqlens, hq, hkv, d, B, topk, seed in cases:
        w = synth.small(seqlens, hq, hkv, d, B, topk, seed=seed)
        x = synth.make_inputs(w, with_dout=False)
        g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
        _, _, sel, _ = moba.forward(g["q"], g["k"], g["v"], g["cu_seqlens"], B, topk)
        ptr_ref, rows_ref = moba.build_index(sel, g["cu_seqlens"], hkv, B)
        ptr_new = torch.full_like(ptr_ref, -1)
        rows_new = torch.full_like(rows_ref, -1)
        shape = moba.make_shape(w.total_tokens, w.batch, hq, hkv, d, B, topk)
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        rc = f(ctypes.c_void_p(sel.data_ptr()), ctypes.c_void_p(g["cu_seqlens"].data_ptr()), ctypes.byref(shape),
               ctypes.c_void_p(ptr_new.data_ptr()), ctypes.c_void_p(rows_new.data_ptr()), stream)
        assert rc == moba.MOBA_OK, moba.status_string(rc)
        torch.cuda.synchronize()
        assert torch.equal(ptr_new, ptr_ref)
        assert _buckets(ptr_new, rows_new) == _buckets(ptr_ref, rows_ref)
        n = int(ptr_ref[-1].item())
        assert n == int((sel >= 0).sum().item())
        assert np.array_equal(np.sort(rows_new[:n].cpu().numpy()), np.sort(rows_ref[:n].cpu().numpy()))
