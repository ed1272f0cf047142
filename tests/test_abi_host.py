"""Host-side checks of the C ABI: the library builds and loads without a GPU,
exports every function include/moba.h declares, sizes workspaces, and
rejects bad arguments before touching the device."""
import ctypes

import pytest

from block_sparse_long_key_b200 import build, moba


@pytest.fixture(scope="module")
def L():
    build.build()
    return moba.lib()


def test_library_exports_every_header_function(L):
    names = moba.header_functions()
    assert {"moba_forward", "moba_backward", "moba_key_conv_centroid", "moba_build_index",
            "moba_fwd_workspace_size", "moba_bwd_workspace_size", "moba_check_status",
            "moba_status_string"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for code in (0, -1, -2, -3, -4, -5):
        assert moba.status_string(code) != "unknown status"
    assert moba.status_string(-99) == "unknown status"


def _shape(**kw):
    base = dict(total_tokens=65536, batch=1, h_q=16, h_kv=16, head_dim=64, block_size=32, topk=32)
    base.update(kw)
    return moba.make_shape(**base)


def test_workspace_sizes_cover_the_buffers(L):
    s = _shape()
    T, hq, d, k = 65536, 16, 64, 32
    nb = T // 32 + 1
    fwd = moba.fwd_workspace_size(s)
    # fp32 accumulator + index rows dominate: T*hq*d*4 + T*hq*k*4 bytes
    assert fwd >= T * hq * d * 4 + T * hq * k * 4 + 16 * nb * d * 8
    bwd = moba.bwd_workspace_size(s)
    assert bwd >= T * hq * d * 4 + T * hq * k * 4
    assert fwd % 256 == 0 and bwd % 256 == 0


@pytest.mark.parametrize("bad", [dict(head_dim=96), dict(block_size=48), dict(topk=0), dict(topk=65),
                                 dict(h_q=6, h_kv=4), dict(batch=0), dict(total_tokens=-1),
                                 dict(total_tokens=1 << 28, h_q=16)])
def test_invalid_shapes_are_rejected(L, bad):
    s = _shape(**bad)
    assert moba.fwd_workspace_size(s) == 0
    assert moba.bwd_workspace_size(s) == 0
    P = ctypes.c_void_p
    fake = P(1 << 20)
    rc = L.moba_forward(fake, fake, fake, fake, ctypes.byref(s), None, 0, None, fake, fake, fake, fake, 1 << 40, None)
    assert rc == moba.MOBA_EINVAL


def test_argument_errors_return_codes_without_a_device(L):
    s = _shape(total_tokens=1024, h_q=2, h_kv=1)
    P = ctypes.c_void_p
    ok = P(1 << 20)            # 256-aligned fake device address: never dereferenced
    mis = P((1 << 20) + 8)     # 8-byte aligned only
    big = 1 << 40
    f = L.moba_forward
    assert f(None, ok, ok, ok, ctypes.byref(s), None, 0, None, ok, ok, ok, ok, big, None) == moba.MOBA_EINVAL
    assert f(mis, ok, ok, ok, ctypes.byref(s), None, 0, None, ok, ok, ok, ok, big, None) == moba.MOBA_EALIGN
    assert f(ok, ok, ok, ok, ctypes.byref(s), None, 0, None, ok, ok, ok, P((1 << 20) + 16), big, None) == \
        moba.MOBA_EALIGN
    assert f(ok, ok, ok, ok, ctypes.byref(s), None, 0, None, ok, ok, ok, ok, 1024, None) == moba.MOBA_EWORKSPACE
    # conv width without weights / out of range
    assert f(ok, ok, ok, ok, ctypes.byref(s), None, 4, ok, ok, ok, ok, ok, big, None) == moba.MOBA_EINVAL
    assert f(ok, ok, ok, ok, ctypes.byref(s), ok, 9, ok, ok, ok, ok, ok, big, None) == moba.MOBA_EINVAL
    # the conv output may not alias the keys
    assert f(ok, ok, ok, ok, ctypes.byref(s), ok, 4, ok, ok, ok, ok, ok, big, None) == moba.MOBA_EINVAL
    b = L.moba_backward
    assert b(ok, ok, ok, ok, ok, ok, ok, ok, ctypes.byref(s), ok, None, ok, ok, big, None, None) == moba.MOBA_EINVAL
    assert b(ok, ok, ok, ok, ok, ok, ok, ok, ctypes.byref(s), ok, ok, ok, ok, 16, None, None) == moba.MOBA_EWORKSPACE
    assert b(ok, ok, ok, ok, ok, ok, ok, ok, ctypes.byref(s), ok, ok, ok, ok, big, mis, None) == moba.MOBA_EALIGN
    assert L.moba_build_index(ok, ok, ctypes.byref(s), ok, None, ok, big, None) == moba.MOBA_EINVAL
    assert L.moba_key_conv_centroid(ok, None, 0, ok, ctypes.byref(s), None, None, ok, big, None) == moba.MOBA_EINVAL
    st = ctypes.c_int32(0)
    assert L.moba_check_status(None, None, ctypes.byref(st)) == moba.MOBA_EINVAL
    assert L.moba_check_path(None, None, ctypes.byref(st)) == moba.MOBA_EINVAL
    sw = L.moba_selftest_bounded_wait
    assert sw(0, ok, 256, None) == moba.MOBA_EINVAL                 # a limit of 0 ns
    assert sw(1 << 40, ok, 256, None) == moba.MOBA_EINVAL           # beyond 10 s
    assert sw(1000, ok, 16, None) == moba.MOBA_EINVAL               # workspace too small
    assert sw(1000, mis, 256, None) == moba.MOBA_EALIGN


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(8, 1, 64, dtype=torch.bfloat16)
    cu = torch.tensor([0, 8], dtype=torch.int32)
    with pytest.raises(TypeError):
        moba.forward(q, q, q, cu, 16, 1)


def test_stage_table_ignores_plans_without_a_stage(L):
    # A fake, never-dereferenced table: entry points whose plan has no stage
    # (index -1) must not read before its start.  Nothing runs on a device:
    # the call stops at the workspace check.
    arr = (ctypes.c_void_p * 4)(None, None, None, None)
    assert L.moba_set_stage_events(arr, 4) == moba.MOBA_OK
    s = _shape(total_tokens=1024, h_q=2, h_kv=1)
    ok = ctypes.c_void_p(1 << 20)
    assert L.moba_key_conv_centroid(ok, None, 0, ok, ctypes.byref(s), None, ok, ok, 16, None) == moba.MOBA_EWORKSPACE
    assert L.moba_set_stage_events(None, 0) == moba.MOBA_OK


def test_workspace_grows_linearly_with_sequence_length(L):
    # Nothing of size N x n (router scores) or N x N is held.  The only
    # term above linear is the index build's per-chunk block histogram
    # (N/1024 x N/B ints per KV head, used only while N/B <= 16384), which
    # stays a fraction of the linear pick buffer: the bytes per token grow
    # by well under 10 % per doubling of N.
    for hq, d, B, k in ((16, 64, 32, 32), (8, 128, 64, 16)):
        sizes = [moba.fwd_workspace_size(_shape(total_tokens=n, h_q=hq, h_kv=hq, head_dim=d, block_size=B, topk=k))
                 + moba.bwd_workspace_size(_shape(total_tokens=n, h_q=hq, h_kv=hq, head_dim=d, block_size=B, topk=k))
                 for n in (1 << 16, 1 << 17, 1 << 18)]
        per_tok = [sz / n for sz, n in zip(sizes, (1 << 16, 1 << 17, 1 << 18))]
        assert per_tok[1] / per_tok[0] < 1.1 and per_tok[2] / per_tok[1] < 1.1
