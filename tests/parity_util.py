"""Shared helpers of the GPU-vs-oracle parity tests.

Tolerances (bf16 inputs, fp32 accumulation on the GPU, fp64 oracle):

* sel_idx: bit-exact, except for queries whose last kept and first rejected
  past-block scores differ by <= 1e-3 relative; those are re-checked under
  the GPU's own selection.
* O: max-abs <= 2e-2 and mean-abs <= 1e-3; LSE: max-abs <= 1e-3.
* dQ/dK/dV, element by element: |g_gpu - g_ref| <= 4 u (s + |g_ref|) with
  u = 2^-8 (bf16 unit roundoff) and s the first-order rounding magnitude of
  that element (``grad_error_scales``), plus mean-abs <= 4e-3 * rms(g_ref).
  Derivation: the GPU rounds one factor of every product to bf16 before the
  MMAs (P for dV, dS for dQ and dK; fp32 sums), forms D_i = dO_i . O_i from
  the bf16 output O as the FlashAttention-style backward does, and rounds the
  results to bf16.  To first order that moves dQ_ic by at most
  u * (sum_t |dS_it| |k_tc| + U_i sum_t P_it |k_tc|) / sqrt(d), with
  U_i = sum_c |dO_ic O_ic| bounding the D rounding (the dS of a query sum to
  zero, so dQ can be far smaller than its terms); dK likewise with q, and
  dV by u * sum_i P_it |dO_ic|; each plus u |g| for the final rounding.  A
  numpy emulation of exactly those roundings reproduces the GPU values and
  stays within 0.45 of this bound (of 4u) on the small cases.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import moba_oracle as orc

GAP = 1e-3
O_MAX, O_MEAN, LSE_MAX = 2e-2, 1e-3, 1e-3
U_BF16 = 2.0 ** -8
G_FACTOR, G_MEAN = 4.0, 4e-3


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def selection_mismatch_rows(sel_gpu: np.ndarray, sel_ref: np.ndarray, gap: np.ndarray, rows=None):
    """Rows (t, h) whose GPU selection differs; asserts each is a near tie."""
    bad = []
    it = rows if rows is not None else [(t, h) for t in range(sel_ref.shape[0]) for h in range(sel_ref.shape[1])]
    for t, h in it:
        if not np.array_equal(sel_gpu[t, h], sel_ref[t, h]):
            assert gap[t, h] <= GAP, ("selection differs outside the near-tie band", t, h, sel_gpu[t, h],
                                      sel_ref[t, h], gap[t, h])
            bad.append((t, h))
    return bad


def check_o_lse(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    err = np.abs(o_gpu - o_ref)
    assert np.isfinite(o_gpu).all() and np.isfinite(lse_gpu).all(), what
    assert err.max() <= O_MAX, (what, "O max-abs", err.max())
    assert err.mean() <= O_MEAN, (what, "O mean-abs", err.mean())
    le = np.abs(lse_gpu - lse_ref)
    assert le.max() <= LSE_MAX, (what, "LSE max-abs", le.max())
    return err.max(), err.mean(), le.max()


def check_grad(g_gpu, g_ref, scale, what=""):
    """Element-wise rounding bound (see module docstring) + mean-abs bound."""
    rms = float(np.sqrt(np.mean(g_ref ** 2))) + 1e-30
    err = np.abs(g_gpu - g_ref)
    assert np.isfinite(g_gpu).all(), what
    bound = G_FACTOR * U_BF16 * (scale + np.abs(g_ref)) + 1e-6 * rms
    ratio = err / bound
    assert ratio.max() <= 1.0, (what, "max err / bound", ratio.max(), "max-abs/rms", err.max() / rms)
    assert err.mean() <= G_MEAN * rms, (what, "mean-abs/rms", err.mean() / rms)
    return ratio.max(), err.mean() / rms


def grad_error_scales(q, k, v, dout, sel, cu, B, lse, o):
    """First-order rounding magnitudes s of dQ, dK, dV (dense, small inputs).

    q, k, v, dout fp64 [T, H, d]; lse, o the oracle's forward results.
    """
    T, hq, d = q.shape
    g = hq // k.shape[1]
    sc = 1.0 / np.sqrt(d)
    sq, sk, sv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for a, b in zip(cu[:-1], cu[1:]):
        a, b = int(a), int(b)
        if a == b:
            continue
        for h in range(hq):
            kv = h // g
            m = orc._mask(sel, a, b, h, B)
            qq, kk, vv, do = q[a:b, h], k[a:b, kv], v[a:b, kv], dout[a:b, h]
            p = np.where(m, np.exp(qq @ kk.T * sc - lse[a:b, h][:, None]), 0.0)
            D = (do * o[a:b, h]).sum(1)
            U = np.abs(do * o[a:b, h]).sum(1)
            ds = np.abs(p * (do @ vv.T - D[:, None]))
            sq[a:b, h] = (ds @ np.abs(kk) + U[:, None] * (p @ np.abs(kk))) * sc
            sk[a:b, kv] += (ds.T @ np.abs(qq) + (p * U[:, None]).T @ np.abs(qq)) * sc
            sv[a:b, kv] += p.T @ np.abs(do)
    return sq, sk, sv


def row_dq_error_scale(q, k, v, dout, sel, cu, B, rows, o_rows, lse_rows):
    """``grad_error_scales``' dQ term for individual rows (large inputs)."""
    T, hq, d = q.shape
    g = hq // k.shape[1]
    sc = 1.0 / np.sqrt(d)
    starts = np.asarray(cu)[:-1]
    out = np.zeros((len(rows), d))
    for r, (t, h) in enumerate(rows):
        s = int(np.searchsorted(starts, t, side="right") - 1)
        vis = orc.visible_tokens(sel[t, h], t, int(cu[s]), int(cu[s + 1]), B)
        kk = np.asarray(k[vis, h // g], dtype=np.float64)
        vv = np.asarray(v[vis, h // g], dtype=np.float64)
        do = np.asarray(dout[t, h], dtype=np.float64)
        p = np.exp(kk @ q[t, h] * sc - lse_rows[r])
        D = do @ o_rows[r]
        U = np.abs(do * o_rows[r]).sum()
        ds = np.abs(p * (vv @ do - D))
        out[r] = (ds @ np.abs(kk) + U * (p @ np.abs(kk))) * sc
    return out


def oracle_forward(x: dict, B: int, topk: int, rows=None):
    """Oracle k', centroids, selection (+gap), O, LSE from CPU inputs."""
    cu = x["cu_seqlens"].numpy()
    q = x["q"].double().numpy()
    k = x["k"].double().numpy()
    v = x["v"].double().numpy()
    if "conv_w" in x:
        k = orc.key_conv(k, x["conv_w"].double().numpy(), cu)
    cents = orc.block_centroids(k, cu, B)
    sel, gap = orc.route(q, cents, cu, B, topk, rows=rows)
    o, lse = orc.attention(q, k, v, sel, cu, B, rows=rows)
    return dict(k=k, cents=cents, sel=sel, gap=gap, o=o, lse=lse, q=q, v=v, cu=cu)
