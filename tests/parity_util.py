"""Shared helpers of the GPU-vs-oracle parity tests.

Tolerances (bf16 inputs, fp32 accumulation on the GPU, fp64 oracle):

* sel_idx: bit-exact, except for queries whose last kept and first rejected
  past-block scores differ by <= 1e-3 relative; those are re-checked under
  the GPU's own selection.
* O: max-abs <= 2e-2 and mean-abs <= 1e-3; LSE: max-abs <= 1e-3.
* dQ/dK/dV, element by element: |g_gpu - g_ref| <= 2e-2 * (rms(g_ref) +
  max|g_ref row|), the row being the d values of one (token, head), and
  mean-abs <= 4e-3 * rms(g_ref).  Derivation: each gradient element is a sum
  of products with one factor rounded to bf16 before the MMA (P for dV, dS
  for dQ and dK; relative error 2^-9 each, fp32 sums), so its error is
  bounded by 2^-9 * sum|terms|, which is of the size of the largest element
  of the same row, not of the element itself (the terms cancel: the dS of a
  query sum to zero); the result is then rounded to bf16 (2^-9), and D_i is
  formed from the bf16 O as in the FlashAttention-style backward.  A numpy
  emulation with exactly those roundings reproduces the GPU values and gives
  max |error| / (rms + row max) = 4.8e-3 and mean 1.6e-3 rms on the 4K
  workload: the bound keeps a 4x margin over that.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import moba_oracle as orc

GAP = 1e-3
O_MAX, O_MEAN, LSE_MAX = 2e-2, 1e-3, 1e-3
G_REL, G_MEAN = 2e-2, 4e-3


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


def check_grad(g_gpu, g_ref, what=""):
    rms = float(np.sqrt(np.mean(g_ref ** 2))) + 1e-30
    err = np.abs(g_gpu - g_ref)
    assert np.isfinite(g_gpu).all(), what
    rowmax = np.abs(g_ref).max(axis=-1, keepdims=True)
    ratio = err / (G_REL * (rms + rowmax))
    assert ratio.max() <= 1.0, (what, "max err/(2e-2*(rms+rowmax))", ratio.max(), "max-abs/rms", err.max() / rms)
    assert err.mean() <= G_MEAN * rms, (what, "mean-abs/rms", err.mean() / rms)
    return ratio.max(), err.mean() / rms


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
