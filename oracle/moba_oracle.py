"""Plain fp64 CPU oracle of the MoBA hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code, constant or helper with the CUDA library under
``block_sparse_long_key_b200/csrc``.

Everything is computed in float64 from the bf16 input values, one sequence,
one head and (where it matters for clarity) one query at a time.  numpy's
matmul is the only library primitive used for dot products.

Source: "Optimizing Mixture of Block Attention" (Xiao, Guo, Mazaheri, Han),
as summarised on the lowest.today pages (Italian: "Ottimizzazione della
Mixture of Block Attention"; German: "Optimierung von Mixture of Block
Attention").  Section names below are the Italian page's.

Readings of points the pages leave open:

* Candidate blocks: a query scores only the strictly earlier blocks of its
  own sequence; its own block is always kept and counts toward ``topk``.
* Fewer candidates than ``topk - 1``: every earlier block is kept; unused
  slots of ``sel_idx`` hold -1.
* Exact score ties: the lower block index wins.  ``sel_idx`` rows are sorted
  ascending, the own block last among the valid entries.
* Router scores are unscaled ``q . c_j``; attention logits are scaled by
  ``1/sqrt(d)``; LSE is the natural-log log-sum-exp of the scaled logits.
* GQA: every query head routes on its own, against the centroids of its KV
  head ``h // (H_q / H_kv)``.
* Varlen: blocks, causality and the key-conv zero padding restart at every
  ``cu_seqlens`` boundary.  A partial last block's centroid is the mean over
  its real tokens (it is never scored: only a query's own block can be
  partial).
* Key conv: ``k'_t = k_t + SiLU(sum_l w_l * k_{t-l})`` with no bias, rounded
  to bf16 (round-to-nearest-even); routing and attention both use ``k'``.
* Backward: the selection is held fixed (top-k has no gradient); the
  gradients are those of the masked softmax attention.

Parity pins: every function here is pinned by a test in
``tests/test_oracle_pins.py`` to something other than itself (brute-force
enumeration, a library attention routine, closed forms, finite differences,
a hand-worked example).  Nothing here is "parity unpinned" except the
relation to the pages' own numbers, of which the pages print none.
"""
from __future__ import annotations

import math
from typing import List, Sequence, Tuple

import numpy as np

__all__ = [
    "round_bf16",
    "silu",
    "key_conv",
    "block_centroids",
    "past_block_scores",
    "route_row",
    "route",
    "visible_tokens",
    "attend_row",
    "attention",
    "attention_backward",
    "backward_rows",
    "block_selected_by",
    "block_index",
    "key_conv_backward",
    "router_snr",
    "router_p_fail",
]

# Largest finite bf16 value, (2 - 2^-7) * 2^127.
_BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


def round_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bf16 value, ties to even.

    bf16 keeps 8 significant bits (1 implicit + 7 stored) and the fp32
    exponent range.  For x = m * 2**e with 0.5 <= |m| < 1 the spacing of bf16
    values around x is 2**(e-8); below the smallest normal (2**-126) the
    spacing stays at 2**-133.  ``np.rint`` rounds half to even.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    e = np.maximum(e, -125)
    q = np.ldexp(np.rint(np.ldexp(x, 8 - e)), e - 8)
    return np.where(np.abs(q) > _BF16_MAX, np.copysign(np.inf, x), q)


def silu(x: np.ndarray) -> np.ndarray:
    """SiLU(x) = x * sigmoid(x) = x / (1 + exp(-x)), in float64."""
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-x))


def _seqs(cu_seqlens) -> List[Tuple[int, int]]:
    cu = [int(c) for c in np.asarray(cu_seqlens).ravel()]
    return [(cu[s], cu[s + 1]) for s in range(len(cu) - 1)]


def key_conv(k: np.ndarray, w: np.ndarray, cu_seqlens, round_output: bool = True) -> np.ndarray:
    """Depthwise causal short convolution on keys, then bf16 rounding.

    Follows §"Progettazione della Convoluzione delle Chiavi (Appendice B)",
    "Forma Formale": k'_t = k_t + SiLU(sum_{l=0}^{W-1} W_l (.) k_{t-l}), one
    filter per channel (groups = channels), left zero padding so that t-l
    before the sequence start contributes nothing.

    k: [T, H, d] float64 values of the bf16 keys.  w: [H, d, W] (tap l
    multiplies k_{t-l}).  Returns k' as float64 values of bf16 numbers
    (``round_output=False``: the unrounded float64 values).
    """
    k = np.asarray(k, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    width = w.shape[2]
    out = np.empty_like(k)
    for a, b in _seqs(cu_seqlens):
        ks = k[a:b]
        acc = np.zeros_like(ks)
        for l in range(width):
            shifted = np.zeros_like(ks)
            if l < ks.shape[0]:
                shifted[l:] = ks[: ks.shape[0] - l]
            acc += w[None, :, :, l] * shifted
        out[a:b] = ks + silu(acc)
    return round_bf16(out) if round_output else out


def block_centroids(k: np.ndarray, cu_seqlens, block_size: int) -> List[np.ndarray]:
    """Mean-pooled key-block centroids, one array [H_kv, n_s, d] per sequence.

    §"Architettura del Modello Statistico" 1: the router's block
    representative is the block mean (1/B) sum_{k in block j} k.  Blocks
    partition each sequence into ceil(L/B) contiguous runs of B tokens
    (§"Definizione del Compito": n = N/B); a partial last block averages its
    real tokens.
    """
    k = np.asarray(k, dtype=np.float64)
    out = []
    for a, b in _seqs(cu_seqlens):
        L = b - a
        n = (L + block_size - 1) // block_size
        c = np.empty((k.shape[1], n, k.shape[2]))
        for j in range(n):
            t0 = a + j * block_size
            t1 = min(a + (j + 1) * block_size, b)
            c[:, j, :] = k[t0:t1].mean(axis=0)
        out.append(c)
    return out


def past_block_scores(q_i: np.ndarray, cent_h: np.ndarray, pos: int, block_size: int) -> np.ndarray:
    """Router scores s_j = q_i . c_j of the earlier blocks j < pos // B of the
    query at local position ``pos`` (§"Architettura del Modello Statistico"
    1), in block order."""
    return cent_h[: pos // block_size] @ q_i


def route_row(q_i: np.ndarray, cent_h: np.ndarray, pos: int, block_size: int,
              topk: int) -> Tuple[List[int], float]:
    """Block selection of one query.

    §"Architettura del Modello Statistico" 1 (router score s_j = q^T k~_j)
    and §"Definizione del Compito" (keep the top-k blocks).  The query at
    local position ``pos`` lives in block b = pos // B; it scores blocks
    j < b, keeps the (topk-1) best (ties: lower j first) and always keeps b.

    Returns (selected blocks sorted ascending, relative gap between the last
    kept and the first rejected past-block score, or +inf when nothing was
    rejected).
    """
    b = pos // block_size
    if b == 0:
        return [0], math.inf
    scores = past_block_scores(q_i, cent_h, pos, block_size)
    order = sorted(range(b), key=lambda j: (-scores[j], j))
    keep = order[: topk - 1]
    gap = math.inf
    if b > topk - 1 and topk > 1:
        s_in = scores[order[topk - 2]]
        s_out = scores[order[topk - 1]]
        den = max(abs(s_in), abs(s_out))
        gap = abs(s_in - s_out) / den if den > 0 else 0.0
    elif b > topk - 1 and topk == 1:
        gap = math.inf  # nothing is scored competitively when only b is kept
    return sorted(keep) + [b], gap


def route(q: np.ndarray, cents: Sequence[np.ndarray], cu_seqlens, block_size: int,
          topk: int, rows=None) -> Tuple[np.ndarray, np.ndarray]:
    """sel_idx [T, H_q, topk] (int64, -1 padded) and gap [T, H_q].

    ``rows`` optionally restricts the work to a list of (token, q_head)
    pairs; other entries are left at -2 / nan.
    """
    q = np.asarray(q, dtype=np.float64)
    T, hq, _ = q.shape
    hkv = cents[0].shape[0]
    g = hq // hkv
    sel = np.full((T, hq, topk), -1, dtype=np.int64)
    gap = np.full((T, hq), np.nan)
    seqs = _seqs(cu_seqlens)
    if rows is None:
        todo = [(t, h) for t in range(T) for h in range(hq)]
    else:
        sel[:] = -2
        todo = [(int(t), int(h)) for t, h in rows]
    starts = np.array([a for a, _ in seqs])
    for t, h in todo:
        s = int(np.searchsorted(starts, t, side="right") - 1)
        pos = t - seqs[s][0]
        blocks, gp = route_row(q[t, h], cents[s][h // g], pos, block_size, topk)
        sel[t, h, :] = -1
        sel[t, h, : len(blocks)] = blocks
        gap[t, h] = gp
    return sel, gap


def visible_tokens(sel_row: Sequence[int], tok: int, seq_start: int, seq_end: int,
                   block_size: int) -> np.ndarray:
    """Tokens query ``tok`` attends to: every token of its selected blocks
    that is not in its future (causal mask; only the own block is cut)."""
    vis = []
    for j in sorted(int(x) for x in sel_row if x >= 0):
        t0 = seq_start + j * block_size
        t1 = min(seq_start + (j + 1) * block_size, seq_end)
        vis.extend(range(t0, min(t1, tok + 1)))
    return np.array(vis, dtype=np.int64)


def attend_row(q_i: np.ndarray, k_h: np.ndarray, v_h: np.ndarray,
               vis: np.ndarray) -> Tuple[np.ndarray, float]:
    """O_i = softmax(q_i K_V^T / sqrt(d)) V_V and its LSE over visible set V.

    §"Definizione del Compito": O = softmax(Q K^T / sqrt(d)) V, restricted
    to the selected tokens.  LSE = log sum exp of the scaled logits
    (max-subtracted for range, natural log).
    """
    d = q_i.shape[0]
    z = (k_h[vis] @ q_i) / math.sqrt(d)
    m = z.max()
    e = np.exp(z - m)
    l = e.sum()
    return (e / l) @ v_h[vis], float(m + math.log(l))


def attention(q, k, v, sel, cu_seqlens, block_size, rows=None):
    """O [T, H_q, d] and LSE [T, H_q] under the given selection (float64).

    ``rows`` optionally restricts to a list of (token, q_head); other
    outputs are nan.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    T, hq, d = q.shape
    g = hq // k.shape[1]
    o = np.full((T, hq, d), np.nan)
    lse = np.full((T, hq), np.nan)
    seqs = _seqs(cu_seqlens)
    starts = np.array([a for a, _ in seqs])
    todo = ((t, h) for t in range(T) for h in range(hq)) if rows is None else rows
    for t, h in todo:
        t, h = int(t), int(h)
        s = int(np.searchsorted(starts, t, side="right") - 1)
        a, b = seqs[s]
        vis = visible_tokens(sel[t, h], t, a, b, block_size)
        o[t, h], lse[t, h] = attend_row(q[t, h], k[:, h // g], v[:, h // g], vis)
    return o, lse


def _mask(sel, a, b, h, block_size):
    """Dense [L, L] visibility mask of sequence [a, b) for query head h."""
    L = b - a
    m = np.zeros((L, L), dtype=bool)
    for p in range(L):
        m[p, visible_tokens(sel[a + p, h], a + p, a, b, block_size) - a] = True
    return m


def attention_backward(q, k, v, dout, sel, cu_seqlens, block_size):
    """dQ [T,H_q,d], dK, dV [T,H_kv,d] in float64 with the selection fixed.

    §"Progettazione del Kernel FlashMoBA", "Backward Pass: Ricalcolo": the
    backward recomputes the attention probabilities; the gradient itself is
    the standard one of softmax attention.  With P the masked softmax,
    D_i = dO_i . O_i, dS = P (.) (dO V^T - D), dQ = dS K / sqrt(d),
    dK = dS^T Q / sqrt(d), dV = P^T dO; dK and dV are summed over the query
    heads sharing a KV head.  Dense per (sequence, head): small inputs only.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(dout, dtype=np.float64)
    T, hq, d = q.shape
    hkv = k.shape[1]
    g = hq // hkv
    scale = 1.0 / math.sqrt(d)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for a, b in _seqs(cu_seqlens):
        if b == a:
            continue  # an empty sequence has no queries and no keys
        for h in range(hq):
            kv = h // g
            msk = _mask(sel, a, b, h, block_size)
            z = (q[a:b, h] @ k[a:b, kv].T) * scale
            z = np.where(msk, z, -np.inf)
            z = z - z.max(axis=1, keepdims=True)
            p = np.exp(z)
            p /= p.sum(axis=1, keepdims=True)
            o = p @ v[a:b, kv]
            D = (do[a:b, h] * o).sum(axis=1)
            dp = do[a:b, h] @ v[a:b, kv].T
            ds = p * (dp - D[:, None])
            dq[a:b, h] = ds @ k[a:b, kv] * scale
            dk[a:b, kv] += ds.T @ q[a:b, h] * scale
            dv[a:b, kv] += p.T @ do[a:b, h]
    return dq, dk, dv


def backward_rows(q, k, v, dout, sel, cu_seqlens, block_size, rows):
    """Per-row backward terms for a list of (token, q_head) rows.

    Returns (dq_rows [R, d], contributions) where contributions is a list,
    per row, of (visible token indices, dK rows [V, d], dV rows [V, d]) this
    row adds to its KV head.  Same formulas as ``attention_backward``,
    evaluated one query at a time; used on sampled rows of large inputs.
    """
    q = np.asarray(q, dtype=np.float64)
    T, hq, d = q.shape
    g = hq // k.shape[1]
    scale = 1.0 / math.sqrt(d)
    seqs = _seqs(cu_seqlens)
    starts = np.array([a for a, _ in seqs])
    dq_rows = np.zeros((len(rows), d))
    contrib = []
    for r, (t, h) in enumerate(rows):
        t, h = int(t), int(h)
        s = int(np.searchsorted(starts, t, side="right") - 1)
        a, b = seqs[s]
        kv = h // g
        vis = visible_tokens(sel[t, h], t, a, b, block_size)
        kk = np.asarray(k[vis, kv], dtype=np.float64)
        vv = np.asarray(v[vis, kv], dtype=np.float64)
        dd = np.asarray(dout[t, h], dtype=np.float64)
        z = kk @ q[t, h] * scale
        p = np.exp(z - z.max())
        p /= p.sum()
        o = p @ vv
        D = dd @ o
        ds = p * (vv @ dd - D)
        dq_rows[r] = ds @ kk * scale
        contrib.append((vis, np.outer(ds, q[t, h]) * scale, np.outer(p, dd)))
    return dq_rows, contrib


def block_selected_by(q_h: np.ndarray, cent_h: np.ndarray, j: int, positions: np.ndarray,
                      block_size: int, topk: int) -> np.ndarray:
    """For queries at local ``positions`` (one head, one sequence), whether
    block ``j`` is among their selected blocks.

    Same rule as ``route_row`` written as a rank test: j is kept iff it is
    the query's own block, or it is an earlier block and fewer than topk-1
    earlier blocks beat it (higher score, or equal score and lower index).
    """
    q_h = np.asarray(q_h, dtype=np.float64)
    out = np.zeros(len(positions), dtype=bool)
    for r, p in enumerate(positions):
        b = int(p) // block_size
        if j == b:
            out[r] = True
            continue
        if j > b:
            continue
        sc = cent_h[:b] @ q_h[r]
        sj = sc[j]
        beat = np.count_nonzero(sc > sj) + np.count_nonzero(sc[:j] == sj)
        out[r] = beat < topk - 1
    return out


def block_index(sel, cu_seqlens, block_size: int, h_kv: int):
    """Key-block-major inversion of the picks (the varlen layout of the
    FlashMoBA Flash TopK stage 3, §"Progettazione del Kernel FlashMoBA",
    "Tre Kernel Fusi" 1).

    Returns {(kv_head, global block): sorted list of query row ids
    t * H_q + h}, global block = (blocks of earlier sequences) + j.  Every
    valid pick (own block included) appears once.
    """
    sel = np.asarray(sel)
    T, hq, topk = sel.shape
    g = hq // h_kv
    seqs = _seqs(cu_seqlens)
    out = {}
    off = 0
    for a, b in seqs:
        for t in range(a, b):
            for h in range(hq):
                for j in sel[t, h]:
                    if j >= 0:
                        out.setdefault((h // g, off + int(j)), []).append(t * hq + h)
        off += (b - a + block_size - 1) // block_size
    return {key: sorted(v) for key, v in out.items()}


def key_conv_backward(k: np.ndarray, w: np.ndarray, cu_seqlens, dk_conv: np.ndarray):
    """Gradients of the key convolution: (dK, dW) from dK' = dL/dk'.

    Differentiates the formula of ``key_conv`` (the final bf16 rounding is
    treated as the identity): with x_t = sum_l W_l (.) k_{t-l} and
    g_t = dK'_t (.) SiLU'(x_t), SiLU'(x) = s(x) (1 + x (1 - s(x))), s the
    logistic function:
      dK_t = dK'_t + sum_l W_l (.) g_{t+l}      (t + l inside the sequence)
      dW_l = sum_t g_t (.) k_{t-l}              (summed over all sequences)
    k, dk_conv: [T, H, d]; w: [H, d, W].  Returns dK [T, H, d], dW [H, d, W].
    """
    k = np.asarray(k, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    g_in = np.asarray(dk_conv, dtype=np.float64)
    width = w.shape[2]
    dk = g_in.copy()
    dw = np.zeros_like(w)
    for a, b in _seqs(cu_seqlens):
        ks = k[a:b]
        L = ks.shape[0]
        x = np.zeros_like(ks)
        shifted = []
        for l in range(width):
            sh = np.zeros_like(ks)
            if l < L:
                sh[l:] = ks[: L - l]
            shifted.append(sh)
            x += w[None, :, :, l] * sh
        sig = 1.0 / (1.0 + np.exp(-x))
        g = g_in[a:b] * sig * (1.0 + x * (1.0 - sig))
        for l in range(width):
            # dK_t gains W_l g_{t+l}; dW_l gains g_t k_{t-l}
            if l < L:
                dk[a:b][: L - l] += w[None, :, :, l] * g[l:]
            dw[:, :, l] += (g * shifted[l]).sum(axis=0)
    return dk, dw


def router_snr(delta_mu_eff: float, d: int, block_size: int) -> float:
    """Signal-to-noise ratio of the block router.

    §"Architettura del Modello Statistico" 2: for the score difference
    D = s_signal - s_noise of a signal block against one noise block,
    E[D] = delta_mu_eff / B and Var(D) = 2 sigma^2 / B with sigma^2 = 1/d
    for unit-scale vectors, so SNR = E[D] / sqrt(Var(D))
    = delta_mu_eff * sqrt(d / (2 B)).
    """
    mean = delta_mu_eff / block_size
    var = 2.0 / (d * block_size)
    return mean / math.sqrt(var)


def router_p_fail(snr: float) -> float:
    """Probability that the noise block outscores the signal block, Phi(-SNR)
    (§"Architettura del Modello Statistico" 2), with Phi the standard normal
    CDF written through the complementary error function."""
    return 0.5 * math.erfc(snr / math.sqrt(2.0))
