"""Pins of the fp64 oracle to things other than itself.

Each test checks one oracle function against brute force, a library routine
used on a special case, a closed form, finite differences, or a hand-worked
example, chosen so that a dropped term, a wrong sign or index, or a
transposed operand in the oracle fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import moba_oracle as orc_np
from oracle import moba_oracle_c as orc_cpp

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# Every pin below runs against both oracles: the numpy one and the fp64
# C++ / OpenMP one (same functions and results).  A few helpers exist only in
# the numpy oracle; their tests use ``orc_np``.
@pytest.fixture(params=["numpy", "cpp"])
def orc(request):
    return orc_np if request.param == "numpy" else orc_cpp


def _rng(seed):
    return np.random.default_rng(seed)


def _bf16(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).double().numpy()


# ---------------------------------------------------------------- bf16 rounding

def test_round_bf16_matches_torch_on_fp32_values(orc):
    r = _rng(0)
    x = np.concatenate([
        r.standard_normal(20000).astype(np.float32),
        (r.standard_normal(2000) * 1e-39).astype(np.float32),   # fp32 subnormals
        (r.standard_normal(2000) * 1e30).astype(np.float32),
        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 0.0, -0.0], np.float32),  # exact ties
    ])
    want = torch.tensor(x).to(torch.bfloat16).double().numpy()
    got = orc.round_bf16(x.astype(np.float64))
    np.testing.assert_array_equal(got, want)


def test_round_bf16_ties_to_even_closed_form(orc):
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: even mantissa is 1.0.
    assert orc.round_bf16(1 + 2 ** -8) == 1.0
    # 1 + 3*2^-8 lies halfway between 1+2^-7 and 1+2^-6: even is 1+2^-6.
    assert orc.round_bf16(1 + 3 * 2 ** -8) == 1 + 2 ** -6
    assert orc.round_bf16(1e39) == np.inf


# ---------------------------------------------------------------- key conv

def test_silu_against_torch(orc):
    x = np.linspace(-30, 30, 1001)
    np.testing.assert_allclose(orc.silu(x), F.silu(torch.tensor(x)).numpy(), rtol=1e-15, atol=1e-300)
    assert orc.silu(np.array([0.0]))[0] == 0.0


def test_key_conv_hand_worked_example(orc):
    g = json.load(open(os.path.join(GOLDEN, "kconv_3token.json")))
    got = orc.key_conv(np.array(g["k"]), np.array(g["w"]), g["cu_seqlens"])
    np.testing.assert_array_equal(got, np.array(g["k_conv_bf16"]))


def test_key_conv_zero_weights_is_identity(orc):
    r = _rng(1)
    k = _bf16(r.standard_normal((37, 3, 8)))
    for W in (1, 3, 4):
        got = orc.key_conv(k, np.zeros((3, 8, W)), [0, 20, 37])
        np.testing.assert_array_equal(got, k)


def test_key_conv_matches_library_conv1d_and_restarts_per_sequence(orc):
    r = _rng(2)
    T, H, d, W = 45, 2, 4, 4
    cu = [0, 13, 14, 45]
    k = _bf16(r.standard_normal((T, H, d)))
    w = r.uniform(-0.5, 0.5, (H, d, W))
    got = orc.key_conv(k, w, cu)
    want = np.empty_like(k)
    for a, b in zip(cu[:-1], cu[1:]):
        x = torch.tensor(k[a:b]).reshape(b - a, H * d).T[None]          # [1, C, L]
        # conv1d is a cross-correlation: weight index m meets x[t + m - (W-1)],
        # so tap l (which multiplies x[t-l]) sits at m = W-1-l.
        wt = torch.tensor(w[:, :, ::-1].copy()).reshape(H * d, 1, W)
        y = F.conv1d(F.pad(x, (W - 1, 0)), wt, groups=H * d)[0].T.reshape(b - a, H, d)
        want[a:b] = k[a:b] + F.silu(y).numpy()
    np.testing.assert_array_equal(got, orc.round_bf16(want))


# ---------------------------------------------------------------- centroids

def test_centroids_closed_form_linear_keys(orc):
    # k_t = (t - a) * u within each sequence: the mean of block j over tokens
    # [t0, t1) is ((t0 + t1 - 1) / 2) * u.
    u = np.array([1.0, -2.0, 0.5])
    cu = [0, 10, 17]
    k = np.zeros((17, 1, 3))
    for a, b in zip(cu[:-1], cu[1:]):
        for t in range(a, b):
            k[t, 0] = (t - a) * u
    cents = orc.block_centroids(k, cu, 4)
    assert [c.shape for c in cents] == [(1, 3, 3), (1, 2, 3)]
    for c, L in zip(cents, (10, 7)):
        for j in range(c.shape[1]):
            t0, t1 = 4 * j, min(4 * j + 4, L)
            np.testing.assert_allclose(c[0, j], (t0 + t1 - 1) / 2 * u, rtol=0, atol=1e-15)


# ---------------------------------------------------------------- routing

def _brute_force_selection(scores, b, topk):
    """Best (topk-1)-subset of past blocks by score sum; ties -> the
    lexicographically smallest sorted tuple (lower indices first)."""
    m = min(topk - 1, b)
    best, best_key = None, None
    for sub in itertools.combinations(range(b), m):
        key = (-sum(scores[j] for j in sub), sub)
        if best_key is None or key < best_key:
            best, best_key = sub, key
    return list(best) + [b]


@pytest.mark.parametrize("B,topk,integer", [(2, 3, False), (3, 4, False), (4, 4, True), (1, 5, True), (2, 1, False)])
def test_route_matches_brute_force_subsets(orc, B, topk, integer):
    r = _rng(3 + B + topk)
    L, d = 10 * B, 5
    for trial in range(3):
        if integer:   # integer values (B a power of two) force exact score ties
            q = r.integers(-2, 3, (L, 1, d)).astype(np.float64)
            k = r.integers(-2, 3, (L, 1, d)).astype(np.float64)
        else:
            q = r.standard_normal((L, 1, d))
            k = r.standard_normal((L, 1, d))
        cents = orc.block_centroids(k, [0, L], B)
        sel, _ = orc.route(q, cents, [0, L], B, topk)
        for p in range(L):
            b = p // B
            scores = [float(np.dot(q[p, 0], k[j * B:(j + 1) * B, 0].mean(axis=0))) for j in range(b)]
            want = _brute_force_selection(scores, b, topk)
            got = [int(x) for x in sel[p, 0] if x >= 0]
            assert got == want, (p, got, want)
            assert list(sel[p, 0, len(want):]) == [-1] * (topk - len(want))


def test_route_gqa_uses_group_kv_head(orc):
    r = _rng(4)
    L, B, d, topk = 48, 4, 6, 3
    q = r.standard_normal((L, 4, d))
    k = r.standard_normal((L, 2, d))
    cents = orc.block_centroids(k, [0, L], B)
    sel, _ = orc.route(q, cents, [0, L], B, topk)
    for h in range(4):
        s1, _ = orc.route(q[:, h:h + 1], [c[h // 2:h // 2 + 1] for c in cents], [0, L], B, topk)
        np.testing.assert_array_equal(sel[:, h], s1[:, 0])


# The near-tie gap: relative difference between the last kept and the first
# rejected earlier-block score, |s_in - s_out| / max(|s_in|, |s_out|) (0 when
# both are 0, +inf when no earlier block is rejected).  With B = 1 every block
# is one token, its centroid is that key, and keys that are the unit vectors
# e_j make the query's scores exactly s_j = q_j; the values below are worked
# out by hand from the chosen scores.
GAP_CASES = [
    # (scores of blocks 0..b-1, topk, kept earlier blocks, gap)
    ([5, 1, 4, 3, 2], 3, [0, 2], 1 / 4),       # kept 5, 4; first rejected 3
    ([5, 4, 3, 1], 3, [0, 1], 1 / 4),          # (a shifted index would give 2/3)
    ([4, 1, 3], 3, [0, 2], 2 / 3),             # exactly one block rejected
    ([1, -3], 2, [0], 4 / 3),                  # denominator: the larger magnitude
    ([-1, -2, -3], 2, [0], 1 / 2),             # all negative
    ([3, 3, 1], 2, [0], 0.0),                  # exact tie at the boundary: lower index kept
    ([0, 0, 0], 2, [0], 0.0),                  # both zero
    ([2, 7], 3, [0, 1], math.inf),             # b <= topk - 1: nothing rejected
    ([2, 7, 1], 1, [], math.inf),              # topk = 1: only the own block
    ([1e-3, 2e-3, 1.5e-3, 1.4e-3], 3, [1, 2], 0.1 / 1.5),
]


@pytest.mark.parametrize("scores,topk,kept,gap", GAP_CASES)
def test_near_tie_gap_hand_worked(orc, scores, topk, kept, gap):
    b = len(scores)
    d = b + 1
    k = np.zeros((b + 1, 1, d))
    for j in range(b):
        k[j, 0, j] = 1.0
    q = np.zeros((b + 1, 1, d))
    q[b, 0, :b] = scores
    sel, g = orc.route(q, orc.block_centroids(k, [0, b + 1], 1), [0, b + 1], 1, topk)
    valid = [int(x) for x in sel[b, 0] if x >= 0]
    assert valid == kept + [b]
    assert list(sel[b, 0, len(valid):]) == [-1] * (topk - len(valid))
    if math.isinf(gap):
        assert math.isinf(g[b, 0])
    else:
        assert g[b, 0] == pytest.approx(gap, rel=1e-12, abs=1e-15)


def test_near_tie_gap_of_route_row_directly():
    cent = np.eye(6)
    for scores, topk, kept, gap in GAP_CASES:
        q = np.zeros(6)
        q[:len(scores)] = scores
        blocks, g = orc_np.route_row(q, cent, len(scores), 1, topk)
        assert blocks == kept + [len(scores)]
        assert (math.isinf(g) and math.isinf(gap)) or g == pytest.approx(gap, rel=1e-12, abs=1e-15)


# ---------------------------------------------------------------- attention

def _sdpa(q, k, v, mask):
    """Library attention in fp64: q [L,d], k/v [L,d], mask [L,L] bool."""
    o = F.scaled_dot_product_attention(torch.tensor(q)[None, None], torch.tensor(k)[None, None],
                                       torch.tensor(v)[None, None], attn_mask=torch.tensor(mask))
    return o[0, 0].numpy()


def _lse_dense(q, k, mask):
    z = torch.tensor(q) @ torch.tensor(k).T / math.sqrt(q.shape[1])
    z = z.masked_fill(~torch.tensor(mask), -math.inf)
    return torch.logsumexp(z, dim=1).numpy()


def test_topk_all_blocks_equals_dense_causal_attention(orc):
    r = _rng(5)
    cu = [0, 37, 100]
    T, hq, hkv, d, B = 100, 4, 2, 8, 8
    q, k, v = (r.standard_normal((T, h, d)) for h in (hq, hkv, hkv))
    cents = orc.block_centroids(k, cu, B)
    sel, _ = orc.route(q, cents, cu, B, topk=64)       # >= every n_s
    o, lse = orc.attention(q, k, v, sel, cu, B)
    for a, b in zip(cu[:-1], cu[1:]):
        causal = np.tril(np.ones((b - a, b - a), dtype=bool))
        for h in range(hq):
            np.testing.assert_allclose(o[a:b, h], _sdpa(q[a:b, h], k[a:b, h // 2], v[a:b, h // 2], causal),
                                       rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(lse[a:b, h], _lse_dense(q[a:b, h], k[a:b, h // 2], causal),
                                       rtol=1e-12, atol=1e-12)


def test_topk1_is_block_diagonal_causal_attention(orc):
    r = _rng(6)
    T, d, B = 40, 4, 8
    q, k, v = (r.standard_normal((T, 1, d)) for _ in range(3))
    sel, _ = orc.route(q, orc.block_centroids(k, [0, T], B), [0, T], B, topk=1)
    o, _ = orc.attention(q, k, v, sel, [0, T], B)
    blockdiag = np.zeros((T, T), dtype=bool)
    for i in range(T):
        for t in range(T):
            blockdiag[i, t] = (i // B == t // B) and t <= i
    np.testing.assert_allclose(o[:, 0], _sdpa(q[:, 0], k[:, 0], v[:, 0], blockdiag), rtol=1e-12, atol=1e-12)


def test_block1_topk1_attends_to_itself_only(orc):
    r = _rng(7)
    T, d = 9, 4
    q, k, v = (r.standard_normal((T, 1, d)) for _ in range(3))
    sel, _ = orc.route(q, orc.block_centroids(k, [0, T], 1), [0, T], 1, topk=1)
    o, lse = orc.attention(q, k, v, sel, [0, T], 1)
    np.testing.assert_allclose(o[:, 0], v[:, 0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse[:, 0], (q[:, 0] * k[:, 0]).sum(1) / 2.0, rtol=1e-15)


def test_zero_keys_give_uniform_attention(orc):
    r = _rng(8)
    T, d, B, topk = 50, 4, 4, 3
    q = r.standard_normal((T, 1, d))
    k = np.zeros((T, 1, d))
    v = r.standard_normal((T, 1, d))
    sel, _ = orc.route(q, orc.block_centroids(k, [0, T], B), [0, T], B, topk)
    o, lse = orc.attention(q, k, v, sel, [0, T], B)
    for i in range(T):
        b = i // B
        # all scores tie at 0: the lowest-index past blocks win
        blocks = list(range(min(topk - 1, b))) + [b]
        vis = [t for j in blocks for t in range(j * B, min(j * B + B, i + 1))]
        assert [int(x) for x in sel[i, 0] if x >= 0] == blocks
        np.testing.assert_allclose(lse[i, 0], math.log(len(vis)), rtol=1e-14)
        np.testing.assert_allclose(o[i, 0], v[vis, 0].mean(axis=0), rtol=1e-12, atol=1e-14)


def test_permuting_a_past_block_leaves_output_unchanged(orc):
    r = _rng(9)
    T, d, B, topk = 64, 8, 8, 3
    q, k, v = (r.standard_normal((T, 1, d)) for _ in range(3))
    cents = orc.block_centroids(k, [0, T], B)
    sel, _ = orc.route(q, cents, [0, T], B, topk)
    o, lse = orc.attention(q, k, v, sel, [0, T], B)
    perm = np.arange(T)
    perm[8:16] = perm[8:16][::-1].copy()       # a full block, past for tokens >= 16
    k2, v2 = k[perm], v[perm]
    sel2, _ = orc.route(q, orc.block_centroids(k2, [0, T], B), [0, T], B, topk)
    np.testing.assert_array_equal(sel2[16:], sel[16:])
    o2, lse2 = orc.attention(q, k2, v2, sel2, [0, T], B)
    np.testing.assert_allclose(o2[16:], o[16:], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse2[16:], lse[16:], rtol=1e-13)


def test_split_and_merge_reproduces_single_pass(orc):
    # LSE is what lets partial results over a partition of the visible set be
    # combined: O = sum_s exp(lse_s - LSE) O_s with LSE = log sum_s exp(lse_s).
    # Here the parts are disjoint groups of one query's selected blocks.
    r = _rng(10)
    T, d, B = 40, 16, 4
    q = r.standard_normal((T, 1, d)) * 3
    k = r.standard_normal((T, 1, d))
    v = r.standard_normal((T, 1, d))
    t = 38                                         # block 9, its own block cut at t

    def run(blocks):
        sel = np.full((T, 1, 4), -1, dtype=np.int64)
        sel[t, 0, :len(blocks)] = blocks
        o, lse = orc.attention(q, k, v, sel, [0, T], B, rows=[(t, 0)])
        return o[t, 0], lse[t, 0]

    o, lse = run([0, 2, 5, 9])
    res = [run(p) for p in ([0], [2, 5], [9])]
    L = np.logaddexp.reduce([x[1] for x in res])
    om = sum(np.exp(x[1] - L) * x[0] for x in res)
    assert abs(L - lse) < 1e-12
    np.testing.assert_allclose(om, o, rtol=1e-12, atol=1e-12)


def test_split_and_merge_of_single_rows():
    r = _rng(10)
    d = 16
    q = r.standard_normal(d) * 3
    k = r.standard_normal((40, d))
    v = r.standard_normal((40, d))
    vis = np.arange(40)
    o, lse = orc_np.attend_row(q, k, v, vis)
    parts = [vis[:7], vis[7:8], vis[8:31], vis[31:]]
    res = [orc_np.attend_row(q, k, v, p) for p in parts]
    L = np.logaddexp.reduce([x[1] for x in res])
    om = sum(np.exp(x[1] - L) * x[0] for x in res)
    assert abs(L - lse) < 1e-12
    np.testing.assert_allclose(om, o, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- backward

def _loss(orc, q, k, v, dout, sel, cu, B):
    o, _ = orc.attention(q, k, v, sel, cu, B)
    return float((o * dout).sum())


def test_backward_matches_central_finite_differences(orc):
    r = _rng(11)
    cu = [0, 11, 24]
    T, hq, hkv, d, B, topk = 24, 2, 1, 3, 3, 2
    q, k, v = r.standard_normal((T, hq, d)), r.standard_normal((T, hkv, d)), r.standard_normal((T, hkv, d))
    dout = r.standard_normal((T, hq, d))
    sel, _ = orc.route(q, orc.block_centroids(k, cu, B), cu, B, topk)
    dq, dk, dv = orc.attention_backward(q, k, v, dout, sel, cu, B)
    eps = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args = dict(q=q, k=k, v=v)
            args[name] = xp
            lp = _loss(orc, args["q"], args["k"], args["v"], dout, sel, cu, B)
            args[name] = xm
            lm = _loss(orc, args["q"], args["k"], args["v"], dout, sel, cu, B)
            num[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8, err_msg=name)


@pytest.mark.parametrize("cu", [[0, 30], [0, 0, 30, 30]])
def test_backward_topk_all_equals_library_autograd(orc, cu):
    r = _rng(12)
    T, hq, hkv, d, B = 30, 2, 1, 8, 4
    q, k, v = r.standard_normal((T, hq, d)), r.standard_normal((T, hkv, d)), r.standard_normal((T, hkv, d))
    dout = r.standard_normal((T, hq, d))
    sel, _ = orc.route(q, orc.block_centroids(k, cu, B), cu, B, topk=100)
    dq, dk, dv = orc.attention_backward(q, k, v, dout, sel, cu, B)
    tq = torch.tensor(q).permute(1, 0, 2)[None].requires_grad_()
    tk = torch.tensor(k).permute(1, 0, 2)[None].requires_grad_()
    tv = torch.tensor(v).permute(1, 0, 2)[None].requires_grad_()
    o = F.scaled_dot_product_attention(tq, tk.repeat_interleave(2, 1), tv.repeat_interleave(2, 1),
                                       is_causal=True)
    o.backward(torch.tensor(dout).permute(1, 0, 2)[None])
    np.testing.assert_allclose(dq, tq.grad[0].permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad[0].permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad[0].permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)


def test_backward_rows_sum_to_dense_backward():
    r = _rng(13)
    cu = [0, 20, 52]
    T, hq, hkv, d, B, topk = 52, 4, 2, 4, 4, 3
    q, k, v = r.standard_normal((T, hq, d)), r.standard_normal((T, hkv, d)), r.standard_normal((T, hkv, d))
    dout = r.standard_normal((T, hq, d))
    sel, _ = orc_np.route(q, orc_np.block_centroids(k, cu, B), cu, B, topk)
    dq, dk, dv = orc_np.attention_backward(q, k, v, dout, sel, cu, B)
    rows = [(t, h) for t in range(T) for h in range(hq)]
    dqr, contrib = orc_np.backward_rows(q, k, v, dout, sel, cu, B, rows)
    dk2, dv2 = np.zeros_like(dk), np.zeros_like(dv)
    for (t, h), (vis, a, b) in zip(rows, contrib):
        dk2[vis, h // 2] += a
        dv2[vis, h // 2] += b
    np.testing.assert_allclose(dqr.reshape(T, hq, d), dq, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dk2, dk, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dv2, dv, rtol=1e-12, atol=1e-12)


def test_cpp_row_and_block_backward_equal_dense_backward():
    # The per-row dQ and the per-block dK / dV of the C++ oracle (used on
    # full-size inputs) against its dense backward, which the finite
    # difference and library autograd pins above fix.
    r = _rng(13)
    cu = [0, 20, 20, 61]
    T, hq, hkv, d, B, topk = 61, 4, 2, 4, 4, 3
    q, k, v = r.standard_normal((T, hq, d)), r.standard_normal((T, hkv, d)), r.standard_normal((T, hkv, d))
    dout = r.standard_normal((T, hq, d))
    sel, _ = orc_cpp.route(q, orc_cpp.block_centroids(k, cu, B), cu, B, topk)
    dq, dk, dv = orc_cpp.attention_backward(q, k, v, dout, sel, cu, B)
    rows = [(t, h) for t in range(T) for h in range(hq)]
    idx = tuple(np.array(rows).T)
    dqr = orc_cpp.backward_rows(q, k, v, dout, sel[idx], cu, B, rows)
    np.testing.assert_allclose(dqr.reshape(T, hq, d), dq, rtol=1e-12, atol=1e-12)
    nb = [5, 0, 11]                                  # blocks per sequence (the last one partial)
    blocks = [(kv, gb) for kv in range(hkv) for gb in range(sum(nb))]
    dkb, dvb = orc_cpp.block_grads(q, k, v, dout, sel, cu, B, blocks)
    starts = [0, 20, 20]
    offs = [0, 5, 5]
    for i, (kv, gb) in enumerate(blocks):
        s = 0 if gb < 5 else 2
        t0 = starts[s] + (gb - offs[s]) * B
        t1 = min(t0 + B, cu[s + 1])
        np.testing.assert_allclose(dkb[i, :t1 - t0], dk[t0:t1, kv], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dvb[i, :t1 - t0], dv[t0:t1, kv], rtol=1e-12, atol=1e-12)
        assert not dkb[i, t1 - t0:].any() and not dvb[i, t1 - t0:].any()


def test_block_selected_by_agrees_with_route():
    r = _rng(14)
    L, d, B, topk = 80, 4, 4, 4
    q = r.integers(-2, 3, (L, 1, d)).astype(np.float64)    # ties included
    k = r.integers(-2, 3, (L, 1, d)).astype(np.float64)
    cents = orc_np.block_centroids(k, [0, L], B)
    sel, _ = orc_np.route(q, cents, [0, L], B, topk)
    for j in range(L // B):
        flags = orc_np.block_selected_by(q[:, 0], cents[0][0], j, np.arange(L), B, topk)
        want = np.array([j in sel[p, 0] for p in range(L)])
        np.testing.assert_array_equal(flags, want)


def test_planted_needles_are_selected(orc):
    from block_sparse_long_key_b200 import synth
    w = synth.Workload("needles", (2048,), 2, 2, 64, 32, 8, conv_width=4, needles_per_head=16, seed=5)
    x = synth.make_inputs(w, with_dout=False)
    k = orc.key_conv(x["k"].double().numpy(), x["conv_w"].double().numpy(), x["cu_seqlens"].numpy())
    cents = orc.block_centroids(k, x["cu_seqlens"].numpy(), w.block_size)
    rows = [(i, hq) for (_, hq, i, _) in x["needles"]]
    sel, _ = orc.route(x["q"].double().numpy(), cents, x["cu_seqlens"].numpy(), w.block_size, w.topk, rows=rows)
    for (_, hq, i, j) in x["needles"]:
        assert j in sel[i, hq], (i, hq, j)


def test_block_index_is_a_partition_of_the_picks(orc):
    r = _rng(15)
    cu = [0, 30, 31, 90]
    T, hq, hkv, d, B, topk = 90, 4, 2, 4, 8, 3
    q = r.standard_normal((T, hq, d))
    k = r.standard_normal((T, hkv, d))
    sel, _ = orc.route(q, orc.block_centroids(k, cu, B), cu, B, topk)
    idx = orc.block_index(sel, cu, B, hkv)
    picks = [(t * hq + h, j) for t in range(T) for h in range(hq) for j in sel[t, h] if j >= 0]
    assert sum(len(v) for v in idx.values()) == len(picks)
    offs = [0, 4, 5]                                          # ceil(30/8), ceil(1/8)
    for t in range(T):
        s = 0 if t < 30 else (1 if t < 31 else 2)
        for h in range(hq):
            for j in sel[t, h]:
                if j >= 0:
                    assert t * hq + h in idx[(h // 2, offs[s] + int(j))]


# ---------------------------------------------------------------- key conv backward

def test_key_conv_backward_matches_finite_differences(orc):
    r = _rng(16)
    cu = [0, 7, 12]
    T, H, d, W = 12, 2, 3, 3
    k = r.standard_normal((T, H, d))
    w = r.uniform(-0.5, 0.5, (H, d, W))
    g = r.standard_normal((T, H, d))
    dk, dw = orc.key_conv_backward(k, w, cu, g)
    loss = lambda kk, ww: float((orc.key_conv(kk, ww, cu, round_output=False) * g).sum())
    eps = 1e-6
    for name, x, grad in (("k", k, dk), ("w", w, dw)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[i] += eps
            xm[i] -= eps
            lp = loss(xp, w) if name == "k" else loss(k, xp)
            lm = loss(xm, w) if name == "k" else loss(k, xm)
            num[i] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8, err_msg=name)


def test_key_conv_backward_matches_library_autograd(orc):
    r = _rng(17)
    cu = [0, 20, 20, 45]
    T, H, d, W = 45, 2, 4, 4
    k = r.standard_normal((T, H, d))
    w = r.uniform(-0.5, 0.5, (H, d, W))
    g = r.standard_normal((T, H, d))
    dk, dw = orc.key_conv_backward(k, w, cu, g)
    tk = torch.tensor(k, requires_grad=True)
    tw = torch.tensor(w, requires_grad=True)
    outs = []
    for a, b in zip(cu[:-1], cu[1:]):
        if a == b:
            continue   # an empty sequence contributes nothing
        x = tk[a:b].reshape(b - a, H * d).T[None]
        wt = tw.flip(-1).reshape(H * d, 1, W)
        y = F.conv1d(F.pad(x, (W - 1, 0)), wt, groups=H * d)[0].T.reshape(b - a, H, d)
        outs.append(tk[a:b] + F.silu(y))
    torch.cat(outs).backward(torch.tensor(g))
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dw, tw.grad.numpy(), rtol=1e-12, atol=1e-12)
