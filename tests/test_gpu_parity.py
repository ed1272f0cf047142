"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs.  Small cases compare every element; the full-size
workloads compare seeded samples of rows, and dK / dV of chosen key blocks,
that the oracle computes one by one.  Every case also checks which kernel
families ran (the tcgen05 router and attention kernels)."""
import numpy as np
import pytest
import torch

from block_sparse_long_key_b200 import moba, synth
from oracle import moba_oracle_c as orc
import parity_util as pu

FWD_PATH = moba.PATH_ROUTE_TCGEN05 | moba.PATH_FWD_TCGEN05

pytestmark = pytest.mark.gpu

# (seqlens, h_q, h_kv, d, B, topk, conv width)
SMALL = [
    ((4096,), 1, 1, 64, 128, 8, 0),                 # the 4K, one-head workload in full
    ((100, 257, 1000, 33), 4, 2, 128, 64, 4, 0),    # ragged varlen, GQA 2:1
    ((700, 1, 15, 300), 2, 2, 64, 16, 5, 0),        # B=16, sequences of 1 and < B tokens
    ((2048,), 2, 2, 64, 32, 32, 4),                 # small blocks + key conv width 4
    ((1500, 0, 600), 2, 1, 128, 128, 3, 0),         # empty sequence in the middle, B=128
    ((900,), 2, 2, 64, 32, 1, 0),                   # topk=1: block-diagonal causal
    ((600,), 1, 1, 128, 32, 64, 0),                 # topk=64 >= n: dense causal
    ((3000,), 8, 2, 64, 64, 16, 3),                 # GQA 4:1, conv width 3
    ((2500, 77), 4, 1, 64, 16, 6, 0),               # GQA 4:1, B=16: buckets of many 128-row tiles
]

# Key-conv widths beyond the SMALL cases (the register windows of both conv
# kernels are unrolled per width): ragged sequences, blocks shorter than and
# equal to twice the halo.
CONV_WIDTHS = [((300, 5, 700), 2, 2, 64, 32, 4, W) for W in (1, 2, 6, 7, 8)] + \
    [((260, 33), 2, 1, 128, 16, 3, 8)]


def _ids(c):
    return "L%s_h%dx%d_d%d_B%d_k%d_w%d" % ("-".join(map(str, c[0])), c[1], c[2], c[3], c[4], c[5], c[6])


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    moba.lib()
    return torch.device("cuda:0")


def _inputs(case, seed=11):
    seqlens, hq, hkv, d, B, topk, W = case
    w = synth.small(seqlens, hq, hkv, d, B, topk, conv_width=W, seed=seed)
    return w, synth.make_inputs(w)


def _gpu(x, dev):
    return {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def _forward(g, w, workspace=None):
    shape = moba.shape_of(g["q"], g["k"], g["cu_seqlens"], w.block_size, w.topk)
    ws = workspace if workspace is not None else moba.alloc_workspace(moba.fwd_workspace_size(shape), g["q"].device)
    res = moba.forward(g["q"], g["k"], g["v"], g["cu_seqlens"], w.block_size, w.topk, conv_w=g.get("conv_w"),
                       workspace=ws)
    return res, ws


@pytest.mark.parametrize("case", SMALL, ids=_ids)
def test_forward_matches_oracle(dev, case):
    w, x = _inputs(case)
    g = _gpu(x, dev)
    (out, lse, sel, _), ws = _forward(g, w)
    assert moba.check_status(ws) == 0
    assert moba.check_path(ws) & FWD_PATH == FWD_PATH, moba.check_path(ws)
    ref = pu.oracle_forward(x, w.block_size, w.topk)
    sel_g = sel.cpu().numpy()
    bad = pu.validate_selection(sel_g, ref, w.block_size, w.topk, what=_ids(case))
    o_g, lse_g = pu.to64(out), pu.to64(lse)
    o_ref, lse_ref = ref["o"].copy(), ref["lse"].copy()
    if bad:   # near ties: re-check those rows under the GPU's own selection
        o2, l2 = orc.attention(ref["q"], ref["k"], ref["v"], sel_g, ref["cu"], w.block_size, rows=bad)
        for t, h in bad:
            o_ref[t, h], lse_ref[t, h] = o2[t, h], l2[t, h]
    pu.check_o_lse(o_g, lse_g, o_ref, lse_ref, _ids(case))


@pytest.mark.parametrize("case", [c for c in SMALL if c[6] > 0] + [SMALL[1]] + CONV_WIDTHS, ids=_ids)
def test_conv_and_centroids_match_oracle(dev, case):
    w, x = _inputs(case)
    g = _gpu(x, dev)
    k_conv, cent = moba.key_conv_centroid(g["k"], g["cu_seqlens"], w.block_size, conv_w=g.get("conv_w"))
    torch.cuda.synchronize()
    cu = x["cu_seqlens"].numpy()
    k = x["k"].double().numpy()
    if w.conv_width:
        k_ref = orc.key_conv(k, x["conv_w"].double().numpy(), cu)
        k_g = pu.to64(k_conv)
        diff = k_g != k_ref
        # fp32 (GPU) vs fp64 (oracle) before the bf16 rounding: the two may
        # straddle a rounding midpoint, never by more than one bf16 step.
        ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(k_ref), 1e-30))) - 7)
        assert np.all(np.abs(k_g - k_ref)[diff] <= ulp[diff] * 1.0001)
        assert diff.mean() < 1e-3, diff.mean()
        k = k_ref
        kdiff = np.abs(k_g - k_ref)
    else:
        kdiff = np.zeros_like(k)
    cents = orc.block_centroids(k, cu, w.block_size)
    # A one-step difference in a key moves its block mean by that step / n;
    # those known key differences widen the bound of their block only.
    slack = orc.block_centroids(kdiff, cu, w.block_size)
    c_g = cent.cpu().double().numpy()
    off = 0
    for c, sl in zip(cents, slack):
        n = c.shape[1]
        err = np.abs(c_g[:, off:off + n] - c)
        assert np.all(err <= 1e-6 + 1e-5 * np.abs(c) + sl * 1.0001), err.max()
        off += n


@pytest.mark.parametrize("case", SMALL[:5], ids=_ids)
def test_block_index_matches_oracle(dev, case):
    w, x = _inputs(case)
    ref = pu.oracle_forward(x, w.block_size, w.topk)
    sel = torch.tensor(ref["sel"], dtype=torch.int32, device=dev)
    ptr, rows = moba.build_index(sel, x["cu_seqlens"].to(dev), w.h_kv, w.block_size)
    torch.cuda.synchronize()
    want = orc.block_index(ref["sel"], ref["cu"], w.block_size, w.h_kv)
    ptr, rows = ptr.cpu().numpy(), rows.cpu().numpy()
    nb = w.total_tokens // w.block_size + w.batch
    got = {}
    for kvh in range(w.h_kv):
        for gb in range(nb):
            b = kvh * nb + gb
            if ptr[b + 1] > ptr[b]:
                got[(kvh, gb)] = sorted(rows[ptr[b]:ptr[b + 1]].tolist())
    assert got == want
    assert ptr[-1] == sum(len(v) for v in want.values())


def _random_picks(seqlen, hq, B, seed):
    """Valid picks for every row of one sequence: two distinct past blocks
    (fewer when there are fewer), then the own block, then -1."""
    rng = np.random.default_rng(seed)
    own = np.repeat(np.arange(seqlen) // B, hq)
    sel = np.full((seqlen * hq, 3), -1, dtype=np.int32)
    a = rng.integers(0, np.maximum(own, 1))
    b = (a + 1 + rng.integers(0, np.maximum(own - 1, 1))) % np.maximum(own, 1)
    two = own >= 2
    sel[two, 0] = np.minimum(a, b)[two]
    sel[two, 1] = np.maximum(a, b)[two]
    sel[two, 2] = own[two]
    one = own == 1
    sel[one, 0], sel[one, 1] = 0, 1
    sel[own == 0, 0] = 0
    return sel.reshape(seqlen, hq, 3)


# Blocks per KV head: staged fill (<= 8192), shared-memory cursors (<= 16384),
# one global atomic per pick (> 16384).
@pytest.mark.parametrize("seqlen", [100_000, 200_000, 300_000])
def test_block_index_large_block_counts(dev, seqlen):
    B, hq, hkv = 16, 2, 1
    sel = _random_picks(seqlen, hq, B, seed=seqlen)
    cu = np.array([0, seqlen], dtype=np.int32)
    ptr, rows = moba.build_index(torch.from_numpy(sel).to(dev), torch.from_numpy(cu).to(dev), hkv, B)
    torch.cuda.synchronize()
    want = orc.block_index(sel, cu, B, hkv)
    ptr, rows = ptr.cpu().numpy(), rows.cpu().numpy()
    nb = seqlen // B + 1
    assert ptr[-1] == sum(len(v) for v in want.values())
    for (kvh, gb), lst in want.items():
        b = kvh * nb + gb
        assert sorted(rows[ptr[b]:ptr[b + 1]].tolist()) == lst, (kvh, gb)
    assert all(ptr[kvh * nb + gb + 1] == ptr[kvh * nb + gb] for kvh in range(hkv) for gb in range(nb)
               if (kvh, gb) not in want)


@pytest.mark.parametrize("case", SMALL, ids=_ids)
def test_backward_matches_oracle(dev, case):
    w, x = _inputs(case)
    g = _gpu(x, dev)
    (out, lse, sel, k_used), _ = _forward(g, w)
    shape = moba.shape_of(g["q"], g["k"], g["cu_seqlens"], w.block_size, w.topk)
    ws_b = moba.alloc_workspace(moba.bwd_workspace_size(shape), dev)
    dq, dk, dv = moba.backward(g["q"], k_used, g["v"], out, lse, g["dout"], sel, g["cu_seqlens"], w.block_size,
                               workspace=ws_b)
    assert moba.check_status(ws_b) == 0
    assert moba.check_path(ws_b) & moba.PATH_BWD_TCGEN05, moba.check_path(ws_b)
    ref = pu.oracle_forward(x, w.block_size, w.topk)
    bad = pu.validate_selection(sel.cpu().numpy(), ref, w.block_size, w.topk, what=_ids(case))
    do64 = x["dout"].double().numpy()
    dq_r, dk_r, dv_r = orc.attention_backward(ref["q"], ref["k"], ref["v"], do64, ref["sel"], ref["cu"], w.block_size)
    sq, sk, sv = pu.grad_error_scales(ref["q"], ref["k"], ref["v"], do64, ref["sel"], ref["cu"], w.block_size,
                                      ref["lse"], ref["o"])
    dq_g, dk_g, dv_g = pu.to64(dq), pu.to64(dk), pu.to64(dv)
    if bad:
        # Rows selected differently (near ties) change dQ of that row and
        # dK/dV of the blocks involved; leave those out.
        keep_q = np.ones(dq_r.shape[:2], bool)
        keep_kv = np.ones(dk_r.shape[:2], bool)
        g_ = w.h_q // w.h_kv
        sel_g = sel.cpu().numpy()
        for t, h in bad:
            keep_q[t, h] = False
            s = int(np.searchsorted(ref["cu"], t, side="right") - 1)
            for j in set(sel_g[t, h]) ^ set(ref["sel"][t, h]):
                if j >= 0:
                    a = ref["cu"][s] + j * w.block_size
                    keep_kv[a:a + w.block_size, h // g_] = False
        dq_r, dq_g, sq = dq_r[keep_q], dq_g[keep_q], sq[keep_q]
        dk_r, dk_g, dv_r, dv_g = dk_r[keep_kv], dk_g[keep_kv], dv_r[keep_kv], dv_g[keep_kv]
        sk, sv = sk[keep_kv], sv[keep_kv]
    pu.check_grad(dq_g, dq_r, sq, "dq " + _ids(case))
    pu.check_grad(dk_g, dk_r, sk, "dk " + _ids(case))
    pu.check_grad(dv_g, dv_r, sv, "dv " + _ids(case))


def test_status_flags_bad_seqlens_without_fault(dev):
    w, x = _inputs(((256, 256), 1, 1, 64, 32, 4, 0))
    g = _gpu(x, dev)
    cu = torch.tensor([0, 300, 200], dtype=torch.int32, device=dev)   # not monotone, wrong end
    ws = moba.alloc_workspace(moba.fwd_workspace_size(moba.shape_of(g["q"], g["k"], cu, 32, 4)), dev)
    moba.forward(g["q"], g["k"], g["v"], cu, 32, 4, workspace=ws)
    assert moba.check_status(ws) & moba.STATUS_BAD_SEQLENS
    ws2 = moba.alloc_workspace(moba.fwd_workspace_size(moba.shape_of(g["q"], g["k"], g["cu_seqlens"], 32, 4)), dev)
    moba.forward(g["q"], g["k"], g["v"], g["cu_seqlens"], 32, 4, workspace=ws2)
    assert moba.check_status(ws2) == 0


def test_status_flags_bad_sel_idx_in_backward(dev):
    w, x = _inputs(((512,), 2, 2, 64, 32, 4, 0))
    g = _gpu(x, dev)
    out, lse, sel, _ = moba.forward(g["q"], g["k"], g["v"], g["cu_seqlens"], 32, 4)
    sel = sel.clone()
    sel[3, 0, 0] = 9      # token 3 lives in block 0: block 9 is in its future
    sel[400, 1, 0] = -7
    shape = moba.shape_of(g["q"], g["k"], g["cu_seqlens"], 32, 4)
    ws = moba.alloc_workspace(moba.bwd_workspace_size(shape), dev)
    dq, dk, dv = moba.backward(g["q"], g["k"], g["v"], out, lse, g["dout"], sel, g["cu_seqlens"], 32, workspace=ws)
    assert moba.check_status(ws) & moba.STATUS_BAD_SEL_IDX
    assert torch.isfinite(dq.float()).all() and torch.isfinite(dk.float()).all()


def test_repeat_calls_are_stable(dev):
    w, x = _inputs(((1024,), 2, 2, 64, 32, 8, 0))
    g = _gpu(x, dev)
    a = moba.forward(g["q"], g["k"], g["v"], g["cu_seqlens"], 32, 8)
    b = moba.forward(g["q"], g["k"], g["v"], g["cu_seqlens"], 32, 8)
    assert torch.equal(a[2], b[2])
    assert (a[0].float() - b[0].float()).abs().max().item() <= 2 ** -7


# ------------------------------------------------------------- full sizes

def _sample_rows(w, per_head, seed):
    r = np.random.default_rng(seed)
    rows = []
    for h in range(w.h_q):
        ts = r.choice(w.total_tokens, size=min(per_head, w.total_tokens), replace=False)
        rows += [(int(t), h) for t in sorted(ts)]
    return rows


def _check_blocks(w, seed):
    """Key blocks whose dK / dV are compared at full size, per checked KV head:
    the first four of each sequence (the longest buckets, the longest CTAs),
    the last one inside the window the attention kernels issue early, one in
    the middle, the last two (the last may be partial) and two at random."""
    r = np.random.default_rng(seed)
    nbs = [(L + w.block_size - 1) // w.block_size for L in w.seqlens]
    nb_max = w.total_tokens // w.block_size + w.batch
    offs = np.concatenate([[0], np.cumsum(nbs)])
    kvs = sorted({0, w.h_kv - 1}) if w.h_q == w.h_kv else [w.h_kv - 1]
    blocks = []
    for kv in kvs:
        for s, n in enumerate(nbs):
            js = {0, 1, 3, max(nb_max // 8 - 1, 0), n // 2, n - 2, n - 1, int(r.integers(0, max(n, 1)))}
            blocks += [(kv, int(offs[s] + j)) for j in sorted(js) if 0 <= j < n]
    return blocks, offs


@pytest.mark.slow
@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_full_size_sampled_rows(dev, name):
    w = synth.WORKLOADS[name]
    B, topk = w.block_size, w.topk
    x = synth.make_inputs(w)
    g = _gpu(x, dev)
    (out, lse, sel, k_used), ws = _forward(g, w)
    assert moba.check_status(ws) == 0
    assert moba.check_path(ws) & FWD_PATH == FWD_PATH
    dq = None
    if w.backward:
        shape = moba.shape_of(g["q"], g["k"], g["cu_seqlens"], B, topk)
        ws_b = moba.alloc_workspace(moba.bwd_workspace_size(shape), dev)
        dq, dk, dv = moba.backward(g["q"], k_used, g["v"], out, lse, g["dout"], sel, g["cu_seqlens"], B,
                                   workspace=ws_b)
        assert moba.check_status(ws_b) == 0
        assert moba.check_path(ws_b) & moba.PATH_BWD_TCGEN05
    torch.cuda.synchronize()
    del g
    cu = x["cu_seqlens"].numpy()
    q = x["q"].double().numpy()
    k = x["k"].double().numpy()
    if "conv_w" in x:
        k = orc.key_conv(k, x["conv_w"].double().numpy(), cu)
    v = x["v"].double().numpy()
    cents = orc.block_centroids(k, cu, B)
    rows = _sample_rows(w, 512, 7)
    idx = tuple(np.array(rows).T)
    sel_all = sel.cpu().numpy()
    sel_g = sel_all[idx]
    sel_r, gap_r = orc.route_rows(q, cents, cu, B, topk, rows)
    bad = pu.validate_selection_rows(sel_g, sel_r, gap_r, rows, q, cents, cu, B, topk, what=name)
    sel_use = sel_r.copy()
    for i, (t, h) in enumerate(rows):           # near ties: re-checked under the GPU's selection
        if (t, h) in bad:
            sel_use[i] = sel_g[i]
    o_ref, lse_ref = orc.attention_rows(q, k, v, sel_use, cu, B, rows)
    pu.check_o_lse(pu.to64(out)[idx], pu.to64(lse)[idx], o_ref, lse_ref, name)
    for kv, hq, i, j in x["needles"]:          # planted blocks are always picked
        assert j in sel_all[i, hq], (kv, hq, i, j)
    if w.total_tokens * w.h_q <= (1 << 21):     # every row's selection where the oracle is quick enough
        every = [(t, h) for t in range(w.total_tokens) for h in range(w.h_q)]
        sel_full, gap_full = orc.route(q, cents, cu, B, topk)
        pu.validate_selection_rows(sel_all.reshape(-1, topk), sel_full.reshape(-1, topk), gap_full.reshape(-1),
                                   every, q, cents, cu, B, topk, what=name + " all rows")
    if dq is None:
        return
    do = x["dout"].double().numpy()
    dq_r = orc.backward_rows(q, k, v, do, sel_use, cu, B, rows)
    s_r = pu.row_dq_error_scale(q, k, v, do, sel_all, cu, B, rows, o_ref, lse_ref)
    pu.check_grad(pu.to64(dq)[idx], dq_r, s_r, "dq " + name)
    # dK / dV of chosen key blocks, under the GPU's own selection of every
    # query (its agreement with the oracle's is checked on the rows above).
    blocks, offs = _check_blocks(w, 11)
    dk_r, dv_r, sk, sv = orc.block_grads(q, k, v, do, sel_all, cu, B, blocks, magnitudes=True)
    dk_g, dv_g = pu.to64(dk), pu.to64(dv)
    gk, gv, rk, rv, ak, av = [], [], [], [], [], []
    for i, (kv, gb) in enumerate(blocks):
        s = int(np.searchsorted(offs, gb, side="right") - 1)
        t0 = int(cu[s]) + (gb - int(offs[s])) * B
        t1 = min(t0 + B, int(cu[s + 1]))
        gk.append(dk_g[t0:t1, kv]); gv.append(dv_g[t0:t1, kv])
        rk.append(dk_r[i, :t1 - t0]); rv.append(dv_r[i, :t1 - t0])
        ak.append(sk[i, :t1 - t0]); av.append(sv[i, :t1 - t0])
    pu.check_grad(np.concatenate(gk), np.concatenate(rk), np.concatenate(ak), "dk blocks " + name)
    pu.check_grad(np.concatenate(gv), np.concatenate(rv), np.concatenate(av), "dv blocks " + name)


@pytest.mark.parametrize("case", [SMALL[1], SMALL[3]], ids=_ids)
def test_backward_reusing_forward_index_matches_oracle(dev, case):
    w, x = _inputs(case)
    g = _gpu(x, dev)
    shape = moba.shape_of(g["q"], g["k"], g["cu_seqlens"], w.block_size, w.topk)
    wsf = moba.alloc_workspace(moba.fwd_workspace_size(shape), dev)
    out, lse, sel, k_used = moba.forward(g["q"], g["k"], g["v"], g["cu_seqlens"], w.block_size, w.topk,
                                         conv_w=g.get("conv_w"), workspace=wsf)
    dq, dk, dv = moba.backward(g["q"], k_used, g["v"], out, lse, g["dout"], sel, g["cu_seqlens"], w.block_size,
                               fwd_workspace=wsf)
    torch.cuda.synchronize()
    ref = pu.oracle_forward(x, w.block_size, w.topk)
    assert not pu.validate_selection(sel.cpu().numpy(), ref, w.block_size, w.topk, what="reuse")
    do64 = x["dout"].double().numpy()
    dq_r, dk_r, dv_r = orc.attention_backward(ref["q"], ref["k"], ref["v"], do64, ref["sel"], ref["cu"], w.block_size)
    sq, sk, sv = pu.grad_error_scales(ref["q"], ref["k"], ref["v"], do64, ref["sel"], ref["cu"], w.block_size,
                                      ref["lse"], ref["o"])
    pu.check_grad(pu.to64(dq), dq_r, sq, "dq reuse")
    pu.check_grad(pu.to64(dk), dk_r, sk, "dk reuse")
    pu.check_grad(pu.to64(dv), dv_r, sv, "dv reuse")


@pytest.mark.parametrize("case", [SMALL[3], SMALL[7], ((300, 5, 700), 2, 2, 128, 16, 4, 5)] + CONV_WIDTHS, ids=_ids)
def test_key_conv_backward_matches_oracle(dev, case):
    w, x = _inputs(case)
    g = _gpu(x, dev)
    dkc = synth.randn_bf16(x["k"].shape, seed=21)
    dk, dw = moba.key_conv_backward(g["k"], g["conv_w"], g["cu_seqlens"], w.block_size, dkc.to(dev))
    torch.cuda.synchronize()
    dk_r, dw_r = orc.key_conv_backward(x["k"].double().numpy(), x["conv_w"].double().numpy(), x["cu_seqlens"].numpy(),
                                       dkc.double().numpy())
    # dK: fp32 arithmetic, then one bf16 rounding (relative 2^-9 of the value).
    err = np.abs(pu.to64(dk) - dk_r)
    rms = np.sqrt((dk_r ** 2).mean())
    assert np.all(err <= 2.0 ** -8 * np.abs(dk_r) + 1e-5 * rms), (err / (np.abs(dk_r) + rms)).max()
    # dW: fp32 sums over every token of a head.
    np.testing.assert_allclose(pu.to64(dw), dw_r, rtol=1e-3, atol=1e-4 * np.abs(dw_r).max())


@pytest.mark.parametrize("d,B", [(64, 32), (128, 64)])
def test_rows_far_above_the_reference_take_the_exact_path(dev, d, B):
    # A key far above its block's mean along a later query (its logit ~190
    # natural-log units above the centroid-based reference M_i) would
    # overflow the fixed-reference sums; such rows are flagged and
    # recomputed exactly (online softmax) and must still match the oracle.
    w = synth.small((2048,), 2, 2, d, B, 8, seed=17)
    x = synth.make_inputs(w)
    i, h, j = 1500, 0, 5                      # query token, head, block of the planted key
    qh = x["q"][i, h].float()
    x["k"][j * B + 7, h] = (200.0 * qh / qh.norm()).to(torch.bfloat16)
    g = _gpu(x, dev)
    out, lse, sel, _ = moba.forward(g["q"], g["k"], g["v"], g["cu_seqlens"], B, w.topk)
    torch.cuda.synchronize()
    ref = pu.oracle_forward(x, B, w.topk)
    assert j in ref["sel"][i, h]               # the planted block is picked by that query
    sel_g = sel.cpu().numpy()
    bad = pu.validate_selection(sel_g, ref, B, w.topk, what="overflow")   # near ties only
    o_g, lse_g = pu.to64(out), pu.to64(lse)
    assert np.isfinite(o_g).all() and np.isfinite(lse_g).all()
    assert lse_g[i, h] > 100.0                 # the huge logit dominates
    o_ref, lse_ref = ref["o"].copy(), ref["lse"].copy()
    if bad:
        o2, l2 = orc.attention(ref["q"], ref["k"], ref["v"], sel_g, ref["cu"], B, rows=bad)
        for t, hh in bad:
            o_ref[t, hh], lse_ref[t, hh] = o2[t, hh], l2[t, hh]
    pu.check_o_lse(o_g, lse_g, o_ref, lse_ref, "overflow_d%d_B%d" % (d, B))


def test_forward_backward_replay_from_a_cuda_graph(dev):
    # The entry points allocate nothing, never synchronise and take the
    # stream, so a whole forward + backward (+ key-conv backward) step can be
    # captured once and replayed; the replay must give what eager calls give.
    case = ((2048,), 2, 2, 64, 32, 8, 4)
    w, x = _inputs(case)
    g = _gpu(x, dev)
    B, k = w.block_size, w.topk
    shape = moba.shape_of(g["q"], g["k"], g["cu_seqlens"], B, k)
    ws_f = moba.alloc_workspace(moba.fwd_workspace_size(shape), dev)
    ws_b = moba.alloc_workspace(moba.bwd_workspace_size(shape), dev)
    out, lse = torch.empty_like(g["q"]), torch.empty(g["q"].shape[:2], dtype=torch.float32, device=dev)
    sel = torch.empty(g["q"].shape[:2] + (k,), dtype=torch.int32, device=dev)
    kc = torch.empty_like(g["k"])
    dq, dk, dv = torch.empty_like(g["q"]), torch.empty_like(g["k"]), torch.empty_like(g["v"])
    dk_in, dw = torch.empty_like(g["k"]), torch.empty_like(g["conv_w"])

    def step():
        _, _, _, ku = moba.forward(g["q"], g["k"], g["v"], g["cu_seqlens"], B, k, conv_w=g["conv_w"],
                                   workspace=ws_f, out=out, lse=lse, sel_idx=sel, k_conv=kc)
        moba.backward(g["q"], ku, g["v"], out, lse, g["dout"], sel, g["cu_seqlens"], B, workspace=ws_b,
                      dq=dq, dk=dk, dv=dv, fwd_workspace=ws_f)
        moba.key_conv_backward(g["k"], g["conv_w"], g["cu_seqlens"], B, dk, workspace=ws_b, dk=dk_in, dw=dw)

    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        step()                                   # eager, on the capture stream
    torch.cuda.current_stream(dev).wait_stream(s)
    torch.cuda.synchronize()
    eager = [t.clone() for t in (out, lse, sel, dq, dv, dk_in, dw)]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        step()
    for t in (out, lse, dq, dv, dk_in, dw):
        t.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert moba.check_status(ws_f) == 0 and moba.check_status(ws_b) == 0
    got = (out, lse, sel, dq, dv, dk_in, dw)
    assert torch.equal(got[2], eager[2])
    for a, b in zip(got, eager):
        # fp32 reductions may add in another order: compare to bf16 resolution
        assert (a.float() - b.float()).abs().max().item() <= 2e-2 * max(1.0, b.float().abs().max().item())
    del graph


def test_bounded_wait_gives_up_and_reports_a_timeout(dev):
    # A device wait that can never complete (an mbarrier short of one
    # arrival, nothing in flight) must give up after its limit, record
    # MOBA_STATUS_TIMEOUT and return; the next call on a fresh workspace
    # runs clean.
    ws = moba.alloc_workspace(256, dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    moba.selftest_bounded_wait(1_000_000, ws)          # 1 ms
    e1.record()
    assert moba.check_status(ws) == moba.STATUS_TIMEOUT
    ms = e0.elapsed_time(e1)
    assert 1.0 <= ms < 500.0, ms
    w, x = _inputs(((512,), 2, 2, 64, 32, 4, 0))
    g = _gpu(x, dev)
    (out, lse, sel, _), ws2 = _forward(g, w)
    assert moba.check_status(ws2) == 0
    assert moba.check_path(ws2) & FWD_PATH == FWD_PATH
    assert torch.isfinite(out.float()).all()
