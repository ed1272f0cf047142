"""Routing signal-to-noise harness.

"Optimizing Mixture of Block Attention", §"Architettura del Modello
Statistico" 2: the router's score difference between a signal block and a
noise block has mean delta_mu_eff / B and variance 2 / (d B) (unit-scale
vectors), so a noise block outscores the signal block with probability
p_fail = Phi(-SNR), SNR = delta_mu_eff * sqrt(d / (2B)).  The pages fix
d = 64 and vary B in {128, 256, 512}.

The harness builds sequences of 2B + 1 tokens whose measured query (the
first token of block 2) keeps its own block and the better of blocks 0 and 1
(topk = 2); one of the two carries the planted shift.  With Gaussian keys the
score difference is exactly normal, so the empirical failure rate must match
Phi(-SNR) within its binomial error.  This pins the router (oracle and GPU)
to the pages' closed form, and the closed form to a Monte-Carlo estimate.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_long_key_b200 import synth
from oracle import moba_oracle as O

D = 64


def _delta_for(snr, B):
    return snr / math.sqrt(D / (2 * B))


def _oracle_trials(B, snr, n_seq, h, m=1, seed=11):
    """Per trial: (failed, D = s_signal - s_noise) through the oracle route."""
    delta = _delta_for(snr, B)
    fails, diffs = [], []
    for i in range(n_seq):
        one = synth.snr_sequence(B, D, h, delta, m, seed, i, full=False)
        k = O.round_bf16(one["k"])
        cents = O.block_centroids(k, [0, 2 * B + 1], B)[0]        # [h, 3, d]
        for hh in range(h):
            qi = O.round_bf16(one["q_last"][hh])
            blocks, _ = O.route_row(qi, cents[hh], 2 * B, B, 2)
            sig = int(one["signal"][hh])
            fails.append(blocks[0] != sig)
            s = cents[hh][:2] @ qi
            diffs.append(s[sig] - s[1 - sig])
    return np.array(fails), np.array(diffs)


def test_p_fail_is_the_normal_tail():
    from scipy.stats import norm
    for x in (0.0, 0.25, 0.5, 1.0, 1.5, 2.0, 3.0):
        assert abs(O.router_p_fail(x) - norm.cdf(-x)) < 1e-14
    assert O.router_p_fail(0.0) == 0.5


@pytest.mark.parametrize("B", [128, 256, 512])
def test_score_difference_moments_match_the_model(B):
    # E[D] = delta / B and Var(D) = 2 / (d B): the two halves of the SNR.
    snr = 1.0
    _, diffs = _oracle_trials(B, snr, n_seq=150, h=4)
    n = len(diffs)
    mean, var = diffs.mean(), diffs.var(ddof=1)
    exp_mean, exp_var = _delta_for(snr, B) / B, 2.0 / (D * B)
    assert abs(mean - exp_mean) < 4.5 * math.sqrt(exp_var / n)
    assert abs(var / exp_var - 1.0) < 4.5 * math.sqrt(2.0 / (n - 1))
    assert abs(O.router_snr(_delta_for(snr, B), D, B) - exp_mean / math.sqrt(exp_var)) < 1e-12


@pytest.mark.parametrize("B", [128, 256, 512])
@pytest.mark.parametrize("snr", [0.5, 1.0, 1.5])
def test_oracle_router_failure_rate_is_phi_of_minus_snr(B, snr):
    fails, _ = _oracle_trials(B, snr, n_seq=150, h=4)
    p = O.router_p_fail(O.router_snr(_delta_for(snr, B), D, B))
    n = len(fails)
    assert abs(fails.mean() - p) < 4.5 * math.sqrt(p * (1 - p) / n) + 0.005


def test_aggregation_keeps_the_failure_rate_at_fixed_delta_eff():
    # Key finding 2: what matters is delta_mu_eff; spreading it over m = 8
    # tokens of the block gives the same failure rate.
    B, snr = 128, 1.0
    f1, _ = _oracle_trials(B, snr, n_seq=150, h=4, m=1, seed=3)
    f8, _ = _oracle_trials(B, snr, n_seq=150, h=4, m=8, seed=3)
    p = O.router_p_fail(snr)
    tol = 4.5 * math.sqrt(p * (1 - p) / len(f1)) + 0.005
    assert abs(f1.mean() - p) < tol and abs(f8.mean() - p) < tol


@pytest.mark.gpu
@pytest.mark.parametrize("B", [32, 64, 128])
@pytest.mark.parametrize("snr", [0.5, 1.0, 2.0])
def test_gpu_router_failure_rate_is_phi_of_minus_snr(B, snr):
    from block_sparse_long_key_b200 import moba
    n_seq, h = 512, 8
    x = synth.snr_batch(B, D, h, n_seq, _delta_for(snr, B), seed=5)
    dev = torch.device("cuda:0")
    q, k, v, cu = (x[n].to(dev) for n in ("q", "k", "v", "cu_seqlens"))
    _, _, sel, _ = moba.forward(q, k, v, cu, B, 2)
    torch.cuda.synchronize()
    rows = torch.tensor(x["rows"], dtype=torch.long)
    chosen = sel.cpu()[rows, :, 0].numpy()                         # [n_seq, h]
    fails = chosen != x["signal"]
    p = O.router_p_fail(O.router_snr(_delta_for(snr, B), D, B))
    n = fails.size
    assert abs(fails.mean() - p) < 4.5 * math.sqrt(p * (1 - p) / n) + 0.005
    # and the GPU picks exactly what the oracle picks on these rows
    kk = O.round_bf16(x["k"].float().numpy().astype(np.float64))
    cents = O.block_centroids(kk, x["cu_seqlens"].tolist(), B)
    ref, gap = O.route(x["q"].float().numpy().astype(np.float64), cents, x["cu_seqlens"].tolist(), B, 2,
                       rows=[(t, hh) for t in x["rows"] for hh in range(h)])
    ref_chosen = ref[rows.numpy(), :, 0]
    near_tie = gap[rows.numpy()] <= 1e-3
    assert np.all((ref_chosen == chosen) | near_tie)
