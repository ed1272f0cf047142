"""The bench's exact-useful count against a brute-force count of the keys a
query reads (CPU): every valid pick of a past block is B keys, the own block
the keys up to the query; selections from the oracle router on ragged
sequences (partial last blocks, empty and one-token sequences, fewer past
blocks than top-k)."""
import os
import sys

import numpy as np
import pytest
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from block_sparse_long_key_b200 import synth
from oracle import moba_oracle as orc


@pytest.mark.parametrize("seqlens,hq,hkv,B,topk", [
    ((300, 0, 1, 77), 2, 1, 16, 4),
    ((129,), 1, 1, 32, 8),
    ((500, 33), 4, 2, 64, 3),
])
def test_visible_keys_match_a_brute_force_count(seqlens, hq, hkv, B, topk):
    import bench
    w = synth.small(seqlens, hq, hkv, 64, B, topk, seed=5)
    x = synth.make_inputs(w)
    cu = x["cu_seqlens"].numpy()
    k = x["k"].double().numpy()
    sel, _ = orc.route(x["q"].double().numpy(), orc.block_centroids(k, cu, B), cu, B, topk)
    pos = torch.cat([torch.arange(b - a) for a, b in zip(cu[:-1].tolist(), cu[1:].tolist())]).double()
    pairs = int((sel >= 0).sum())
    brute = 0
    for t in range(w.total_tokens):
        own = int(pos[t]) // B
        for h in range(hq):
            for j in sel[t, h]:
                if j < 0:
                    continue
                brute += B if j < own else int(pos[t]) % B + 1
    assert bench.visible_keys(pos, B, hq, pairs) == brute
    # and never more than the nominal count
    assert brute <= w.total_tokens * hq * topk * B
