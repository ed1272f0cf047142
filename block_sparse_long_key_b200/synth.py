"""Seeded synthetic inputs for the MoBA hot path.

This module only draws numbers: it holds none of the method's arithmetic and
is shared by the tests (for both the CUDA path and the CPU oracle) and by
``bench.py``.  All tensors are created on the CPU with a seeded
``torch.Generator`` and rounded to bf16 (round-to-nearest-even) from fp32
N(0, 1) draws.  Each tensor gets its own generator, seeded from the workload
seed and a fixed tensor id, so that one tensor's values do not depend on the
sizes of the others.

Workloads (sizes follow the MoBA efficiency study summarised on the pages:
N up to 256K tokens, block sizes 32-128, head dim 64/128):

* ``n4k_h1_d64_b128_k8``            tiny, parity and latency
* ``n16k_h16_d128_b128_k8``
* ``n64k_h16_d64_b32_k32_kconv4``   small blocks, key conv width 4 with
  weights U(-0.5, 0.5), 256 planted needles per head (the headline shape)
* ``n256k_h8_d128_b64_k16``         long context
* ``varlen120k_gqa32x8_d128_b64_k16`` four packed sequences 8K/16K/32K/64K,
  32 query heads on 8 KV heads, forward + backward
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Tuple

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seqlens: Tuple[int, ...]
    h_q: int
    h_kv: int
    head_dim: int
    block_size: int
    topk: int
    conv_width: int = 0       # 0: no key conv
    needles_per_head: int = 0
    seed: int = 0
    backward: bool = True

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens))

    @property
    def batch(self) -> int:
        return len(self.seqlens)

    def fwd_flops(self) -> float:
        """Nominal forward FLOPs 4*T*H_q*k*B*d (own block counted in full)."""
        return 4.0 * self.total_tokens * self.h_q * self.topk * self.block_size * self.head_dim

    def bwd_flops(self) -> float:
        """Backward counted as 2.5x the forward (5 GEMMs against 2)."""
        return 2.5 * self.fwd_flops()


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("n4k_h1_d64_b128_k8", (4096,), 1, 1, 64, 128, 8, seed=0),
        Workload("n16k_h16_d128_b128_k8", (16384,), 16, 16, 128, 128, 8, seed=1),
        Workload("n64k_h16_d64_b32_k32_kconv4", (65536,), 16, 16, 64, 32, 32,
                 conv_width=4, needles_per_head=256, seed=2),
        Workload("n256k_h8_d128_b64_k16", (262144,), 8, 8, 128, 64, 16, seed=3),
        Workload("varlen120k_gqa32x8_d128_b64_k16", (8192, 16384, 32768, 65536), 32, 8,
                 128, 64, 16, seed=4),
    ]
}

HEADLINE = "n64k_h16_d64_b32_k32_kconv4"


def _gen(seed: int, tensor_id: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed * 1000003 + tensor_id)
    return g


def _randn_bf16(shape, seed, tensor_id) -> torch.Tensor:
    return torch.randn(shape, generator=_gen(seed, tensor_id), dtype=torch.float32).to(torch.bfloat16)


def randn_bf16(shape, seed: int, tensor_id: int = 7) -> torch.Tensor:
    """A seeded N(0, 1) bf16 tensor (e.g. an incoming gradient)."""
    return _randn_bf16(tuple(shape), seed, tensor_id)


def cu_seqlens_of(seqlens) -> torch.Tensor:
    cu = [0]
    for L in seqlens:
        cu.append(cu[-1] + int(L))
    return torch.tensor(cu, dtype=torch.int32)


def plant_needles(k32: torch.Tensor, q: torch.Tensor, seqlens, block_size: int,
                  per_head: int, seed: int, h_q: int) -> List[Tuple[int, int, int, int]]:
    """Add needles to fp32 keys in place; returns (kv_head, q_head, token, block).

    Per KV head, ``per_head`` pairs (i, j) are drawn: query token i uniform
    in [2B, L) of the first sequence and block j uniform in [0, i//B - 1].
    Every key of block j gets +2 * q_i / |q_i| (q of the group's first query
    head), i.e. the block is shifted by two unit standard deviations toward
    that later query's direction.
    """
    g = _gen(seed, 99)
    L = int(seqlens[0])
    h_kv = k32.shape[1]
    grp = h_q // h_kv
    out = []
    if L < 3 * block_size:
        return out
    for kv in range(h_kv):
        hq = kv * grp
        for _ in range(per_head):
            i = int(torch.randint(2 * block_size, L, (1,), generator=g))
            b = i // block_size
            j = int(torch.randint(0, b, (1,), generator=g))
            qi = q[i, hq].float()
            qhat = qi / qi.norm()
            t0, t1 = j * block_size, (j + 1) * block_size
            k32[t0:t1, kv] += 2.0 * qhat
            out.append((kv, hq, i, j))
    return out


def make_inputs(w: Workload, seed: Optional[int] = None, with_dout: bool = True) -> dict:
    """CPU tensors for workload ``w``.

    Keys: q, k, v [T, H, d] bf16; dout [T, H_q, d] bf16 (if requested);
    conv_w [H_kv, d, W] fp32 (if the workload has a key conv); cu_seqlens
    int32 [batch + 1]; needles (list of (kv_head, q_head, token, block)).
    """
    s = w.seed if seed is None else seed
    T, d = w.total_tokens, w.head_dim
    q = _randn_bf16((T, w.h_q, d), s, 1)
    k32 = torch.randn((T, w.h_kv, d), generator=_gen(s, 2), dtype=torch.float32)
    needles = []
    if w.needles_per_head:
        needles = plant_needles(k32, q, w.seqlens, w.block_size, w.needles_per_head, s, w.h_q)
    k = k32.to(torch.bfloat16)
    del k32
    v = _randn_bf16((T, w.h_kv, d), s, 3)
    out = dict(q=q, k=k, v=v, cu_seqlens=cu_seqlens_of(w.seqlens), needles=needles)
    if with_dout:
        out["dout"] = _randn_bf16((T, w.h_q, d), s, 4)
    if w.conv_width:
        gw = _gen(s, 5)
        out["conv_w"] = torch.rand((w.h_kv, d, w.conv_width), generator=gw,
                                   dtype=torch.float32) - 0.5
    return out


def small(seqlens, h_q, h_kv, d, B, topk, conv_width=0, seed=0, name="small") -> Workload:
    """An ad-hoc workload for parity tests."""
    return Workload(name, tuple(int(x) for x in seqlens), h_q, h_kv, d, B, topk,
                    conv_width=conv_width, seed=seed)


def snr_sequence(B: int, d: int, h: int, delta_mu_eff: float, m: int, seed: int, index: int,
                 full: bool = True) -> dict:
    """One sequence of the routing signal-to-noise harness (CPU, float64).

    2B + 1 tokens, ``h`` heads (KV heads = query heads).  Keys are
    g / sqrt(d) with g ~ N(0, I), so for a unit query q every key score
    q.k ~ N(0, 1/d).  The query rows that are measured are the last token
    (position 2B, the first token of block 2): a unit vector per head.  In
    one of the two earlier blocks (``signal`` per head, uniform) ``m`` tokens
    get + (delta_mu_eff / m) q_hat added, so that block's key sum is shifted
    by delta_mu_eff along q.  Other query rows and V are plain N(0, 1).

    Returns dict(q, k, v) as float64 arrays [2B+1, h, d] and ``signal`` [h]
    (with ``full=False`` only k, the measured query rows ``q_last`` [h, d]
    and ``signal``: enough to route).
    """
    g = _gen(seed, 1000 + index)
    L = 2 * B + 1
    k = torch.randn((L, h, d), generator=g, dtype=torch.float64) / math.sqrt(d)
    qlast = torch.randn((h, d), generator=g, dtype=torch.float64)
    qlast /= qlast.norm(dim=-1, keepdim=True)
    signal = torch.randint(0, 2, (h,), generator=g)
    for hh in range(h):
        j = int(signal[hh])
        toks = torch.randperm(B, generator=g)[:m] + j * B
        k[toks, hh] += (delta_mu_eff / m) * qlast[hh]
    if not full:
        return dict(k=k.numpy(), q_last=qlast.numpy(), signal=signal.numpy())
    q = torch.randn((L, h, d), generator=g, dtype=torch.float64)
    q[L - 1] = qlast
    v = torch.randn((L, h, d), generator=g, dtype=torch.float64)
    return dict(q=q.numpy(), k=k.numpy(), v=v.numpy(), signal=signal.numpy())


def snr_batch(B: int, d: int, h: int, n_seq: int, delta_mu_eff: float, m: int = 1, seed: int = 0) -> dict:
    """``n_seq`` harness sequences packed varlen, as bf16 CPU tensors.

    Keys: q, k, v [T, h, d] bf16, cu_seqlens, rows (token of each measured
    query, per sequence), signal [n_seq, h].
    """
    qs, ks, vs, sig = [], [], [], []
    for i in range(n_seq):
        one = snr_sequence(B, d, h, delta_mu_eff, m, seed, i)
        qs.append(torch.from_numpy(one["q"]))
        ks.append(torch.from_numpy(one["k"]))
        vs.append(torch.from_numpy(one["v"]))
        sig.append(torch.from_numpy(one["signal"]))
    seqlens = [2 * B + 1] * n_seq
    cu = cu_seqlens_of(seqlens)
    return dict(q=torch.cat(qs).float().to(torch.bfloat16), k=torch.cat(ks).float().to(torch.bfloat16),
                v=torch.cat(vs).float().to(torch.bfloat16), cu_seqlens=cu,
                rows=(cu[1:] - 1).tolist(), signal=torch.stack(sig).numpy())
