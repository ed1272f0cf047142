#!/usr/bin/env python
"""Benchmark of the MoBA hot path on B200.

One step = the whole hot path over one batch of synthetic input: key conv +
centroids, routing + top-k, block index, sparse attention forward and
normalisation, then the backward (preprocess, block index, attention, dQ).
Default workload: N = 64K tokens, 16 heads, d = 64, B = 32, top-k = 32, key
conv width 4, 256 planted needles per head (the small-block long-context
shape).  The JSON line reports effective TFLOP/s on the nominal FLOP count
3.5 * 4*N*H*k*B*d (forward 4*N*H*k*B*d, backward 2.5x that) and its
fraction of the measured B200 bf16 tensor peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torchrun) the KV-head groups of one seeded problem
are split over the ranks (a KV head and its query heads stay together, so no
data-path collective is needed; strong scaling); ``--shard replica`` runs an
independent problem of the same shape per rank instead (weak scaling).  The
step time is the max over ranks and ``value`` the whole job's throughput.
``--impl reference`` times the fp64 C++ CPU oracle (every host core) on a
bounded sample instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from block_sparse_long_key_b200 import synth  # noqa: E402

METRIC = "MoBA fwd/bwd effective TFLOP/s & ms at N=64K,B=32; % of B200 bf16 tensor peak"
UNIT = "TFLOP/s"
L2_BYTES = 126 * 2 ** 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic per launch of each kernel, read from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum), keyed by the SHA-256 of the
# kernel source file it was taken with: a changed source voids the figure.
# Headline workload, one timed-step launch each (profiles/dram_traffic_n64k_h16_d64_b32_k32_kconv4.md).
NCU_TRAFFIC = {
    "fwd_route": {"bytes": 278.49e6 + 366.52e6, "sha": "98c2c86de5d6b6fb"},
    "fwd_attn": {"bytes": 1.1745e9 + 721.19e6, "sha": "7a566854044986cd"},
    "bwd_attn": {"bytes": 1.9201e9 + 1.0060e9, "sha": "3ffdaa36749d5531"},
    "conv_bwd": {"bytes": 268.57e6 + 127.72e6, "sha": "cab0cb4e397e800e"},
    "fwd_centroid": {"bytes": 134.25e6 + 102.05e6, "sha": "792b201ba3dbf790"},
    "fwd_index": {"bytes": (134.23e6 + 2.72e6) + 8.40e6 + (172.91e6 + 107.21e6), "sha": "4a2d500ca215863b"},
}


# ----------------------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def src_sha(fname):
    with open(os.path.join(ROOT, "block_sparse_long_key_b200", "csrc", fname), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        maxclk = max(r[1] for r in rows)
        loaded = [r for r in rows if r[2] > 200.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": maxclk, "reasons": reasons,
                "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": max(r[2] for r in rows)}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(value: float, device, world: int) -> float:
    """Max of a float over ranks (identity for one rank)."""
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(total_flops_per_step: float, ms_per_step: float) -> float:
    """Whole-job TFLOP/s: every rank's work over the slowest rank's time."""
    return total_flops_per_step / (ms_per_step * 1e-3) / 1e12


def rank_seed(w: synth.Workload, rank: int) -> int:
    return w.seed + 7919 * rank


def visible_keys(pos: "torch.Tensor", block_size: int, h_q: int, pairs: int) -> float:
    """Keys the attention actually reads, summed over every (query, head):
    `pairs` valid picks (own block included, one per query and head), each
    past block contributing B keys and the own block the (p mod B) + 1 keys
    up to the query at in-sequence position p.  The nominal count assumes k
    full blocks per query and head."""
    own = float(((pos % block_size) + 1).sum().item()) * h_q
    return (pairs - pos.numel() * h_q) * block_size + own


def head_shard(h_kv: int, world: int, rank: int):
    """KV heads [kv0, kv1) of rank `rank` when one problem's KV-head groups
    are split over `world` ranks: contiguous ranges, the first h_kv % world
    ranks taking one more.  A KV head and the query heads that read it stay
    on one rank, so dK / dV never cross ranks and the path needs no
    collective."""
    base, extra = divmod(h_kv, world)
    kv0 = rank * base + min(rank, extra)
    return kv0, kv0 + base + (1 if rank < extra else 0)


def shard_inputs(x: dict, w: synth.Workload, kv0: int, kv1: int):
    """The inputs of KV heads [kv0, kv1) (and their query heads) of one
    problem, as contiguous tensors, and the workload they form."""
    import dataclasses
    g = w.h_q // w.h_kv
    out = {"q": x["q"][:, kv0 * g:kv1 * g].contiguous(), "k": x["k"][:, kv0:kv1].contiguous(),
           "v": x["v"][:, kv0:kv1].contiguous(), "cu_seqlens": x["cu_seqlens"],
           "needles": [(kv - kv0, hq - kv0 * g, i, j) for kv, hq, i, j in x["needles"] if kv0 <= kv < kv1]}
    if "dout" in x:
        out["dout"] = x["dout"][:, kv0 * g:kv1 * g].contiguous()
    if "conv_w" in x:
        out["conv_w"] = x["conv_w"][kv0:kv1].contiguous()
    return out, dataclasses.replace(w, h_kv=kv1 - kv0, h_q=(kv1 - kv0) * g)


def stage_roofline(name, w, pairs, scored, peaks):
    """(bound, algorithmic amount per launch, unit) of one stage."""
    T, hq, hkv, d, B = w.total_tokens, w.h_q, w.h_kv, w.head_dim, w.block_size
    if name == "fwd_attn":
        return "tensor", 4.0 * B * d * pairs, "flop"
    if name == "bwd_attn":
        return "tensor", 10.0 * B * d * pairs, "flop"
    if name == "fwd_route":
        return "tensor", 2.0 * 2.0 * d * scored, "flop"   # hi + lo products
    if name == "fwd_centroid":
        return "hbm", T * hkv * d * 2.0 * (3 if w.conv_width else 1), "byte"
    if name == "fwd_finalize":
        return "hbm", T * hq * (d * 6.0 + 12), "byte"
    if name == "bwd_pre":
        return "hbm", T * hq * (d * 8.0 + 12), "byte"
    if name == "bwd_dq":
        return "hbm", T * hq * d * 6.0, "byte"
    if name in ("fwd_index", "bwd_index"):
        return "hbm", T * hq * w.topk * 4.0 * 2 + pairs * 4.0 * 3, "byte"
    if name == "conv_bwd":
        return "hbm", T * hkv * d * 2.0 * 3, "byte"
    return "hbm", 0.0, "byte"


KERNEL_SRC = {"fwd_attn": "fwd_tc.cu", "bwd_attn": "bwd_tc.cu", "fwd_route": "route.cu", "fwd_centroid": "conv_centroid.cu",
              "fwd_finalize": "fwd.cu", "bwd_pre": "bwd.cu", "bwd_dq": "bwd.cu", "fwd_index": "index.cu",
              "bwd_index": "index.cu", "conv_bwd": "conv_bwd.cu"}

# Kernels of ours launched per step: forward 10 (plan, conv/centroid, route,
# index count, prefix, scan, fill, attention, finalize, fallback), backward 4
# (plan, preprocess, attention, dQ; the forward's block index is reused),
# key-conv backward 3 (plan, per-block pass, dW reduction) when the conv is on.
LAUNCHES_PER_STEP = 14
LAUNCHES_CONV_BWD = 3


# ----------------------------------------------------------------------------- oracle (CPU) timing

def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_sample(w: synth.Workload, seed: int, rows_per_step: int, steps: int, warmup: int):
    """Times the fp64 C++ oracle (OpenMP over rows, every host core) on
    seeded samples of (query, head) rows.  Returns per-step TFLOP/s values,
    a description and the thread count.  Routing against all past centroids,
    attention and the per-row backward run inside the timed region; the key
    conv and centroids (O(N d), computed once for the whole input) are
    prepared outside it."""
    from oracle import moba_oracle_c as orc

    x = synth.make_inputs(w, seed=seed)
    cu = x["cu_seqlens"].numpy()
    q = x["q"].double().numpy()
    k = x["k"].double().numpy()
    if "conv_w" in x:
        k = orc.key_conv(k, x["conv_w"].double().numpy(), cu)
    v = x["v"].double().numpy()
    dout = x["dout"].double().numpy()
    cents = orc.block_centroids(k, cu, w.block_size)
    r = np.random.default_rng(seed)
    n = min(rows_per_step, w.total_tokens * w.h_q)
    flops_row = 3.5 * 4.0 * w.topk * w.block_size * w.head_dim
    vals = []
    for step in range(warmup + steps):
        flat = r.choice(w.total_tokens * w.h_q, size=n, replace=False)
        rows = [(int(f) // w.h_q, int(f) % w.h_q) for f in np.sort(flat)]
        t0 = time.perf_counter()
        sel, _ = orc.route_rows(q, cents, cu, w.block_size, w.topk, rows)
        orc.attention_rows(q, k, v, sel, cu, w.block_size, rows)
        orc.backward_rows(q, k, v, dout, sel, cu, w.block_size, rows)
        dt = time.perf_counter() - t0
        if step >= warmup:
            vals.append(n * flops_row / dt / 1e12)
    threads = orc.num_threads()
    desc = ("%d random (query, head) rows per step (of %d) through the fp64 C++ oracle, OpenMP on %d threads "
            "(host: %d cores, %s): routing against all past centroids, attention and the per-row backward; "
            "FLOPs counted as 3.5*4*k*B*d per row (nominal, as on the GPU); key conv and centroids prepared "
            "outside the timed region" % (n, w.total_tokens * w.h_q, threads, os.cpu_count() or 0, cpu_model()))
    return vals, desc, threads


# ----------------------------------------------------------------------------- our arm

def dense_context(g, hq, hkv, moba_ms):
    """Dense causal attention forward + backward through the library SDPA
    (flash backend only; None if it is unavailable), timed like the step."""
    from torch.nn.attention import SDPBackend, sdpa_kernel
    T, _, d = g["q"].shape
    q = g["q"].view(1, T, hq, d).transpose(1, 2).detach().requires_grad_(True)
    k = g["k"].view(1, T, hkv, d).transpose(1, 2).repeat_interleave(hq // hkv, dim=1).detach().requires_grad_(True)
    v = g["v"].view(1, T, hkv, d).transpose(1, 2).repeat_interleave(hq // hkv, dim=1).detach().requires_grad_(True)
    do = g["dout"].view(1, T, hq, d).transpose(1, 2)
    try:
        with sdpa_kernel([SDPBackend.FLASH_ATTENTION]):
            def one():
                o = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
                o.backward(do)
            for _ in range(2):
                one()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            n = 3
            e0.record()
            for _ in range(n):
                one()
            e1.record()
            torch.cuda.synchronize()
        t = e0.elapsed_time(e1) / n
    except RuntimeError as exc:
        return {"impl": "torch SDPA flash backend", "unavailable": str(exc).splitlines()[0][:160]}
    return {"impl": "torch SDPA flash backend (library), dense causal, same Q/K/V shapes, fwd+bwd",
            "ms_per_step": round(t, 3), "dense_over_moba": round(t / moba_ms, 3)}


def run_ours(args):
    from block_sparse_long_key_b200 import moba

    world, rank, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    w = synth.WORKLOADS[args.workload]
    peaks, peak_src = load_peaks()
    moba.lib()

    # N > 1: KV-head groups of one problem split over the ranks (strong
    # scaling, the default), or one independent problem per rank.
    sharded = world > 1 and args.shard == "heads" and w.h_kv >= world
    total_flops = (w.fwd_flops() + w.bwd_flops()) * (1 if sharded else world)
    if sharded:
        seed = w.seed
        kv0, kv1 = head_shard(w.h_kv, world, rank)
        x, w = shard_inputs(synth.make_inputs(w, seed=seed), w, kv0, kv1)
        parallelism = "KV-head groups of one problem sharded over %d GPUs, no collective" % world
    else:
        seed = rank_seed(w, rank)
        x = synth.make_inputs(w, seed=seed)
        parallelism = "independent problem per GPU" if world > 1 else "single GPU"
    g = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    T, hq, hkv, d, B, topk = w.total_tokens, w.h_q, w.h_kv, w.head_dim, w.block_size, w.topk
    shape = moba.shape_of(g["q"], g["k"], g["cu_seqlens"], B, topk)
    ws_f = moba.alloc_workspace(moba.fwd_workspace_size(shape), dev)
    ws_b = moba.alloc_workspace(moba.bwd_workspace_size(shape), dev)
    out = torch.empty_like(g["q"])
    lse = torch.empty((T, hq), dtype=torch.float32, device=dev)
    sel = torch.empty((T, hq, topk), dtype=torch.int32, device=dev)
    kc = torch.empty_like(g["k"]) if w.conv_width else None
    dq, dk, dv = torch.empty_like(g["q"]), torch.empty_like(g["k"]), torch.empty_like(g["v"])
    conv_w = g.get("conv_w")
    dk_in = torch.empty_like(g["k"]) if conv_w is not None else None
    dw = torch.empty_like(conv_w) if conv_w is not None else None

    def step(qd, kd, vd, dod, cud, cw):
        _, _, _, k_used = moba.forward(qd, kd, vd, cud, B, topk, conv_w=cw, workspace=ws_f, out=out, lse=lse,
                                       sel_idx=sel, k_conv=kc)
        moba.backward(qd, k_used, vd, out, lse, dod, sel, cud, B, workspace=ws_b, dq=dq, dk=dk, dv=dv,
                      fwd_workspace=ws_f)
        if cw is not None:   # through the key conv: gradients of the original keys and of the weights
            moba.key_conv_backward(kd, cw, cud, B, dk, workspace=ws_b, dk=dk_in, dw=dw)

    torch.cuda.reset_peak_memory_stats(dev)
    for _ in range(args.warmup):
        step(g["q"], g["k"], g["v"], g["dout"], g["cu_seqlens"], conv_w)
    torch.cuda.synchronize()
    status = moba.check_status(ws_f) | moba.check_status(ws_b)
    pairs = int((sel >= 0).sum().item())
    pos = torch.cat([torch.arange(b - a) for a, b in zip(x["cu_seqlens"][:-1].tolist(),
                                                         x["cu_seqlens"][1:].tolist())]).double()
    scored = float((pos // B).sum().item()) * hq
    # Exact useful work (the nominal count above assumes k full blocks per
    # row): a past block contributes B keys, the own block the (p mod B) + 1
    # keys up to the query, and early queries hold fewer than k picks.
    n_visible = visible_keys(pos, B, hq, pairs)
    useful_fwd = 4.0 * d * n_visible
    useful_bwd = 2.5 * useful_fwd
    # Planted needles (query, head, block) that the router picked.
    needle_recall = None
    if x.get("needles"):
        nd = torch.tensor([[hq_, i_, j_] for _, hq_, i_, j_ in x["needles"]], dtype=torch.long, device=dev)
        rows_sel = sel[nd[:, 1], nd[:, 0]]
        picked = int((rows_sel == nd[:, 2:3].to(torch.int32)).any(dim=1).sum().item())
        needle_recall = {"planted": int(nd.shape[0]), "picked": picked}

    stream = torch.cuda.current_stream()
    stage_sets = [moba.StageEvents() for _ in range(args.steps)]
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clocks:
        ev0.record(stream)
        for i in range(args.steps):
            with stage_sets[i]:
                step(g["q"], g["k"], g["v"], g["dout"], g["cu_seqlens"], conv_w)
        ev1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = ev0.elapsed_time(ev1) / args.steps
    ms_max = reduce_max(ms, dev, world)
    stage_ms = {}
    for s in moba.STAGES:
        stage_ms[s] = statistics.mean(e.ms()[s] for e in stage_sets)
    fwd_ms = sum(v for k_, v in stage_ms.items() if k_.startswith("fwd"))
    bwd_ms = sum(v for k_, v in stage_ms.items() if k_.startswith("bwd") or k_ == "conv_bwd")

    value = aggregate_value(total_flops, ms_max)
    peak_t = float(peaks["bf16_tflops"])

    dom = max(stage_ms, key=stage_ms.get)
    bound, amount, unit = stage_roofline(dom, w, pairs, scored, peaks)
    if bound == "tensor":
        achieved = amount / (stage_ms[dom] * 1e-3) / 1e12
        peak, runit = peak_t, "TFLOP/s"
    else:
        achieved = amount / (stage_ms[dom] * 1e-3) / 1e9
        peak, runit = float(peaks["hbm_gbs"]), "GB/s"
    # the captured traffic is for one launch of the headline workload on one GPU
    tr = NCU_TRAFFIC.get(dom) if args.workload == synth.HEADLINE and not sharded else None
    traffic = tr["bytes"] if tr and tr.get("sha") == src_sha(KERNEL_SRC.get(dom, "fwd.cu")) else None
    roofline = {"kernel": dom, "bound": bound, "achieved": round(achieved, 3), "peak": peak, "unit": runit,
                "frac": round(achieved / peak, 4), "traffic": traffic,
                "peak_source": "%s (MEASURED_PEAKS.json burst)" % peak_src if bound == "tensor" else peak_src,
                "per_unit": ("%s per (query, head, block) pair; %d pairs per launch" %
                             ("4*B*d FLOP" if dom == "fwd_attn" else "10*B*d FLOP", pairs))
                if dom in ("fwd_attn", "bwd_attn") else unit}

    # Memory: every buffer of the step is a torch allocation, so the peak
    # covers inputs, outputs and both workspaces.  For context, the dense
    # router-score matrix a materialising implementation would hold.
    nb = T // B + w.batch
    memory = {"peak_allocated_bytes": int(torch.cuda.max_memory_allocated(dev)),
              "fwd_workspace_bytes": int(moba.fwd_workspace_size(shape)),
              "bwd_workspace_bytes": int(moba.bwd_workspace_size(shape)),
              "router_scores_if_materialised_bytes": int(T) * hq * nb * 4}

    # End to end through the public API with host buffers: every step copies
    # its inputs from pinned host memory and reads all its results (O, LSE
    # and the gradients) back.  Steps are pipelined the way a user would run
    # them: inputs and outputs double-buffered on the device, host->device
    # copies on one stream, the kernels on another, device->host copies on a
    # third, so step i+1's upload and step i-1's download overlap step i.
    e2e = None
    if not args.no_e2e:
        names_in = ["q", "k", "v", "dout"] + (["conv_w"] if conv_w is not None else []) + ["cu_seqlens"]
        host = {n: x[n].pin_memory() for n in names_in}
        h2d = sum(t.numel() * t.element_size() for t in host.values())

        def out_set():
            o = {"out": torch.empty_like(out), "lse": torch.empty_like(lse), "dq": torch.empty_like(dq),
                 "dk": torch.empty_like(dk), "dv": torch.empty_like(dv)}
            if conv_w is not None:
                o["dk_in"], o["dw"] = torch.empty_like(dk_in), torch.empty_like(dw)
            return o

        dev_in = [{n: torch.empty_like(g[n]) for n in names_in} for _ in range(2)]
        dev_out = [out_set() for _ in range(2)]
        # The step's results: O, LSE, dQ, dV and the key gradients the caller
        # holds (dK and dW of the original keys when the conv is applied; dK'
        # is then an intermediate that stays on the device).
        results = ["out", "lse", "dq", "dv"] + (["dk_in", "dw"] if conv_w is not None else ["dk"])
        host_out = [{n: torch.empty(o[n].shape, dtype=o[n].dtype, pin_memory=True) for n in results} for o in dev_out]
        d2h = sum(dev_out[0][n].numel() * dev_out[0][n].element_size() for n in results)
        s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_fwd = [torch.cuda.Event() for _ in range(2)]
        ev_cmp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        sel_e = torch.empty_like(sel)
        kc_e = torch.empty_like(g["k"]) if w.conv_width else None

        def e2e_step(i):
            b = i % 2
            di, do_, ho = dev_in[b], dev_out[b], host_out[b]
            s_in.wait_event(ev_cmp[b])            # step i-2 is done with this input set
            with torch.cuda.stream(s_in):
                for n in names_in:
                    di[n].copy_(host[n], non_blocking=True)
                ev_in[b].record(s_in)
            s_cmp.wait_event(ev_in[b])
            s_cmp.wait_event(ev_out[b])           # step i-2's results have left this output set
            with torch.cuda.stream(s_cmp):
                cw = di.get("conv_w")
                _, _, _, k_used = moba.forward(di["q"], di["k"], di["v"], di["cu_seqlens"], B, topk, conv_w=cw,
                                               workspace=ws_f, out=do_["out"], lse=do_["lse"], sel_idx=sel_e,
                                               k_conv=kc_e)
                ev_fwd[b].record(s_cmp)
                moba.backward(di["q"], k_used, di["v"], do_["out"], do_["lse"], di["dout"], sel_e,
                              di["cu_seqlens"], B, workspace=ws_b, dq=do_["dq"], dk=do_["dk"], dv=do_["dv"],
                              fwd_workspace=ws_f)
                if cw is not None:
                    moba.key_conv_backward(di["k"], cw, di["cu_seqlens"], B, do_["dk"], workspace=ws_b,
                                           dk=do_["dk_in"], dw=do_["dw"])
                ev_cmp[b].record(s_cmp)
            s_out.wait_event(ev_fwd[b])
            with torch.cuda.stream(s_out):
                ho["out"].copy_(do_["out"], non_blocking=True)
                ho["lse"].copy_(do_["lse"], non_blocking=True)
            s_out.wait_event(ev_cmp[b])
            with torch.cuda.stream(s_out):
                for n in results:
                    if n not in ("out", "lse"):
                        ho[n].copy_(do_[n], non_blocking=True)
                ev_out[b].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        ne = max(3, min(2 * args.steps, 20))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for i in range(ne):
            e2e_step(i)
        e1.record(s_out)
        torch.cuda.synchronize()
        ems = reduce_max(e0.elapsed_time(e1) / ne, dev, world)
        e2e = {"value": round(aggregate_value(total_flops, ems), 3), "unit": UNIT, "ms_per_step": round(ems, 3),
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": ne,
               "pipelining": "inputs/outputs double-buffered; upload, kernels, download on three streams"}
        if moba.check_status(ws_f) | moba.check_status(ws_b):
            status |= moba.check_status(ws_f) | moba.check_status(ws_b)

    # Context only: dense causal attention (the library SDPA, flash backend)
    # forward + backward on the same Q, K, V shapes.
    dense = None
    if rank == 0 and world == 1 and not args.no_dense:
        dense = dense_context(g, hq, hkv, ms_max)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        vals, desc, cores = oracle_sample(w, seed, args.cpu_rows, 1, 0)
        cpu = {"value": round(statistics.mean(vals), 9), "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": desc, "nproc": os.cpu_count(), "cpu_model": cpu_model()}

    if world > 1:
        dist.barrier()
    if rank == 0:
        in_bytes = sum(g[n].numel() * g[n].element_size() for n in ("q", "k", "v", "dout"))
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_max, 4), "higher_is_better": True,
            "scaling": "strong" if sharded else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "seq_len": T, "batch": w.batch, "h_q": hq, "h_kv": hkv, "head_dim": d,
                       "block_size": B, "topk": topk, "conv_width": w.conv_width,
                       "needles_per_head": w.needles_per_head,
                       "l2": "inputs %.0f MB > %d MB L2 (no flush)" % (in_bytes / 1e6, L2_BYTES >> 20),
                       "parallelism": parallelism},
            "fwd_ms": round(fwd_ms, 4), "bwd_ms": round(bwd_ms, 4),
            "fwd_tflops": round(w.fwd_flops() / (fwd_ms * 1e-3) / 1e12, 3),
            "bwd_tflops": round(w.bwd_flops() / (bwd_ms * 1e-3) / 1e12, 3),
            "pct_of_bf16_peak": round(100.0 * value / world / peak_t, 3),
            "peak_bf16_tflops": peak_t, "peak_source": peak_src,
            "stage_ms": {k_: round(v, 4) for k_, v in stage_ms.items()},
            "pairs": pairs,
            # rank 0's useful work (its shard, or its replica) times the ranks
            "useful": {"visible_keys": int(n_visible), "of_nominal": round(n_visible / (T * hq * topk * B), 4),
                       "fwd_tflops": round(useful_fwd / (fwd_ms * 1e-3) / 1e12, 3),
                       "bwd_tflops": round(useful_bwd / (bwd_ms * 1e-3) / 1e12, 3),
                       "step_tflops": round(aggregate_value((useful_fwd + useful_bwd) * world, ms_max), 3)},
            "needle_recall": needle_recall,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "memory": memory,
            "dense_context": dense,
            "gpu_launches": (LAUNCHES_PER_STEP + (LAUNCHES_CONV_BWD if w.conv_width else 0)) * args.steps, "clocks": clocks.summary(), "device_status": status,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    w = synth.WORKLOADS[args.workload]
    vals, desc, cores = oracle_sample(w, w.seed, args.ref_rows, args.steps, args.warmup)
    v = statistics.mean(vals)
    flops_row = 3.5 * 4.0 * w.topk * w.block_size * w.head_dim
    ms = args.ref_rows * flops_row / (v * 1e12) * 1e3
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 9), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "seq_len": w.total_tokens, "batch": w.batch, "h_q": w.h_q,
                       "h_kv": w.h_kv, "head_dim": w.head_dim, "block_size": w.block_size, "topk": w.topk,
                       "conv_width": w.conv_width, "needles_per_head": w.needles_per_head,
                       "sample_rows_per_step": args.ref_rows},
            "cpu_baseline": {"value": round(v, 9), "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc,
                             "nproc": os.cpu_count(), "cpu_model": cpu_model()},
            "e2e": {"value": round(v, 9), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(synth.WORKLOADS), default=synth.HEADLINE)
    ap.add_argument("--shard", choices=["heads", "replica"], default="heads",
                    help="N > 1: split one problem's KV-head groups over the ranks, or run one problem per rank")
    ap.add_argument("--heads", type=int, default=0,
                    help="override the KV head count (query heads scale with it); for small profiling runs")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense-attention context timing")
    ap.add_argument("--cpu-rows", type=int, default=65536, help="oracle rows per CPU-baseline step")
    ap.add_argument("--ref-rows", type=int, default=4096, help="oracle rows per --impl reference step")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")
    if args.heads:
        import dataclasses
        w = synth.WORKLOADS[args.workload]
        g = w.h_q // w.h_kv
        name = "%s_kvheads%d" % (w.name, args.heads)
        synth.WORKLOADS[name] = dataclasses.replace(w, name=name, h_kv=args.heads, h_q=args.heads * g)
        args.workload = name
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
