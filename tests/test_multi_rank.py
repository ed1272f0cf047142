"""Host logic of the multi-GPU bench path on CPU, as two gloo ranks.

* Replicas: the max-over-ranks step time, the whole-job aggregate and
  per-rank seeds (every rank runs an independent problem).
* Head sharding: each rank takes a contiguous range of KV-head groups of one
  seeded problem; run through the oracle, the shards reassemble exactly the
  full problem's results (heads are independent: no collective is needed),
  and the ranges cover every head once.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run(target, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res, key=lambda r: r[0])


def _init(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))


def _replica_worker(rank, world, port, q):
    _init(rank, world, port)
    import bench
    from block_sparse_long_key_b200 import synth
    try:
        ws, r, local = bench.dist_env()
        ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        ms_max = bench.reduce_max(ms, torch.device("cpu"), ws)
        w = synth.WORKLOADS[synth.HEADLINE]
        val = bench.aggregate_value(ws * (w.fwd_flops() + w.bwd_flops()), ms_max)
        seeds = [None] * ws
        dist.all_gather_object(seeds, bench.rank_seed(w, r))
        q.put((rank, ws, r, local, ms_max, val, seeds))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_step_time_and_aggregate():
    res = _run(_replica_worker)
    from block_sparse_long_key_b200 import synth
    w = synth.WORKLOADS[synth.HEADLINE]
    flops = w.fwd_flops() + w.bwd_flops()
    for rank, ws, r, local, ms_max, val, seeds in res:
        assert ws == 2 and r == rank and local == rank
        assert ms_max == 15.0                              # max over ranks
        assert val == pytest.approx(2 * flops / 15e-3 / 1e12)
        assert len(set(seeds)) == 2                        # independent problems


def _oracle_step(x, w):
    """Forward + backward of a (sharded) problem through the fp64 oracle."""
    from oracle import moba_oracle_c as orc
    cu = x["cu_seqlens"].numpy()
    q, k, v = (x[n].double().numpy() for n in ("q", "k", "v"))
    k = orc.key_conv(k, x["conv_w"].double().numpy(), cu)
    cents = orc.block_centroids(k, cu, w.block_size)
    sel, _ = orc.route(q, cents, cu, w.block_size, w.topk)
    o, lse = orc.attention(q, k, v, sel, cu, w.block_size)
    dq, dk, dv = orc.attention_backward(q, k, v, x["dout"].double().numpy(), sel, cu, w.block_size)
    return dict(sel=sel, o=o, lse=lse, dq=dq, dk=dk, dv=dv)


def _shard_worker(rank, world, port, q):
    _init(rank, world, port)
    import bench
    from block_sparse_long_key_b200 import synth
    try:
        w = synth.small((300, 170), 6, 3, 64, 16, 4, conv_width=3, seed=5)   # GQA 2:1, 3 KV heads
        kv0, kv1 = bench.head_shard(w.h_kv, world, rank)
        x = synth.make_inputs(w)                        # the same seeded problem on every rank
        xs, ws_ = bench.shard_inputs(x, w, kv0, kv1)
        mine = _oracle_step(xs, ws_)
        ranges = [None] * world
        dist.all_gather_object(ranges, (kv0, kv1))
        full = _oracle_step(x, w)                       # for the check only
        g = w.h_q // w.h_kv
        ok = {n: bool(np.array_equal(mine[n], full[n][:, kv0 * g:kv1 * g]))
              for n in ("sel", "o", "lse", "dq")}
        ok.update({n: bool(np.array_equal(mine[n], full[n][:, kv0:kv1])) for n in ("dk", "dv")})
        q.put((rank, ranges, ok, ws_.h_kv, ws_.h_q))
    finally:
        dist.destroy_process_group()


def test_head_shards_reassemble_the_full_problem():
    res = _run(_shard_worker)
    ranges = res[0][1]
    assert ranges == res[1][1]
    covered = sorted(h for a, b in ranges for h in range(a, b))
    assert covered == list(range(3))                   # every KV head exactly once
    for rank, _, ok, hkv, hq in res:
        assert all(ok.values()), (rank, ok)
        assert hq == 2 * hkv


@pytest.mark.parametrize("h_kv,world", [(16, 8), (8, 3), (3, 2), (5, 5), (1, 1)])
def test_head_shard_ranges(h_kv, world):
    import bench
    r = [bench.head_shard(h_kv, world, k) for k in range(world)]
    assert r[0][0] == 0 and r[-1][1] == h_kv
    assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
    sizes = [b - a for a, b in r]
    assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
