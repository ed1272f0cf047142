"""Host logic of the multi-GPU bench path on CPU: two gloo ranks check the
max-over-ranks step time, the whole-job aggregate and per-rank seeds (every
rank runs an independent problem: no data-path collective)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    import bench
    from block_sparse_long_key_b200 import synth
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        ws, r, local = bench.dist_env()
        ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        ms_max = bench.reduce_max(ms, torch.device("cpu"), ws)
        w = synth.WORKLOADS[synth.HEADLINE]
        val = bench.aggregate_value(w.fwd_flops() + w.bwd_flops(), ws, ms_max)
        seeds = [None] * ws
        dist.all_gather_object(seeds, bench.rank_seed(w, r))
        q.put((rank, ws, r, local, ms_max, val, seeds))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_step_time_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    from block_sparse_long_key_b200 import synth
    w = synth.WORKLOADS[synth.HEADLINE]
    flops = w.fwd_flops() + w.bwd_flops()
    for rank, ws, r, local, ms_max, val, seeds in res:
        assert ws == 2 and r == rank and local == rank
        assert ms_max == 15.0                              # max over ranks
        assert val == pytest.approx(2 * flops / 15e-3 / 1e12)
        assert len(set(seeds)) == 2                        # independent problems
