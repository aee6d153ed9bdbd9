"""Host logic of the multi-GPU benchmark path on CPU: two gloo ranks.

The attention units (batch, head) are independent, so N GPUs run N replicas with no
data-path collective; the only cross-rank steps are the start/stop barrier and the
maximum of the per-rank times. This test runs exactly those steps of bench.py with
world_size 2 on the gloo backend.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import sys
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist
    import bench
    import workloads
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        r, w, local = bench.dist_env()
        bench.barrier(w)
        t = bench.max_over_ranks(10.0 + 5.0 * rank, w)
        wl = workloads.WORKLOADS["llm_train_causal"]
        out[rank] = (r, w, local, t, bench.shard_seed(wl, rank))
        bench.barrier(w)
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction_and_sharding():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        res = dict(out)
    assert sorted(res) == [0, 1]
    for rank, (r, w, local, t, seed) in res.items():
        assert (r, w, local) == (rank, world, rank)
        assert t == 15.0                     # max over ranks, seen identically by both
    assert res[0][4] != res[1][4]            # each replica draws its own data
