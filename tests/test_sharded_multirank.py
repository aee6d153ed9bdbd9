"""Head-sharded forward, host side, on CPU with gloo ranks (no GPU).

Every rank computes its own contiguous range of the B*H heads and one all-gather
returns the full output to every rank. Here the per-rank compute is the fp64
oracle on the rank's heads (the CUDA library needs a GPU); the partition and the
gather are the product's (exact_attention_forward_11_b200.sharded), and the
gathered O and LSE must equal the unsharded oracle result bit for bit, with
world sizes that split the heads evenly and unevenly (including ranks that own
no head).
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, B, H, out):
    import datetime
    import sys
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch
    import torch.distributed as dist
    import workloads
    from exact_attention_forward_11_b200.sharded import gather_heads, head_range
    from oracle import attention_fp64
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        N, d = 40, 8
        q, k, v = workloads.make_qkv(B, H, N, d, seed=31)
        BH = B * H
        start, cnt = head_range(BH, world, rank)
        flat = [t.double().reshape(BH, N, d)[start:start + cnt] for t in (q, k, v)]
        o_loc, l_loc = attention_fp64(*(t.numpy() for t in flat), 0.35, True)
        o = gather_heads(torch.from_numpy(o_loc), BH)
        lse = gather_heads(torch.from_numpy(l_loc), BH)
        out[rank] = (o.numpy().tobytes(), lse.numpy().tobytes(), (start, cnt))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,B,H", [(2, 2, 3), (3, 1, 4), (4, 1, 2)])
def test_partition_and_gather_reproduce_the_unsharded_result(world, B, H):
    import workloads
    from oracle import attention_fp64
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, B, H, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        res = dict(out)
    N, d = 40, 8
    q, k, v = workloads.make_qkv(B, H, N, d, seed=31)
    o_ref, l_ref = attention_fp64(*(t.double().reshape(B * H, N, d).numpy() for t in (q, k, v)), 0.35, True)
    ranges = sorted(r[2] for r in res.values())
    assert sum(c for _, c in ranges) == B * H and ranges[0][0] == 0
    for (s0, c0), (s1, _) in zip(ranges, ranges[1:]):
        assert s0 + c0 == s1                                  # contiguous, no gap, no overlap
    assert max(c for _, c in ranges) - min(c for _, c in ranges) <= 1
    for rank in range(world):
        o = np.frombuffer(res[rank][0], dtype=np.float64).reshape(o_ref.shape)
        lse = np.frombuffer(res[rank][1], dtype=np.float64).reshape(l_ref.shape)
        np.testing.assert_array_equal(o, o_ref)
        np.testing.assert_array_equal(lse, l_ref)


def test_head_range_rejects_bad_arguments():
    from exact_attention_forward_11_b200.sharded import head_range
    with pytest.raises(ValueError):
        head_range(8, 0, 0)
    with pytest.raises(ValueError):
        head_range(8, 2, 2)
    assert head_range(5, 8, 7) == (5, 0)
