"""The head-sharded forward on one GPU: every rank's share computed on its
pointer offsets equals the corresponding heads of the unsharded launch bit for
bit (the kernels compute each head alone), and the whole path - partition,
attn_fwd on the rank's heads, NCCL all-gather - runs end to end in a one-rank
NCCL group. (Several GPUs are not available to the tests; the gather across
ranks is covered on CPU by tests/test_sharded_multirank.py.)"""
import os
import socket

import pytest
import torch

import workloads
from exact_attention_forward_11_b200.sharded import forward_heads, forward_sharded, head_range

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 3, 5])
@pytest.mark.parametrize("causal", [False, True])
def test_rank_shares_equal_the_unsharded_heads(cuda_lib, world, causal):
    dev = torch.device("cuda:0")
    B, H, N, d = 2, 3, 300, 128
    q, k, v = (x.to(dev) for x in workloads.make_qkv(B, H, N, d, seed=17))
    o, lse = cuda_lib.forward(q, k, v, causal=causal)
    parts_o, parts_l = [], []
    for r in range(world):
        start, cnt = head_range(B * H, world, r)
        o_r, l_r = forward_heads(q, k, v, start, cnt, causal=causal)
        parts_o.append(o_r)
        parts_l.append(l_r)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts_o).view(B, H, N, d).view(torch.int16), o.view(torch.int16))
    assert torch.equal(torch.cat(parts_l).view(B, H, N).view(torch.int32), lse.view(torch.int32))


def test_one_rank_nccl_group_end_to_end(cuda_lib):
    import datetime
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda:0"))
    try:
        dev = torch.device("cuda:0")
        q, k, v = (x.to(dev) for x in workloads.make_qkv(1, 4, 257, 64, seed=5))
        o, lse = forward_sharded(q, k, v, causal=True)
        o_ref, lse_ref = cuda_lib.forward(q, k, v, causal=True)
        torch.cuda.synchronize()
        assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16))
        assert torch.equal(lse.view(torch.int32), lse_ref.view(torch.int32))
    finally:
        dist.destroy_process_group()
