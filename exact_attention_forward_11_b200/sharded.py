"""Head-sharded attention forward over several GPUs (one process per GPU).

The (batch, head) problems of attention are independent ("Self-Attention, CUDA
kernels and FlashAttention", section 1, multi-head paragraph: every head attends
on its own), so a job splits the B*H heads of one batch across ranks with no
exchange while it computes. When every rank needs the whole output (the way a
tensor-parallel layer hands its sharded result on, "FlashAttention scaling,
multi-GPU training and weight quantization", section 2, the All-Gather of
sharded tensors over NVLink), one all-gather of O (and LSE) follows.

Layout: heads are numbered over the flattened B*H axis; rank r owns the
contiguous range head_range(BH, world, r) (sizes differ by at most one). Inputs
are [B, H, N, d] on every rank; only the rank's own heads are read (pointer
offsets into the contiguous tensors, no copy). The gather sends equal-sized
blocks (the largest range, padded), as NCCL's all-gather requires, and the
result is cut back to B*H heads.

The collective is the only cross-rank step and runs through torch.distributed
(NCCL on GPUs; the same code runs on CPU tensors with gloo, which is how the
partition and the gather are tested without GPUs).
"""
from __future__ import annotations


def head_range(BH: int, world: int, rank: int):
    """(first head, head count) of `rank` when BH heads are split over `world`
    ranks in contiguous ranges whose sizes differ by at most one."""
    if world < 1 or not 0 <= rank < world or BH < 0:
        raise ValueError("bad partition arguments")
    base, extra = divmod(BH, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def gather_heads(local, BH: int, group=None):
    """All-gather of per-rank head blocks.

    local: tensor [count, ...] holding this rank's heads (count from head_range).
    Returns the tensor [BH, ...] on every rank, identical to the unsharded one.
    """
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    per = -(-BH // world)                       # largest range
    tail = tuple(local.shape[1:])
    send = torch.zeros((per,) + tail, dtype=local.dtype, device=local.device)
    send[:local.shape[0]] = local
    recv = torch.empty((world * per,) + tail, dtype=local.dtype, device=local.device)
    dist.all_gather_into_tensor(recv, send, group=group)
    parts = []
    for r in range(world):
        _, cnt = head_range(BH, world, r)
        parts.append(recv[r * per:r * per + cnt])
    return torch.cat(parts, dim=0)


def forward_heads(q, k, v, start, count, causal=False, scale=None, stream=None):
    """O [count, N, d] and LSE [count, N] of the heads [start, start + count) of the
    flattened B*H axis, computed by attn_fwd on pointer offsets into q, k, v (no copy)."""
    import torch

    from . import _check, _expect, _shape4, _stream_ptr, attn_fwd, ATTN_BF16
    B, H, N, d = _shape4(q)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _expect(t, name, (B, H, N, d), torch.bfloat16, q.device)
    if start < 0 or count < 0 or start + count > B * H:
        raise ValueError("head range outside the tensor")
    o_loc = torch.empty((count, N, d), dtype=torch.bfloat16, device=q.device)
    l_loc = torch.empty((count, N), dtype=torch.float32, device=q.device)
    if count > 0:
        off = start * N * d * q.element_size()
        sc = 0.0 if scale is None else float(scale)
        _check(attn_fwd(q.data_ptr() + off, k.data_ptr() + off, v.data_ptr() + off, o_loc.data_ptr(),
                        l_loc.data_ptr(), 1, count, N, d, sc, int(bool(causal)), ATTN_BF16,
                        _stream_ptr(q, stream)), "attn_fwd")
    return o_loc, l_loc


def forward_sharded(q, k, v, causal=False, scale=None, group=None, stream=None):
    """O, LSE of attention over q, k, v [B, H, N, d] (bf16 CUDA, the same on every
    rank), computed head-sharded: this rank runs attn_fwd on its own heads only,
    then one all-gather gives every rank the full O [B, H, N, d] and LSE [B, H, N]."""
    import torch.distributed as dist
    B, H, N, d = q.shape
    BH = B * H
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    start, cnt = head_range(BH, world, rank)
    o_loc, l_loc = forward_heads(q, k, v, start, cnt, causal=causal, scale=scale, stream=stream)
    o = gather_heads(o_loc, BH, group).view(B, H, N, d)
    lse = gather_heads(l_loc, BH, group).view(B, H, N)
    return o, lse
