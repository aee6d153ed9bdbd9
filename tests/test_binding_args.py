"""The Python binding refuses, before anything reaches the library, every tensor the
kernels could not use: a host tensor, another device, a wrong shape, dtype or layout,
or an undersized output. (The CPU tests need no GPU; the GPU tests launch nothing.)"""
import pytest
import torch

import exact_attention_forward_11_b200 as attn


def test_host_tensors_are_refused_on_cpu():
    q = torch.zeros(1, 1, 16, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        attn.forward(q, q, q)
    with pytest.raises(ValueError):
        attn.quantize_fp8(torch.zeros(1, 1, 16, 128, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        attn.forward(q[..., ::2], q[..., ::2], q[..., ::2])   # not contiguous


@pytest.mark.gpu
def test_every_argument_is_checked(cuda_lib):
    dev = torch.device("cuda:0")
    B, H, N, d = 1, 2, 130, 128
    q = torch.zeros(B, H, N, d, dtype=torch.bfloat16, device=dev)
    bad_cases = [
        dict(k=q.cpu()),                                                   # host tensor
        dict(v=q.float()),                                                 # wrong dtype
        dict(k=q[:, :, :N - 1].contiguous()),                              # wrong shape
        dict(out=torch.empty(B, H, N - 1, d, dtype=torch.bfloat16, device=dev)),   # undersized output
        dict(out=torch.empty(B, H, d, N, dtype=torch.bfloat16, device=dev).transpose(2, 3)),  # not contiguous
        dict(lse=torch.empty(B, H, N, dtype=torch.float16, device=dev)),   # wrong LSE dtype
        dict(lse=torch.empty(B, H, N - 1, dtype=torch.float32, device=dev)),
    ]
    for case in bad_cases:
        args = dict(k=q, v=q)
        args.update(case)
        with pytest.raises(ValueError):
            cuda_lib.forward(q, args.pop("k"), args.pop("v"), **args)
    with pytest.raises(ValueError):
        cuda_lib.quantize_fp8(q, torch.zeros(d, d - 1, dtype=torch.bfloat16, device=dev))
    with pytest.raises(ValueError):
        cuda_lib.quantize_fp8(q.float())
    c = torch.zeros(B, H, N, d, dtype=torch.uint8, device=dev)
    s = torch.ones(B, H, 2, dtype=torch.float32, device=dev)
    with pytest.raises(ValueError):
        cuda_lib.forward_fp8(c, c, c, s, s, s[:, :, :1].contiguous())    # scales must cover ceil(N/128) tiles
    with pytest.raises(ValueError):
        cuda_lib.forward_fp8(c, c.cpu(), c, s, s, s)
    torch.cuda.synchronize()
    assert cuda_lib.attn_get_device_status(None) == cuda_lib.ATTN_OK


def test_w4a16_workspace_cache_is_zeroed_after_a_failed_status(monkeypatch):
    """The split-K workspaces w4a16_matmul caches per (device, stream) hold tickets
    that a timed-out launch may leave set: a device status other than ATTN_OK
    zeroes every cached workspace; ATTN_OK leaves them alone. (Host logic only: a
    fake library answers the status call and the cache holds CPU tensors.)"""
    class FakeLib:
        status = attn.ATTN_OK

        def attn_get_device_status(self, stream):
            return self.status

    fake = FakeLib()
    monkeypatch.setattr(attn, "load", lambda: fake)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    cache = {(0, 1): torch.full((64,), 7, dtype=torch.uint8), (0, 2): torch.full((32,), 9, dtype=torch.uint8)}
    monkeypatch.setattr(attn, "_W4_WORKSPACES", cache)
    assert attn.attn_get_device_status(None) == attn.ATTN_OK
    assert all(bool((t != 0).all()) for t in cache.values())
    fake.status = attn.ATTN_ERR_TIMEOUT
    assert attn.attn_get_device_status(None) == attn.ATTN_ERR_TIMEOUT
    assert all(int(t.count_nonzero()) == 0 for t in cache.values())
    assert set(cache) == {(0, 1), (0, 2)}                  # kept, zeroed, not dropped
