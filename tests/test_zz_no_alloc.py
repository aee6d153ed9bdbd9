"""attn_bwd_noalloc: the backward pass for callers that cannot allocate device memory.

Some users of this library run the backward pass where they may not call
cudaMalloc: an operator plugin inside a framework that owns the whole device
memory pool and gives plugins no scratch buffer, or a latency-critical service
where an allocation could synchronise the device. attn_bwd_noalloc serves them:
it takes no workspace and keeps its scratch in a fixed array inside the library.

This file checks, on the GPU and through the C ABI, that the entry point gives
the same dQ, dK, dV as attn_bwd (within the backward tests' tolerance: 2 % of the
largest magnitude per element, 1 % in Frobenius norm), on two calls in a row
(the second call reuses the array the first one left behind), and that it
refuses shapes beyond its limit. It is collected last so that a run stopping at
the first failure has run every other test; it also passes on its own in a
fresh process, where its first call does the one-time set-up.
"""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


def _close(got, want, name):
    got, want = got.float().cpu().numpy(), want.float().cpu().numpy()
    assert np.isfinite(got).all(), name
    err = np.abs(got - want)
    assert err.max() <= 2e-2 * np.abs(want).max() + 1e-5, f"{name}: max err {err.max()}"
    assert np.linalg.norm(got - want) <= 1e-2 * np.linalg.norm(want) + 1e-5 * np.sqrt(want.size), name


@pytest.mark.parametrize("B,H,N,d,causal", [(2, 3, 700, 128, True), (1, 2, 300, 64, False)])
def test_noalloc_matches_attn_bwd_on_two_calls(cuda_lib, B, H, N, d, causal):
    lib = cuda_lib
    dev = torch.device("cuda:0")
    q, k, v = (x.to(dev) for x in workloads.make_qkv(B, H, N, d, seed=N + d))
    g = torch.Generator().manual_seed(N)
    dout = torch.randn((B, H, N, d), generator=g).to(torch.bfloat16).to(dev)
    o, lse = lib.forward(q, k, v, causal=causal)
    want = lib.backward(q, k, v, o, lse, dout, causal=causal)      # the entry point with a workspace
    torch.cuda.synchronize()
    for call in range(2):
        got = [torch.full_like(q, float("nan")) for _ in range(3)]
        st = lib.attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                  dout.data_ptr(), *(t.data_ptr() for t in got), B, H, N, d, 0.0, int(causal),
                                  None)
        assert st == lib.ATTN_OK, lib.attn_status_string(st)
        torch.cuda.synchronize()
        assert lib.attn_get_device_status(None) == lib.ATTN_OK
        for a, b, name in zip(got, want, ("dq", "dk", "dv")):
            _close(a, b, f"{name} (call {call + 1})")


def test_noalloc_refuses_shapes_beyond_its_limit(cuda_lib):
    lib = cuda_lib
    fake = 0x100000          # 16-byte aligned, never touched: the size check comes first
    rows = lib.ATTN_BWD_NOALLOC_MAX_ROWS
    st = lib.attn_bwd_noalloc(*([fake] * 9), 1, 1, rows + 128, 128, 0.0, 0, None)
    assert st == lib.ATTN_ERR_UNSUPPORTED
