"""The bounded-wait failure path on the GPU, with the failure planted on purpose
(include/attn_b200_testing.h): one work unit's first K tile is never loaded, so
the MMA warp's wait on it can only run out. The launch must end by itself, the
host must read ATTN_ERR_TIMEOUT from the status word, every unit that was not
starved must still be exact, and the next ordinary call must succeed (the CUDA
context stays usable). No GPU fault, trap or endless wait is involved: every
wait of the kernel has a cycle limit, here 2^22 cycles (about 2-3 ms).
"""
import time

import numpy as np
import pytest
import torch

import workloads
from oracle import attention_fp64

pytestmark = pytest.mark.gpu

WAIT_LIMIT = 1 << 22


def _inputs(B, H, N, d, seed):
    return workloads.make_qkv(B, H, N, d, seed)


def test_starved_unit_times_out_and_context_survives(cuda_lib):
    lib = cuda_lib
    dev = torch.device("cuda:0")
    B, H, N, d = 1, 4, 1024, 128          # 4 heads x 4 Q-tile pairs = 16 units, one per CTA
    q, k, v = _inputs(B, H, N, d, seed=2024)
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    o = torch.full((B, H, N, d), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=dev)
    assert lib.attn_get_device_status(None) == lib.ATTN_OK   # nothing pending from earlier tests

    fault_unit = 5                        # head 1, Q-tile pair 2 (units count pairs down, heads fastest)
    t0 = time.time()
    st = lib.attn_fwd_inject_timeout(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                     B, H, N, d, 0.0, 0, fault_unit, WAIT_LIMIT, None)
    assert st == lib.ATTN_OK, lib.attn_status_string(st)
    assert lib.attn_get_device_status(None) == lib.ATTN_ERR_TIMEOUT
    assert time.time() - t0 < 30.0
    assert lib.attn_get_device_status(None) == lib.ATTN_OK   # the word was cleared

    # every other unit finished normally: check the rows of the heads that were not starved
    # (unit u -> pair NPAIR-1-u//H, head u%H with NPAIR = 4; unit 5 is head 1)
    o_h = o.float().cpu().numpy()
    lse_h = lse.cpu().numpy()
    scale = 1.0 / np.sqrt(d)
    rows = np.array([0, 131, 517, 1023])
    o_ref, lse_ref = attention_fp64(q.double().numpy(), k.double().numpy(), v.double().numpy(), scale, False,
                                    rows=rows)
    for h in (0, 2, 3):
        assert np.abs(o_h[0, h, rows] - o_ref[0, h]).max() <= 2e-2
        assert np.abs(lse_h[0, h, rows] - lse_ref[0, h]).max() <= 1e-3

    # the context is usable: an ordinary call on the same buffers is exact everywhere
    lib.forward(qd, kd, vd, causal=False, out=o, lse=lse)
    torch.cuda.synchronize()
    assert lib.attn_get_device_status(None) == lib.ATTN_OK
    o_h = o.float().cpu().numpy()
    assert np.isfinite(o_h).all()
    o_ref, _ = attention_fp64(q.double().numpy(), k.double().numpy(), v.double().numpy(), scale, False,
                              rows=np.arange(256, 512))
    assert np.abs(o_h[0, 1, 256:512] - o_ref[0, 1]).max() <= 2e-2


def test_inject_timeout_validates_arguments(cuda_lib):
    lib = cuda_lib
    bad = lib.attn_fwd_inject_timeout(0, 0, 0, 0, 0, 1, 1, 128, 128, 0.0, 0, 0, WAIT_LIMIT, None)
    assert bad == lib.ATTN_ERR_INVALID_ARG


def test_one_tile_starved_unit_times_out_and_context_survives(cuda_lib):
    """The same planted failure on the one-Q-tile schedule (the kernel behind
    small attn_fwd launches and attn_fwd_mxfp8)."""
    lib = cuda_lib
    dev = torch.device("cuda:0")
    B, H, N, d = 1, 4, 1024, 128          # 4 heads x 8 Q tiles = 32 units, one per CTA
    q, k, v = _inputs(B, H, N, d, seed=2025)
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    o = torch.full((B, H, N, d), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=dev)
    assert lib.attn_get_device_status(None) == lib.ATTN_OK

    fault_unit = 5                        # unit u -> tile 7 - u // 4 of head u % 4: head 1, rows 768..895
    t0 = time.time()
    st = lib.attn_fwd_one_tile_inject_timeout(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(),
                                              lse.data_ptr(), B, H, N, d, 0.0, 0, fault_unit, WAIT_LIMIT, None)
    assert st == lib.ATTN_OK, lib.attn_status_string(st)
    assert lib.attn_get_device_status(None) == lib.ATTN_ERR_TIMEOUT
    assert time.time() - t0 < 30.0
    assert lib.attn_get_device_status(None) == lib.ATTN_OK

    o_h = o.float().cpu().numpy()
    lse_h = lse.cpu().numpy()
    scale = 1.0 / np.sqrt(d)
    rows = np.array([0, 131, 517, 767, 896, 1023])
    o_ref, lse_ref = attention_fp64(q.double().numpy(), k.double().numpy(), v.double().numpy(), scale, False,
                                    rows=rows)
    for h in range(H):                    # every tile but the starved one is exact, head 1 included
        assert np.abs(o_h[0, h, rows] - o_ref[0, h]).max() <= 2e-2
        assert np.abs(lse_h[0, h, rows] - lse_ref[0, h]).max() <= 1e-3

    lib.forward(qd, kd, vd, causal=False, out=o, lse=lse)
    torch.cuda.synchronize()
    assert lib.attn_get_device_status(None) == lib.ATTN_OK
    o_ref, _ = attention_fp64(q.double().numpy(), k.double().numpy(), v.double().numpy(), scale, False,
                              rows=np.arange(768, 896))
    assert np.abs(o.float().cpu().numpy()[0, 1, 768:896] - o_ref[0, 1]).max() <= 2e-2


@pytest.mark.parametrize("causal", [False, True])
def test_mxfp8_starved_unit_times_out_and_context_survives(cuda_lib, causal):
    """The planted failure in the MXFP8 forward: beyond the producer / MMA waits it
    runs out the converter warps' waits, the half-row exchange between the two
    softmax warpgroups and the hand-over of the V scale maxima. Every other unit
    (one per CTA here) is bit-identical to an ordinary launch, and the next
    ordinary launch is too."""
    lib = cuda_lib
    dev = torch.device("cuda:0")
    B, H, N, d = 1, 4, 1024, 128          # 4 heads x 8 Q tiles = 32 units, one per CTA
    q, k, v = (x.to(dev) for x in _inputs(B, H, N, d, seed=2027))
    (q8, qs), (k8, ks), (v8, vs) = (lib.quantize_mxfp8(x) for x in (q, k, v))
    o_ref, lse_ref = lib.forward_mxfp8(q8, k8, v8, qs, ks, vs, causal=causal)
    torch.cuda.synchronize()
    assert lib.attn_get_device_status(None) == lib.ATTN_OK

    o = torch.full((B, H, N, d), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=dev)
    # unit 5: non-causal, tile 7 - 5 // 4 of head 5 % 4 (rows 768..895 of head 1); causal
    # units are numbered the same way (heaviest tiles first), so also rows 768..895 of head 1
    fault_unit, h_f, rows_f = 5, 1, slice(768, 896)
    t0 = time.time()
    st = lib.attn_fwd_mxfp8_inject_timeout(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), qs.data_ptr(),
                                           ks.data_ptr(), vs.data_ptr(), o.data_ptr(), lse.data_ptr(), B, H, N, d,
                                           0.0, int(causal), fault_unit, WAIT_LIMIT, None)
    assert st == lib.ATTN_OK, lib.attn_status_string(st)
    assert lib.attn_get_device_status(None) == lib.ATTN_ERR_TIMEOUT
    assert time.time() - t0 < 30.0
    assert lib.attn_get_device_status(None) == lib.ATTN_OK

    keep = torch.ones((B, H, N), dtype=torch.bool, device=dev)
    keep[0, h_f, rows_f] = False
    assert torch.equal(o[keep].view(torch.int16), o_ref[keep].view(torch.int16))
    assert torch.equal(lse[keep], lse_ref[keep])

    o2, lse2 = lib.forward_mxfp8(q8, k8, v8, qs, ks, vs, causal=causal)
    torch.cuda.synchronize()
    assert lib.attn_get_device_status(None) == lib.ATTN_OK
    assert torch.equal(o2.view(torch.int16), o_ref.view(torch.int16)) and torch.equal(lse2, lse_ref)


def test_mxfp8_inject_timeout_validates_arguments(cuda_lib):
    lib = cuda_lib
    f = lib.attn_fwd_mxfp8_inject_timeout
    assert f(16, 16, 16, 16, 16, 16, 16, 16, 1, 1, 128, 128, 0.0, 0, -1, WAIT_LIMIT, None) == lib.ATTN_ERR_INVALID_ARG
    assert f(16, 16, 16, 16, 16, 16, 16, 16, 1, 1, 128, 128, 0.0, 0, 0, 100, None) == lib.ATTN_ERR_INVALID_ARG
    assert f(None, 16, 16, 16, 16, 16, 16, 16, 1, 1, 128, 128, 0.0, 0, 0, WAIT_LIMIT, None) == lib.ATTN_ERR_INVALID_ARG
