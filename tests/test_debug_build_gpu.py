"""The debug build (libattn_b200_debug.so, -DATTN_DEBUG) on the GPU.

1. With no failing check it computes exactly what the release build computes:
   every entry point (BF16 forward on both schedules and both head widths, FP8
   and MXFP8 quantisation and forward, backward, W4A16 GEMM) gives bit-identical
   outputs, and the status word and the failure record stay clear.
2. A check that fails is recorded and its access skipped, without a fault: the
   testing hook attn_fwd_debug_row_limit tells the forward kernels that O / LSE
   hold fewer rows than the caller's buffers do, so the stores past the limit
   are rejected while every address stays inside the buffers. The host then
   reads ATTN_ERR_BOUNDS and the site and index of a rejected row; rows below
   the limit are exact, rows past it keep their NaN fill, and the next ordinary
   call on the same context is exact with a clear status.
"""
import pytest
import torch

import workloads
from exact_attention_forward_11_b200 import build as lib_build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def libs(cuda_lib):
    """(release outputs runner, debug outputs runner): the binding switched to
    the debug build inside `debug()`, back to the release build afterwards."""
    lib_build.build(debug=True)
    return cuda_lib


class _Debug:
    def __init__(self, lib):
        self.lib = lib

    def __enter__(self):
        self.prev = self.lib.use_library(self.lib.DEBUG_LIB_PATH)
        assert self.lib.attn_debug_build() == 1
        return self.lib

    def __exit__(self, *exc):
        self.lib.use_library(self.prev)
        return False


def _clear(lib):
    assert lib.attn_get_device_status(None) == lib.ATTN_OK
    assert lib.attn_debug_last_failure(None) == (0, 0)


def _both(lib, fn):
    """fn(lib) -> tuple of tensors, run on the release build and on the debug build."""
    assert lib.attn_debug_build() == 0
    rel = [t.clone() for t in fn(lib)]
    torch.cuda.synchronize()
    assert lib.attn_get_device_status(None) == lib.ATTN_OK
    with _Debug(lib) as dbg:
        _clear(dbg)
        deb = [t.clone() for t in fn(dbg)]
        torch.cuda.synchronize()
        _clear(dbg)
    return rel, deb


def _same(rel, deb):
    for a, b in zip(rel, deb):
        assert a.dtype == b.dtype and a.shape == b.shape
        assert torch.equal(a.view(torch.uint8) if a.dtype.is_floating_point else a,
                           b.view(torch.uint8) if b.dtype.is_floating_point else b)


FWD_CASES = [  # (B, H, N, d, causal): one-Q-tile and two-Q-tile schedules, both head widths
    (1, 3, 1000, 128, True),
    (2, 5, 300, 64, False),
    (2, 16, 2048, 128, True),
    (64, 12, 196, 64, False),
]


@pytest.mark.parametrize("B,H,N,d,causal", FWD_CASES)
def test_debug_forward_bit_identical(libs, B, H, N, d, causal):
    dev = torch.device("cuda:0")
    q, k, v = (x.to(dev) for x in workloads.make_qkv(B, H, N, d, seed=B * 1000 + N + d))
    rel, deb = _both(libs, lambda L: L.forward(q, k, v, causal=causal))
    _same(rel, deb)


def test_debug_fp8_and_mxfp8_bit_identical(libs):
    dev = torch.device("cuda:0")
    B, H, N, d = 1, 4, 1000, 128
    q, k, v = (x.to(dev) for x in workloads.make_qkv(B, H, N, d, seed=77))
    _, rot = workloads.make_rotation(d, seed=78)
    rot = rot.to(dev)

    def fp8(L):
        q8, qs = L.quantize_fp8(q, rot)
        k8, ks = L.quantize_fp8(k, rot)
        v8, vs = L.quantize_fp8(v)
        o, lse = L.forward_fp8(q8, k8, v8, qs, ks, vs, causal=True)
        return q8, qs, k8, ks, v8, vs, o, lse

    def mx(L):
        q8, qf = L.quantize_mxfp8(q)
        k8, kf = L.quantize_mxfp8(k)
        v8, vf = L.quantize_mxfp8(v)
        o, lse = L.forward_mxfp8(q8, k8, v8, qf, kf, vf, causal=True)
        return q8, qf, k8, kf, v8, vf, o, lse

    for fn in (fp8, mx):
        rel, deb = _both(libs, fn)
        _same(rel, deb)


@pytest.mark.parametrize("d,causal", [(128, True), (64, False)])
def test_debug_backward_bit_identical(libs, d, causal):
    dev = torch.device("cuda:0")
    B, H, N = 1, 4, 700
    q, k, v = (x.to(dev) for x in workloads.make_qkv(B, H, N, d, seed=91 + d))
    dout = torch.randn((B, H, N, d), generator=torch.Generator().manual_seed(5)).to(torch.bfloat16).to(dev)
    o, lse = libs.forward(q, k, v, causal=causal)
    torch.cuda.synchronize()
    rel, deb = _both(libs, lambda L: L.backward(q, k, v, o, lse, dout, causal=causal))
    _same(rel, deb)


def test_debug_w4a16_bit_identical(libs):
    dev = torch.device("cuda:0")
    x, qw, s, z = (t.to(dev) for t in workloads.make_w4a16(16, 1024, 2048, seed=19))
    rel, deb = _both(libs, lambda L: (L.w4a16_matmul(x, qw, s, z),))
    _same(rel, deb)


# (B, H, N, d, causal, limit): one-Q-tile (site 2) and two-Q-tile (site 1) schedules
LIMIT_CASES = [
    (1, 3, 1000, 128, True, 1234, 2),
    (2, 16, 2048, 64, False, 20000, 1),
]


@pytest.mark.parametrize("B,H,N,d,causal,limit,site", LIMIT_CASES)
def test_debug_check_fires_skips_and_records(libs, B, H, N, d, causal, limit, site):
    dev = torch.device("cuda:0")
    q, k, v = (x.to(dev) for x in workloads.make_qkv(B, H, N, d, seed=N + limit))
    o_ref, lse_ref = libs.forward(q, k, v, causal=causal)
    torch.cuda.synchronize()
    assert libs.attn_get_device_status(None) == libs.ATTN_OK
    rows = B * H * N
    with _Debug(libs) as dbg:
        _clear(dbg)
        o = torch.full((B, H, N, d), float("nan"), dtype=torch.bfloat16, device=dev)
        lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device=dev)
        st = dbg.attn_fwd_debug_row_limit(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                          B, H, N, d, 0.0, int(causal), limit, None)
        assert st == dbg.ATTN_OK
        assert dbg.attn_get_device_status(None) == dbg.ATTN_ERR_BOUNDS
        got_site, index = dbg.attn_debug_last_failure(None)
        assert got_site == site and limit <= index < rows
        assert dbg.attn_debug_last_failure(None) == (0, 0)   # read and cleared
        of, lf = o.view(rows, d), lse.view(rows)
        assert torch.equal(of[:limit].view(torch.uint8), o_ref.view(rows, d)[:limit].view(torch.uint8))
        assert torch.equal(lf[:limit], lse_ref.view(rows)[:limit])
        assert torch.isnan(of[limit:].float()).all() and torch.isnan(lf[limit:]).all()
        # the context is still usable: an ordinary call is exact, the status clear
        o2, lse2 = dbg.forward(q, k, v, causal=causal)
        torch.cuda.synchronize()
        _clear(dbg)
        assert torch.equal(o2.view(torch.uint8), o_ref.view(torch.uint8)) and torch.equal(lse2, lse_ref)


def test_debug_hook_validates_and_release_refuses(libs):
    f = libs.attn_fwd_debug_row_limit
    assert f(16, 16, 16, 16, 16, 1, 1, 128, 128, 0.0, 0, 0, None) == libs.ATTN_ERR_UNSUPPORTED
    with _Debug(libs) as dbg:
        assert dbg.attn_fwd_debug_row_limit(16, 16, 16, 16, 16, 1, 1, 128, 128, 0.0, 0, -1, None) == \
            dbg.ATTN_ERR_INVALID_ARG
        assert dbg.attn_fwd_debug_row_limit(16, 16, 16, 16, 16, 1, 1, 128, 128, 0.0, 0, 129, None) == \
            dbg.ATTN_ERR_INVALID_ARG
