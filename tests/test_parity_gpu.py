"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Tolerances (bf16 inputs, fp32 accumulation): max |O - O_ref| <= 2e-2, mean
|O - O_ref| <= 2e-3, |LSE - LSE_ref| <= 1e-3. FP8 path: max |O - O_ref| <= 1e-1
and |LSE - LSE_ref| <= 1e-3 against the oracle run on the oracle's own
dequantised values; FP8 codes and scales are compared bit for bit.
Outputs are pre-filled with NaN and fenced by canaries, so an unwritten element or
an out-of-bounds write fails the test.
"""
import math

import numpy as np
import pytest
import torch

import workloads
from oracle import attention_fp64, prepare_fp8, dequantize
from fp8_bounds import check_rotated

pytestmark = pytest.mark.gpu

TOL_MAX, TOL_MEAN, TOL_LSE, TOL_FP8 = 2e-2, 2e-3, 1e-3, 1e-1
CANARY = 4096


def f64(t):
    return t.to(torch.float64).numpy()


class Guarded:
    """Device buffer of `shape` with NaN fill and canary words on both sides."""

    def __init__(self, shape, dtype, dev):
        n = int(np.prod(shape))
        self.raw = torch.full((n + 2 * CANARY,), float("nan"), dtype=dtype, device=dev)
        self.raw[:CANARY] = 7.0
        self.raw[-CANARY:] = 7.0
        self.t = self.raw[CANARY:CANARY + n].view(shape)

    def canaries_intact(self):
        return bool((self.raw[:CANARY] == 7.0).all()) and bool((self.raw[-CANARY:] == 7.0).all())


def run_bf16(lib, q, k, v, causal, scale=None):
    dev = torch.device("cuda:0")
    B, H, N, d = q.shape
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    o = Guarded((B, H, N, d), torch.bfloat16, dev)
    lse = Guarded((B, H, N), torch.float32, dev)
    lib.forward(qd, kd, vd, causal=causal, scale=scale, out=o.t, lse=lse.t)
    torch.cuda.synchronize()
    assert o.canaries_intact() and lse.canaries_intact(), "write outside the output"
    assert lib.attn_get_device_status(None) == lib.ATTN_OK
    return o.t.float().cpu().numpy(), lse.t.cpu().numpy()


def check_bf16(o, lse, o_ref, lse_ref, tol_max=TOL_MAX, tol_mean=TOL_MEAN):
    assert np.isfinite(o).all(), "NaN/inf in O (unwritten element?)"
    assert np.isfinite(lse).all(), "NaN/inf in LSE"
    err = np.abs(o - o_ref)
    assert err.max() <= tol_max, f"max abs err {err.max()}"
    assert err.mean() <= tol_mean, f"mean abs err {err.mean()}"
    lerr = np.abs(lse - lse_ref).max()
    assert lerr <= TOL_LSE, f"LSE err {lerr}"


SMALL = [
    # (B, H, N, d)
    (1, 1, 1, 64), (1, 1, 2, 128), (1, 2, 17, 64), (2, 1, 127, 128), (1, 1, 128, 128),
    (1, 2, 129, 64), (1, 1, 196, 64), (1, 3, 255, 128), (2, 2, 256, 128), (1, 1, 257, 128),
    (1, 2, 383, 64), (1, 1, 512, 128), (1, 1, 640, 64), (1, 2, 1000, 128), (3, 5, 300, 64),
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("causal", [False, True])
def test_bf16_small_full_parity(cuda_lib, shape, causal):
    B, H, N, d = shape
    q, k, v = workloads.make_qkv(B, H, N, d, seed=hash(shape) % 100000 + causal)
    o, lse = run_bf16(cuda_lib, q, k, v, causal)
    o_ref, lse_ref = attention_fp64(f64(q), f64(k), f64(v), 1 / math.sqrt(d), causal)
    check_bf16(o, lse, o_ref, lse_ref)


def test_bf16_custom_scale_and_outliers(cuda_lib):
    q, k, v = workloads.make_qkv(1, 2, 384, 128, seed=77, outliers=("q", "k"))
    for scale, causal in ((0.02, False), (0.3, True)):
        o, lse = run_bf16(cuda_lib, q, k, v, causal, scale=scale)
        o_ref, lse_ref = attention_fp64(f64(q), f64(k), f64(v), scale, causal)
        check_bf16(o, lse, o_ref, lse_ref)


def test_bf16_identical_keys_closed_form(cuda_lib):
    """All keys equal: uniform weights, O_i = mean of the visible V rows."""
    B, H, N, d = 1, 1, 300, 64
    q, _, v = workloads.make_qkv(B, H, N, d, seed=5)
    k = torch.randn(d).to(torch.bfloat16).expand(B, H, N, d).contiguous()
    for causal in (False, True):
        o, lse = run_bf16(cuda_lib, q, k, v, causal)
        vv = f64(v)[0, 0]
        cnt = np.arange(1, N + 1) if causal else np.full(N, N)
        mean = np.cumsum(vv, 0) / cnt[:, None] if causal else np.broadcast_to(vv.mean(0), (N, d))
        assert np.abs(o[0, 0] - mean).max() <= TOL_MAX


def test_bf16_deterministic(cuda_lib):
    q, k, v = workloads.make_qkv(2, 3, 700, 128, seed=9)
    dev = torch.device("cuda:0")
    qd, kd, vd = (x.to(dev) for x in (q, k, v))
    outs = [cuda_lib.forward(qd, kd, vd, causal=True) for _ in range(5)]
    torch.cuda.synchronize()
    for o, l in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0][0].view(torch.int16))
        assert torch.equal(l.view(torch.int32), outs[0][1].view(torch.int32))


def test_bf16_lse_optional(cuda_lib):
    q, k, v = workloads.make_qkv(1, 2, 200, 64, seed=3)
    dev = torch.device("cuda:0")
    o1, _ = cuda_lib.forward(q.to(dev), k.to(dev), v.to(dev), with_lse=False)
    o2, _ = cuda_lib.forward(q.to(dev), k.to(dev), v.to(dev))
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


# ---------------------------------------------------------------- full-size workloads
BF16_WORKLOADS = ["vit_b16_single", "vit_b16_batch", "llm_train_causal", "long_seq_causal", "noncausal_8k_bf16"]


@pytest.mark.parametrize("name", BF16_WORKLOADS)
def test_bf16_workload_parity(cuda_lib, name):
    """Each workload at its full size, in the launch configuration the benchmark
    times; the oracle checks sampled rows of every head (all rows for small N),
    and convexity (min V <= O <= max V over visible keys) holds on every row."""
    w = workloads.WORKLOADS[name]
    x = workloads.make_workload(w)
    dev = torch.device("cuda:0")
    qd, kd, vd = (x[n].to(dev) for n in ("q", "k", "v"))
    o, lse = cuda_lib.forward(qd, kd, vd, causal=w.causal)
    torch.cuda.synchronize()
    assert cuda_lib.attn_get_device_status(None) == cuda_lib.ATTN_OK
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    # convexity on the full output: a causal row sees a prefix, so compare
    # against running extrema (prefix min / max over keys)
    vf = vd.float()
    if w.causal:
        vmin = torch.cummin(vf, dim=2).values
        vmax = torch.cummax(vf, dim=2).values
    else:
        vmin = vf.amin(dim=2, keepdim=True)
        vmax = vf.amax(dim=2, keepdim=True)
    of = o.float()
    slack = 1e-2 + 4e-3 * vf.abs().amax()
    assert bool((of >= vmin - slack).all()) and bool((of <= vmax + slack).all())
    # oracle on sampled rows
    rows = list(range(w.N)) if w.N <= 256 else workloads.sample_rows(w.N, 64 if w.N > 8192 else 128, w.seed)
    heads = range(w.B * w.H)
    if w.B * w.H > 64:
        heads = range(0, w.B * w.H, (w.B * w.H) // 48)
    q64, k64, v64 = (f64(x[n]).reshape(w.B * w.H, w.N, w.d) for n in ("q", "k", "v"))
    o_gpu = o.float().cpu().numpy().reshape(w.B * w.H, w.N, w.d)
    l_gpu = lse.cpu().numpy().reshape(w.B * w.H, w.N)
    errs, lerr = [], 0.0
    for h in heads:
        o_ref, l_ref = attention_fp64(q64[h:h + 1], k64[h:h + 1], v64[h:h + 1], w.scale, w.causal, rows=rows)
        e = np.abs(o_gpu[h, rows] - o_ref[0])
        errs.append(e)
        lerr = max(lerr, float(np.abs(l_gpu[h, rows] - l_ref[0]).max()))
    e = np.concatenate([x.ravel() for x in errs])
    assert e.max() <= TOL_MAX, e.max()
    assert e.mean() <= TOL_MEAN, e.mean()
    assert lerr <= TOL_LSE, lerr


# ---------------------------------------------------------------- FP8
def run_quant(lib, x, rot):
    dev = torch.device("cuda:0")
    x8, sc = lib.quantize_fp8(x.to(dev), None if rot is None else rot.to(dev))
    torch.cuda.synchronize()
    return x8.cpu().numpy(), sc.cpu().numpy()


@pytest.mark.parametrize("N", [1, 100, 128, 300, 1024])
@pytest.mark.parametrize("rotate", [False, True])
def test_fp8_quantize(cuda_lib, N, rotate):
    """Without rotation the codes and scales are unique and compared bit for bit;
    with rotation every code lies in the interval the tensor cores' fp32
    accumulation error allows (tests/fp8_bounds.py) and moved codes are rare."""
    q, _, _ = workloads.make_qkv(2, 3, N, 128, seed=N + 31 * rotate, outliers=("q",))
    rot = workloads.make_rotation(128, 99)[1] if rotate else None
    codes, scales = run_quant(cuda_lib, q, rot)
    if rotate:
        check_rotated(q.reshape(6, N, 128), rot, codes.reshape(6, N, 128), scales.reshape(6, -1))
        return
    codes_ref, scales_ref = prepare_fp8(q, rot)
    np.testing.assert_array_equal(scales, scales_ref)
    np.testing.assert_array_equal(codes, codes_ref)


def test_fp8_quantize_edge_tiles(cuda_lib):
    """All-zero tiles (scale 1, codes 0), a tile whose amax saturates exactly, and
    tails of 1 and 127 rows, with and without rotation; codes past N untouched."""
    dev = torch.device("cuda:0")
    rot = workloads.make_rotation(128, 5)[1]
    for N in (1, 127, 129, 383):
        x, _, _ = workloads.make_qkv(1, 2, N, 128, seed=N)
        x[0, 0, :min(N, 128)] = 0.0                      # head 0, tile 0: all zeros
        x[0, 1, 0, 0] = 448.0 * 1024                     # head 1, tile 0: one large value
        for r in (None, rot):
            xd = x.to(dev)
            T = (N + 127) // 128
            c_out = torch.empty((1, 2, N, 128), dtype=torch.uint8, device=dev)
            s_out = torch.empty((1, 2, T), dtype=torch.float32, device=dev)
            st = cuda_lib.attn_quantize_fp8(xd.data_ptr(), None if r is None else r.to(dev).data_ptr(),
                                            c_out.data_ptr(), s_out.data_ptr(), 1, 2, N, 128, None)
            assert st == cuda_lib.ATTN_OK
            torch.cuda.synchronize()
            codes, scales = c_out.cpu().numpy(), s_out.cpu().numpy()
            # (a rotated zero may come out as -0: only the magnitude is fixed)
            assert scales[0, 0, 0] == 1.0 and not (codes[0, 0, :min(N, 128)] & 0x7F).any()
            if r is None:
                cr, sr = prepare_fp8(x, None)
                np.testing.assert_array_equal(codes, cr)
                np.testing.assert_array_equal(scales, sr)
                assert codes[0, 1, 0, 0] == 0x7E
            else:
                check_rotated(x.reshape(2, N, 128), r, codes.reshape(2, N, 128), scales.reshape(2, -1))
    assert cuda_lib.attn_get_device_status(None) == cuda_lib.ATTN_OK


def test_fp8_quantize_writes_nothing_past_n(cuda_lib):
    """The codes of rows >= N and the scales past ceil(N/128) stay untouched: the
    outputs are views into larger guard-filled buffers (per head, so a tail write
    would land in the next head's rows or the trailing guard)."""
    dev = torch.device("cuda:0")
    rot = workloads.make_rotation(128, 5)[1].to(dev)
    B, H, N = 1, 3, 200
    x, _, _ = workloads.make_qkv(B, H, N, 128, seed=3)
    xd = x.to(dev)
    T = (N + 127) // 128
    for r in (None, rot):
        guard = torch.full((B * H * N * 128 + 4096,), 0xAB, dtype=torch.uint8, device=dev)
        sguard = torch.full((B * H * T + 64,), -1.0, dtype=torch.float32, device=dev)
        st = cuda_lib.attn_quantize_fp8(xd.data_ptr(), None if r is None else r.data_ptr(), guard.data_ptr(),
                                        sguard.data_ptr(), B, H, N, 128, None)
        assert st == cuda_lib.ATTN_OK
        torch.cuda.synchronize()
        assert bool((guard[B * H * N * 128:] == 0xAB).all())
        assert bool((sguard[B * H * T:] == -1.0).all())
        assert bool((sguard[:B * H * T] > 0).all())


def fp8_inputs(lib, q, k, v, rot):
    dev = torch.device("cuda:0")
    rd = rot.to(dev)
    q8, qs = lib.quantize_fp8(q.to(dev), rd)
    k8, ks = lib.quantize_fp8(k.to(dev), rd)
    v8, vs = lib.quantize_fp8(v.to(dev), None)
    return q8, k8, v8, qs, ks, vs


def fp8_reference(q, k, v, rot, scale, causal, rows=None, heads=None):
    """Oracle O, LSE on the oracle's own quantised values (heads sliced first:
    quantisation is per (batch, head) tile, so a slice quantises identically)."""
    B, H, N, d = q.shape
    hs = list(range(B * H)) if heads is None else list(heads)
    sl = [x.reshape(B * H, N, d)[hs].unsqueeze(0) for x in (q, k, v)]
    qc, qs = prepare_fp8(sl[0], rot)
    kc, ks = prepare_fp8(sl[1], rot)
    vc, vs = prepare_fp8(sl[2], None)
    qd, kd, vd = dequantize(qc, qs)[0], dequantize(kc, ks)[0], dequantize(vc, vs)[0]
    o, l = attention_fp64(qd, kd, vd, scale, causal, rows=rows)
    return o, l, (qc[0], qs[0], kc[0], ks[0], vc[0], vs[0])


def run_fp8(lib, q8, k8, v8, qs, ks, vs, causal):
    """attn_fwd_fp8 into NaN-prefilled, canary-fenced O and LSE; the canaries and
    the device status word are checked after the launch."""
    dev = torch.device("cuda:0")
    B, H, N, d = q8.shape
    o = Guarded((B, H, N, d), torch.bfloat16, dev)
    lse = Guarded((B, H, N), torch.float32, dev)
    lib.forward_fp8(q8, k8, v8, qs, ks, vs, causal=causal, out=o.t, lse=lse.t)
    torch.cuda.synchronize()
    assert o.canaries_intact() and lse.canaries_intact(), "write outside the output"
    assert lib.attn_get_device_status(None) == lib.ATTN_OK
    return o.t.float().cpu().numpy(), lse.t.cpu().numpy()


@pytest.mark.parametrize("shape", [(1, 1, 128, 128), (1, 2, 300, 128), (2, 1, 1000, 128), (1, 1, 17, 128),
                                   (1, 1, 1, 128), (2, 3, 257, 128)],
                         ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("causal", [False, True])
def test_fp8_small_parity(cuda_lib, shape, causal):
    B, H, N, d = shape
    q, k, v = workloads.make_qkv(B, H, N, d, seed=N + 5, outliers=("q", "k", "v"))
    rot = workloads.make_rotation(d, 17)[1]
    q8, k8, v8, qs, ks, vs = fp8_inputs(cuda_lib, q, k, v, rot)
    o, lse = run_fp8(cuda_lib, q8, k8, v8, qs, ks, vs, causal)
    o_ref, l_ref, _ = fp8_reference(q, k, v, rot, 1 / math.sqrt(d), causal)
    o = o.reshape(B * H, N, d)
    lse = lse.reshape(B * H, N)
    assert np.isfinite(o).all(), "NaN/inf in O (unwritten element?)"
    assert np.isfinite(lse).all(), "NaN/inf in LSE"
    assert np.abs(o - o_ref).max() <= TOL_FP8
    assert np.abs(lse - l_ref).max() <= TOL_LSE


def test_fp8_every_code_through_pv_exact(cuda_lib):
    """One key per head: P = 1, so O is the dequantised V itself. V holds every
    finite E4M3 code (0x7F / 0xFF are the format's NaNs, never written by the
    quantiser) and O must equal decode(code) * scale bit for bit (every such
    value is a bf16 value): the on-chip widening of V is exact."""
    from oracle.fp8 import e4m3_decode
    dev = torch.device("cuda:0")
    B, H, N, d = 1, 2, 1, 128
    codes = np.arange(256, dtype=np.uint8)
    codes[codes == 0x7F] = 0x00
    codes[codes == 0xFF] = 0x80
    v8 = torch.from_numpy(codes.reshape(B, H, N, d).copy()).to(dev)
    zero8 = torch.zeros((B, H, N, d), dtype=torch.uint8, device=dev)
    one = torch.ones((B, H, 1), dtype=torch.float32, device=dev)
    vs = torch.tensor([1.0, 0.125], dtype=torch.float32, device=dev).view(B, H, 1)
    o, lse = cuda_lib.forward_fp8(zero8, zero8, v8, one, one, vs)
    torch.cuda.synchronize()
    assert cuda_lib.attn_get_device_status(None) == cuda_lib.ATTN_OK
    ref = e4m3_decode(codes).reshape(B, H, N, d) * np.array([1.0, 0.125]).reshape(B, H, 1, 1)
    assert np.array_equal(ref, torch.from_numpy(ref).to(torch.bfloat16).double().numpy())
    assert np.array_equal(o.double().cpu().numpy(), ref)
    assert np.all(lse.cpu().numpy() == 0.0)


def test_fp8_zero_scale_tiles(cuda_lib):
    """Tiles whose scale is 0 dequantise to zeros: a zero V tile contributes
    nothing and a zero K tile gives scores of exactly 0, with no NaN anywhere."""
    B, H, N, d = 1, 2, 384, 128
    q, k, v = workloads.make_qkv(B, H, N, d, seed=404)
    rot = workloads.make_rotation(d, 17)[1]
    q8, k8, v8, qs, ks, vs = fp8_inputs(cuda_lib, q, k, v, rot)
    vs[0, 0, 1] = 0.0            # head 0: V tile 1 is zero
    ks[0, 1, 2] = 0.0            # head 1: K tile 2 is zero
    vs[0, 1, 0] = 0.0            # head 1: V tile 0 is zero too
    for causal in (False, True):
        o, lse = run_fp8(cuda_lib, q8, k8, v8, qs, ks, vs, causal)
        assert np.isfinite(o).all() and np.isfinite(lse).all()
        codes = [x.cpu().numpy() for x in (q8, k8, v8)]
        scs = [x.cpu().numpy() for x in (qs, ks, vs)]
        qd, kd, vd = (dequantize(c, sc) for c, sc in zip(codes, scs))
        o_ref, l_ref = attention_fp64(qd, kd, vd, 1 / math.sqrt(d), causal)
        assert np.abs(o - o_ref).max() <= TOL_FP8
        assert np.abs(lse - l_ref).max() <= TOL_LSE


def test_fp8_deterministic(cuda_lib):
    q, k, v = workloads.make_qkv(2, 3, 700, 128, seed=19, outliers=("q", "k", "v"))
    rot = workloads.make_rotation(128, 17)[1]
    q8, k8, v8, qs, ks, vs = fp8_inputs(cuda_lib, q, k, v, rot)
    for causal in (False, True):
        outs = [cuda_lib.forward_fp8(q8, k8, v8, qs, ks, vs, causal=causal) for _ in range(5)]
        torch.cuda.synchronize()
        for o, l in outs[1:]:
            assert torch.equal(o.view(torch.int16), outs[0][0].view(torch.int16))
            assert torch.equal(l.view(torch.int32), outs[0][1].view(torch.int32))
    # the preparation kernel is deterministic as well
    again = fp8_inputs(cuda_lib, q, k, v, rot)
    torch.cuda.synchronize()
    for a, b in zip((q8, k8, v8, qs, ks, vs), again):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))


def test_fp8_workload_parity(cuda_lib):
    w = workloads.WORKLOADS["fp8_rotated"]
    x = workloads.make_workload(w)
    q8, k8, v8, qs, ks, vs = fp8_inputs(cuda_lib, x["q"], x["k"], x["v"], x["rot"])
    o, lse = cuda_lib.forward_fp8(q8, k8, v8, qs, ks, vs, causal=w.causal)
    torch.cuda.synchronize()
    assert cuda_lib.attn_get_device_status(None) == cuda_lib.ATTN_OK
    assert bool(torch.isfinite(o.float()).all()) and bool(torch.isfinite(lse).all())
    heads = list(range(0, w.B * w.H, 8))
    rows = workloads.sample_rows(w.N, 96, w.seed)
    o_ref, l_ref, ref_codes = fp8_reference(x["q"], x["k"], x["v"], x["rot"], w.scale, w.causal, rows=rows,
                                            heads=heads)
    # the preparation step at full size on those heads: V (no rotation) bit-exact,
    # Q and K within the intervals the rotation's fp32 accumulation allows
    def sel(t):
        g = t.cpu().numpy()
        return g.reshape((w.B * w.H,) + g.shape[2:])[heads]
    np.testing.assert_array_equal(sel(v8), ref_codes[4])
    np.testing.assert_array_equal(sel(vs), ref_codes[5])
    for x8, xs, name in ((q8, qs, "q"), (k8, ks, "k")):
        xh = x[name].reshape(w.B * w.H, w.N, w.d)[heads]
        check_rotated(xh, x["rot"], sel(x8), sel(xs))
    o = o.float().cpu().numpy().reshape(w.B * w.H, w.N, w.d)[heads][:, rows]
    lse = lse.cpu().numpy().reshape(w.B * w.H, w.N)[heads][:, rows]
    assert np.abs(o - o_ref).max() <= TOL_FP8
    assert np.abs(lse - l_ref).max() <= TOL_LSE


def test_one_tile_and_two_tile_schedules_agree(cuda_lib):
    """attn_fwd runs launches with fewer two-Q-tile units than SMs on the one-Q-tile
    schedule (attn_fwd1_kernel.cuh); the testing hook attn_fwd_inject_timeout with
    no tile withheld runs any shape on the two-tile schedule (attn_fwd_kernel.cuh).
    Both take every row through the same operations in the same order, so O and LSE
    agree bit for bit, and a head-sharded run gives the same bytes whichever
    schedule each shard's size selects."""
    dev = torch.device("cuda:0")
    # (the hook takes d = 128 only)
    for (B, H, N, d, causal) in [(2, 3, 300, 128, False), (2, 3, 300, 128, True), (1, 4, 257, 128, True),
                                 (1, 2, 1000, 128, False), (1, 1, 129, 128, False)]:
        q, k, v = (x.to(dev) for x in workloads.make_qkv(B, H, N, d, seed=N + d))
        o1, l1 = cuda_lib.forward(q, k, v, causal=causal)
        o2 = torch.empty_like(o1)
        l2 = torch.empty_like(l1)
        st = cuda_lib.attn_fwd_inject_timeout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o2.data_ptr(), l2.data_ptr(),
                                              B, H, N, d, 0.0, int(causal), 1 << 30, 1 << 31, None)
        assert st == cuda_lib.ATTN_OK
        torch.cuda.synchronize()
        assert cuda_lib.attn_get_device_status(None) == cuda_lib.ATTN_OK
        assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)), (B, H, N, d, causal)
        assert torch.equal(l1.view(torch.int32), l2.view(torch.int32)), (B, H, N, d, causal)


def test_forward_from_host_matches_forward(cuda_lib):
    """The host-to-host entry (inputs copied in and outputs copied out by head
    groups on three streams) returns the same bytes as forward() on device
    copies, for any number of groups (including more groups than heads) and for
    N that is not a multiple of 4 (per-group LSE buffers)."""
    dev = torch.device("cuda:0")
    for (B, H, N, d, causal), chunks in [((2, 3, 300, 128, True), 4), ((1, 5, 257, 64, False), 1),
                                          ((1, 2, 129, 128, False), 7), ((3, 4, 1000, 128, True), 3)]:
        q, k, v = (x.pin_memory() for x in workloads.make_qkv(B, H, N, d, seed=N + 3 * d))
        o_h, l_h = cuda_lib.forward_from_host(q, k, v, causal=causal, chunks=chunks)
        o_d, l_d = cuda_lib.forward(q.to(dev), k.to(dev), v.to(dev), causal=causal)
        torch.cuda.synchronize()
        assert torch.equal(o_h.view(torch.int16), o_d.cpu().view(torch.int16)), (B, H, N, d, causal, chunks)
        assert torch.equal(l_h.view(torch.int32), l_d.cpu().view(torch.int32)), (B, H, N, d, causal, chunks)
