"""A seeded sweep of random shapes through every forward entry point, the backward
and the W4A16 GEMM, against the fp64 oracle.

The fixed shape lists of the other parity tests pick the edge cases by hand. This
sweep draws B, H, N (1 .. 700) and the head width at random from a fixed seed,
causal or not, so ragged last blocks, odd tile counts and the number of work
units per CTA vary together. It adds launches whose two-Q-tile unit count sits
just below, at and above the SM count, where attn_fwd switches between the
one- and two-tile schedules. Outputs are NaN-prefilled and fenced by canaries;
the device status word must read ATTN_OK after every launch. Tolerances as in the
other parity tests: BF16 and MXFP8 max |O - O_ref| <= 2e-2, mean <= 2e-3, FP8
max <= 1e-1, LSE within 1e-3 (the quantised paths against the oracle run on the
oracle's own dequantised values); the backward and W4A16 bounds are those of their
own tests.
"""
import math

import numpy as np
import pytest
import torch

import workloads
from oracle import attention_fp64, dequantize, prepare_fp8
from oracle.mxfp8 import mx_dequantize, mx_quantize

pytestmark = pytest.mark.gpu

TOL_MAX, TOL_MEAN, TOL_LSE, TOL_FP8 = 2e-2, 2e-3, 1e-3, 1e-1
CANARY = 4096
DEV = "cuda:0"
SMS = 148


def _draw(n_shapes, seed, widths):
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(n_shapes):
        B = int(rng.integers(1, 4))
        H = int(rng.integers(1, 6))
        N = int(rng.integers(1, 701))
        d = int(rng.choice(widths))
        out.append((B, H, N, d, bool(rng.integers(0, 2))))
    return out


BF16_SHAPES = _draw(24, 20261203, (64, 128))
FP8_SHAPES = _draw(8, 20261204, (128,))
MX_SHAPES = _draw(8, 20261205, (128,))
# attn_fwd runs the one-tile schedule when B*H*ceil(N/256) (two-tile units) < SMs:
# 147 units (one-tile), 148 and 149 (two-tile), and with a ragged second tile per
# pair (N = 300) 146 and 148
BOUNDARY = [(1, SMS - 1, 200, 128, False), (1, SMS, 200, 64, True), (1, SMS + 1, 200, 128, True),
            (1, SMS // 2 - 1, 300, 64, False), (1, SMS // 2, 300, 128, True)]


def _ids(s):
    return "x".join(map(str, s[:4])) + ("c" if s[4] else "")


class Guarded:
    """Device buffer of `shape`, NaN-filled, with canary words on both sides."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape))
        self.raw = torch.full((n + 2 * CANARY,), float("nan"), dtype=dtype, device=DEV)
        self.raw[:CANARY] = 7
        self.raw[-CANARY:] = 7
        self.t = self.raw[CANARY:CANARY + n].view(shape)

    def intact(self):
        return bool((self.raw[:CANARY] == 7).all()) and bool((self.raw[-CANARY:] == 7).all())


def _rows(N, rng):
    """Every row for short sequences, else a sample that keeps the ends."""
    if N <= 160:
        return None
    return np.unique(np.concatenate([[0, N - 1], rng.integers(0, N, 40)]))


def _launch(lib, fn, B, H, N, d):
    o, lse = Guarded((B, H, N, d), torch.bfloat16), Guarded((B, H, N), torch.float32)
    fn(o.t, lse.t)
    torch.cuda.synchronize()
    assert o.intact() and lse.intact(), "write outside the output"
    assert lib.attn_get_device_status(None) == lib.ATTN_OK
    o_h, lse_h = o.t.float().cpu().numpy(), lse.t.cpu().numpy()
    assert np.isfinite(o_h).all(), "NaN/inf in O (unwritten element?)"
    assert np.isfinite(lse_h).all(), "NaN/inf in LSE"
    return o_h, lse_h


def _check(o, lse, o_ref, lse_ref, rows, tol_max, tol_mean):
    if rows is not None:
        o, lse = o[:, :, rows], lse[:, :, rows]
    err = np.abs(o - o_ref)
    assert err.max() <= tol_max, f"max abs err {err.max()}"
    if tol_mean is not None:
        assert err.mean() <= tol_mean, f"mean abs err {err.mean()}"
    assert np.abs(lse - lse_ref).max() <= TOL_LSE, f"LSE err {np.abs(lse - lse_ref).max()}"


@pytest.mark.parametrize("shape", BF16_SHAPES + BOUNDARY, ids=_ids)
def test_bf16_random_shape(cuda_lib, shape):
    lib = cuda_lib
    B, H, N, d, causal = shape
    q, k, v = workloads.make_qkv(B, H, N, d, seed=(B * 7 + H * 131 + N * 17 + d) % 100003)
    qd, kd, vd = (x.to(DEV) for x in (q, k, v))
    o, lse = _launch(lib, lambda ot, lt: lib.forward(qd, kd, vd, causal=causal, out=ot, lse=lt), B, H, N, d)
    rows = _rows(N, np.random.default_rng(N))
    f64 = [x.to(torch.float64).numpy() for x in (q, k, v)]
    o_ref, lse_ref = attention_fp64(*f64, 1 / math.sqrt(d), causal, rows=rows)
    _check(o, lse, o_ref, lse_ref, rows, TOL_MAX, TOL_MEAN)


@pytest.mark.parametrize("shape", FP8_SHAPES, ids=_ids)
def test_fp8_random_shape(cuda_lib, shape):
    lib = cuda_lib
    B, H, N, d, causal = shape
    q, k, v = workloads.make_qkv(B, H, N, d, seed=N + 11, outliers=("q", "k", "v"))
    rot = workloads.make_rotation(d, 23)[1]
    rd = rot.to(DEV)
    (q8, qs), (k8, ks), (v8, vs) = (lib.quantize_fp8(x.to(DEV), r) for x, r in ((q, rd), (k, rd), (v, None)))
    o, lse = _launch(lib, lambda ot, lt: lib.forward_fp8(q8, k8, v8, qs, ks, vs, causal=causal, out=ot, lse=lt),
                     B, H, N, d)
    rows = _rows(N, np.random.default_rng(N + 1))
    qc, qsc = prepare_fp8(q, rot)
    kc, ksc = prepare_fp8(k, rot)
    vc, vsc = prepare_fp8(v, None)
    o_ref, lse_ref = attention_fp64(dequantize(qc, qsc), dequantize(kc, ksc), dequantize(vc, vsc),
                                    1 / math.sqrt(d), causal, rows=rows)
    _check(o, lse, o_ref, lse_ref, rows, TOL_FP8, None)


@pytest.mark.parametrize("shape", MX_SHAPES, ids=_ids)
def test_mxfp8_random_shape(cuda_lib, shape):
    lib = cuda_lib
    B, H, N, d, causal = shape
    q, k, v = workloads.make_qkv(B, H, N, d, seed=N + 29)
    (q8, qs), (k8, ks), (v8, vs) = (lib.quantize_mxfp8(x.to(DEV)) for x in (q, k, v))
    o, lse = _launch(lib, lambda ot, lt: lib.forward_mxfp8(q8, k8, v8, qs, ks, vs, causal=causal, out=ot, lse=lt),
                     B, H, N, d)
    rows = _rows(N, np.random.default_rng(N + 2))
    deq = [mx_dequantize(*mx_quantize(x.to(torch.float64).numpy())) for x in (q, k, v)]
    o_ref, lse_ref = attention_fp64(*deq, 1 / math.sqrt(d), causal, rows=rows)
    _check(o, lse, o_ref, lse_ref, rows, TOL_MAX, TOL_MEAN)


# ---------------------------------------------------------------- backward and W4A16
BWD_SHAPES = _draw(10, 20261206, (64, 128))


@pytest.mark.parametrize("shape", [(B, H, min(N, 520), d, c) for B, H, N, d, c in BWD_SHAPES], ids=_ids)
def test_bwd_random_shape(cuda_lib, shape):
    """The backward through attn_bwd, with the tolerance the backward tests derive
    (largest element error 2 % of the tensor's largest magnitude, Frobenius 1 %)."""
    from oracle import attention_bwd_fp64
    lib = cuda_lib
    B, H, N, d, causal = shape
    q, k, v = workloads.make_qkv(B, H, N, d, seed=N * 5 + d + 1)
    gen = torch.Generator().manual_seed(N + 17)
    dout = torch.randn((B, H, N, d), generator=gen).to(torch.bfloat16)
    qd, kd, vd, dod = (x.to(DEV) for x in (q, k, v, dout))
    o, lse = lib.forward(qd, kd, vd, causal=causal)
    grads = [Guarded((B, H, N, d), torch.bfloat16) for _ in range(3)]
    lib.backward(qd, kd, vd, o, lse, dod, causal=causal, dq=grads[0].t, dk=grads[1].t, dv=grads[2].t)
    torch.cuda.synchronize()
    assert all(g.intact() for g in grads), "write outside a gradient"
    assert lib.attn_get_device_status(None) == lib.ATTN_OK
    want = attention_bwd_fp64(*(x.to(torch.float64).numpy() for x in (q, k, v, dout)), 1 / math.sqrt(d), causal)
    for g, ref, name in zip(grads, want, ("dq", "dk", "dv")):
        got = g.t.float().cpu().numpy()
        assert np.isfinite(got).all(), f"{name}: NaN/inf (unwritten element?)"
        err = np.abs(got - ref)
        assert err.max() <= 2e-2 * np.abs(ref).max() + 1e-5, f"{name}: max err {err.max()}"
        assert np.linalg.norm(got - ref) <= 1e-2 * np.linalg.norm(ref) + 1e-5 * np.sqrt(ref.size), name


def _draw_gemm(n, seed):
    rng = np.random.default_rng(seed)
    return [(int(rng.integers(1, 129)), 128 * int(rng.integers(1, 9)), 128 * int(rng.integers(1, 7)))
            for _ in range(n)]


@pytest.mark.parametrize("M,K,N", _draw_gemm(8, 20261207))
def test_w4a16_random_shape(cuda_lib, M, K, N):
    """W4A16 GEMM of random M (1 .. 128), K and N (multiples of 128), against the
    fp64 product of the dequantised weights with the W4A16 tests' element bound
    (2^-11 relative plus 2^-16 of the sum of |x||w|: fp16 output rounding and fp32
    accumulation of fp16 products)."""
    from oracle.w4a16 import dequantize_weights, w4a16_gemm_fp64
    lib = cuda_lib
    x, qw, s, z = workloads.make_w4a16(M, N, K, seed=M * 3 + K + N)
    raw = torch.full((M * N + 2 * CANARY,), float("nan"), dtype=torch.float16, device=DEV)
    raw[:CANARY] = 5.0
    raw[-CANARY:] = 5.0
    y = raw[CANARY:CANARY + M * N].view(M, N)
    lib.w4a16_matmul(x.to(DEV), qw.to(DEV), s.to(DEV), z.to(DEV), out=y)
    torch.cuda.synchronize()
    assert bool((raw[:CANARY] == 5.0).all()) and bool((raw[-CANARY:] == 5.0).all()), "write outside Y"
    assert lib.attn_get_device_status(None) == lib.ATTN_OK
    xn, qn, sn, zn = (t.numpy() for t in (x, qw, s, z))
    ref = w4a16_gemm_fp64(xn, qn, sn, zn)
    w = dequantize_weights(qn, sn, zn).astype(np.float64)
    bound = 2.0 ** -11 * np.abs(ref) + 2.0 ** -16 * (np.abs(xn.astype(np.float64)) @ np.abs(w)) + 1e-7
    got = y.float().cpu().numpy()
    assert np.isfinite(got).all(), "NaN/inf in Y (unwritten element?)"
    assert np.all(np.abs(got - ref) <= bound), f"max err {np.abs(got - ref).max()}"
