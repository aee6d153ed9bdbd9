"""GPU parity of the backward pass (attn_bwd through the C ABI) against the fp64 oracle.

The gradients have no tolerance of their own in the method's statement (it gives
one for the forward only), so it is derived from the arithmetic: each gradient
is a sum of products in which one factor (P, or dS) is rounded to bf16
(relative 2^-9), D_i is formed from the bf16 O (2^-9), and the result is
rounded to bf16 once more (2^-9): a few times 2^-9, about 0.5 %, relative to
the tensor's scale. The tests allow, per tensor, a largest element error of 2 %
of the tensor's largest magnitude and a Frobenius-norm error of 1 %.
A gradient that is exactly zero in the oracle gets an absolute floor of 1e-5
(fp32 rounding of dP - D). Outputs are NaN-prefilled and fenced by canaries.
"""
import math

import numpy as np
import pytest
import torch

import workloads
from oracle import attention_bwd_fp64, attention_fp64

pytestmark = pytest.mark.gpu

TOL_MAX_REL, TOL_FRO = 2e-2, 1e-2
CANARY = 2048


def f64(t):
    return t.to(torch.float64).cpu().numpy()


def make_dout(B, H, N, d, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn((B, H, N, d), generator=g).to(torch.bfloat16)


class Guarded:
    def __init__(self, shape, dev):
        n = int(np.prod(shape))
        self.raw = torch.full((n + 2 * CANARY,), float("nan"), dtype=torch.bfloat16, device=dev)
        self.raw[:CANARY] = 3.0
        self.raw[-CANARY:] = 3.0
        self.t = self.raw[CANARY:CANARY + n].view(shape)

    def intact(self):
        return bool((self.raw[:CANARY] == 3.0).all()) and bool((self.raw[-CANARY:] == 3.0).all())


def run_bwd(lib, q, k, v, dout, causal, scale=None):
    dev = torch.device("cuda:0")
    B, H, N, d = q.shape
    qd, kd, vd, dod = (x.to(dev) for x in (q, k, v, dout))
    o, lse = lib.forward(qd, kd, vd, causal=causal, scale=scale)
    g = [Guarded((B, H, N, d), dev) for _ in range(3)]
    lib.backward(qd, kd, vd, o, lse, dod, causal=causal, scale=scale, dq=g[0].t, dk=g[1].t, dv=g[2].t)
    torch.cuda.synchronize()
    assert all(x.intact() for x in g), "write outside a gradient"
    assert lib.attn_get_device_status(None) == lib.ATTN_OK
    return [x.t.float().cpu().numpy() for x in g]


# a gradient that is exactly zero (one key, causal row 0) comes out as fp32
# rounding noise: dS = P (dP - D) with dP and D two fp32 sums of the same
# products in different orders; the floor covers that (inputs are O(1))
ABS_FLOOR = 1e-5


def check(got, want, name):
    assert np.isfinite(got).all(), f"{name}: NaN/inf (unwritten element?)"
    scale = np.abs(want).max()
    err = np.abs(got - want)
    assert err.max() <= TOL_MAX_REL * scale + ABS_FLOOR, f"{name}: max err {err.max()} vs scale {scale}"
    fro = np.linalg.norm(got - want)
    assert fro <= TOL_FRO * np.linalg.norm(want) + ABS_FLOOR * np.sqrt(want.size), \
        f"{name}: Frobenius error {fro} vs norm {np.linalg.norm(want)}"


SHAPES = [(1, 1, 128, 128), (1, 2, 200, 128), (2, 1, 257, 64), (1, 1, 1, 128), (1, 3, 383, 64),
          (1, 1, 17, 128), (2, 2, 512, 128), (1, 1, 640, 64)]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_small_parity(cuda_lib, shape, causal):
    B, H, N, d = shape
    q, k, v = workloads.make_qkv(B, H, N, d, seed=N * 7 + d + causal)
    dout = make_dout(B, H, N, d, seed=N + 3)
    dq, dk, dv = run_bwd(cuda_lib, q, k, v, dout, causal)
    rq, rk, rv = attention_bwd_fp64(f64(q), f64(k), f64(v), f64(dout), 1 / math.sqrt(d), causal)
    check(dq, rq, "dq")
    check(dk, rk, "dk")
    check(dv, rv, "dv")


def test_bwd_custom_scale_and_outliers(cuda_lib):
    """Magnitude-20 Q/K outliers make rows so peaked that dP - D cancels: the error
    of D taken from a bf16 O (2^-9 of sum |dO||O|) then dominates dS. The method
    takes O as an input, so here both sides get the same O, the oracle's own
    rounded to bf16 (and its LSE), and the oracle forms D from it as well."""
    dev = torch.device("cuda:0")
    B, H, N, d = 1, 2, 300, 128
    q, k, v = workloads.make_qkv(B, H, N, d, seed=91, outliers=("q", "k"))
    dout = make_dout(B, H, N, d, seed=5)
    for scale, causal in ((0.03, False), (0.2, True)):
        o_ref, l_ref = attention_fp64(f64(q), f64(k), f64(v), scale, causal)
        o_in = torch.from_numpy(o_ref).to(torch.bfloat16)
        l_in = torch.from_numpy(l_ref).to(torch.float32)
        g = [Guarded((B, H, N, d), dev) for _ in range(3)]
        cuda_lib.backward(*(x.to(dev) for x in (q, k, v, o_in)), l_in.to(dev), dout.to(dev), causal=causal,
                          scale=scale, dq=g[0].t, dk=g[1].t, dv=g[2].t)
        torch.cuda.synchronize()
        assert all(x.intact() for x in g)
        assert cuda_lib.attn_get_device_status(None) == cuda_lib.ATTN_OK
        rq, rk, rv = attention_bwd_fp64(f64(q), f64(k), f64(v), f64(dout), scale, causal, o=f64(o_in))
        check(g[0].t.float().cpu().numpy(), rq, "dq")
        check(g[1].t.float().cpu().numpy(), rk, "dk")
        check(g[2].t.float().cpu().numpy(), rv, "dv")


def test_bwd_closed_forms(cuda_lib):
    """Identical keys give dQ = 0; causal row 0 gives dQ_0 = 0; with one key
    (N = 1) dQ = dK = 0 and dV = dO."""
    B, H, N, d = 1, 1, 256, 128
    q, _, v = workloads.make_qkv(B, H, N, d, seed=12)
    k = torch.randn(d).to(torch.bfloat16).expand(B, H, N, d).contiguous()
    dout = make_dout(B, H, N, d, seed=13)
    for causal in (False, True):
        dq, dk, dv = run_bwd(cuda_lib, q, k, v, dout, causal)
        rv = attention_bwd_fp64(f64(q), f64(k), f64(v), f64(dout), 1 / math.sqrt(d), causal)[2]
        assert np.abs(dq).max() <= 1e-2 * np.abs(rv).max()
        check(dv, rv, "dv")
    q1, k1, v1 = workloads.make_qkv(1, 2, 1, 128, seed=1)
    do1 = make_dout(1, 2, 1, 128, seed=2)
    dq, dk, dv = run_bwd(cuda_lib, q1, k1, v1, do1, False)
    # dS = P (dP - D) with dP and D two fp32 sums of the same products in
    # different orders: zero up to fp32 rounding
    assert np.abs(dq).max() <= 1e-3 and np.abs(dk).max() <= 1e-3
    np.testing.assert_array_equal(dv, do1.float().numpy())


def test_bwd_deterministic(cuda_lib):
    dev = torch.device("cuda:0")
    q, k, v = (x.to(dev) for x in workloads.make_qkv(2, 2, 700, 128, seed=4))
    dout = make_dout(2, 2, 700, 128, seed=6).to(dev)
    o, lse = cuda_lib.forward(q, k, v, causal=True)
    outs = [cuda_lib.backward(q, k, v, o, lse, dout, causal=True) for _ in range(5)]
    torch.cuda.synchronize()
    for res in outs[1:]:
        for a, b in zip(res, outs[0]):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("name", ["llm_train_causal", "vit_b16_batch"])
def test_bwd_workload_parity(cuda_lib, name):
    """The workload at full size in the launch configuration the benchmark times;
    the oracle recomputes a sample of heads in full."""
    w = workloads.WORKLOADS[name]
    x = workloads.make_workload(w)
    dev = torch.device("cuda:0")
    qd, kd, vd = (x[n].to(dev) for n in ("q", "k", "v"))
    dout = make_dout(w.B, w.H, w.N, w.d, seed=w.seed + 1)
    dod = dout.to(dev)
    o, lse = cuda_lib.forward(qd, kd, vd, causal=w.causal)
    dq, dk, dv = cuda_lib.backward(qd, kd, vd, o, lse, dod, causal=w.causal)
    torch.cuda.synchronize()
    assert cuda_lib.attn_get_device_status(None) == cuda_lib.ATTN_OK
    for t in (dq, dk, dv):
        assert bool(torch.isfinite(t.float()).all())
    BH = w.B * w.H
    heads = sorted({0, 1, BH // 2, BH - 1})
    resh = lambda t: t.reshape(BH, w.N, w.d)  # noqa: E731
    for h in heads:
        sl = lambda t: f64(resh(t)[h:h + 1])  # noqa: E731
        rq, rk, rv = attention_bwd_fp64(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(dout), w.scale, w.causal)
        check(resh(dq)[h:h + 1].float().cpu().numpy(), rq, f"dq head {h}")
        check(resh(dk)[h:h + 1].float().cpu().numpy(), rk, f"dk head {h}")
        check(resh(dv)[h:h + 1].float().cpu().numpy(), rv, f"dv head {h}")
