"""GPU parity of the MXFP8 path through the C ABI: attn_quantize_mxfp8 against
oracle/mxfp8.py bit for bit, and attn_fwd_mxfp8 against the fp64 attention oracle
run on the oracle's own dequantised values.

Tolerances: inputs without outliers, max |O - O_ref| <= 2e-2 and mean <= 2e-3
(the BF16 path's: the scores leave the block-scaled MMA exact up to fp32
accumulation, V is widened to f16 exactly, P is rounded to f16 and O to bf16);
with magnitude-20 outliers in V, |O| reaches 20 where one bf16 step of the output
is 0.125, so the max bound is the FP8 path's 1e-1. |LSE - LSE_ref| <= 1e-3.
Outputs are NaN-prefilled and fenced by canaries.
"""
import math

import numpy as np
import pytest
import torch

import workloads
from oracle import attention_fp64
from oracle.mxfp8 import mx_dequantize, mx_quantize

pytestmark = pytest.mark.gpu

TOL_MAX, TOL_MEAN, TOL_LSE, TOL_MAX_OUTLIERS = 2e-2, 2e-3, 1e-3, 1e-1
CANARY = 4096
DEV = "cuda:0"


def oracle_quant(x_bf16):
    return mx_quantize(x_bf16.to(torch.float64).numpy())


def gpu_quant(lib, x_bf16):
    codes, sf = lib.quantize_mxfp8(x_bf16.to(DEV))
    torch.cuda.synchronize()
    return codes, sf


def oracle_dequant(x_bf16):
    c, s = oracle_quant(x_bf16)
    return mx_dequantize(c, s)


class Guarded:
    def __init__(self, shape, dtype, fill):
        n = int(np.prod(shape))
        self.raw = torch.full((n + 2 * CANARY,), fill, dtype=dtype, device=DEV)
        self.raw[:CANARY] = 7
        self.raw[-CANARY:] = 7
        self.t = self.raw[CANARY:CANARY + n].view(shape)

    def intact(self):
        return bool((self.raw[:CANARY] == 7).all()) and bool((self.raw[-CANARY:] == 7).all())


def run_mx(lib, q, k, v, causal, scale=None):
    """GPU quantisation of q, k, v, then attn_fwd_mxfp8 into guarded outputs."""
    B, H, N, d = q.shape
    (q8, qs), (k8, ks), (v8, vs) = (gpu_quant(lib, x) for x in (q, k, v))
    o = Guarded((B, H, N, d), torch.bfloat16, float("nan"))
    lse = Guarded((B, H, N), torch.float32, float("nan"))
    lib.forward_mxfp8(q8, k8, v8, qs, ks, vs, causal=causal, scale=scale, out=o.t, lse=lse.t)
    torch.cuda.synchronize()
    assert o.intact() and lse.intact(), "write outside the output"
    assert lib.attn_get_device_status(None) == lib.ATTN_OK
    return o.t.float().cpu().numpy(), lse.t.cpu().numpy()


def reference(q, k, v, scale, causal, rows=None):
    return attention_fp64(oracle_dequant(q), oracle_dequant(k), oracle_dequant(v), scale, causal, rows=rows)


def check(o, lse, o_ref, lse_ref, tol_max=TOL_MAX, tol_mean=TOL_MEAN):
    assert np.isfinite(o).all() and np.isfinite(lse).all()
    err = np.abs(o - o_ref)
    assert err.max() <= tol_max, f"max abs err {err.max()}"
    assert err.mean() <= tol_mean, f"mean abs err {err.mean()}"
    lerr = np.abs(lse - lse_ref).max()
    assert lerr <= TOL_LSE, f"LSE err {lerr}"


# ---------------------------------------------------------------- quantisation
QSHAPES = [(1, 1, 1, 32), (1, 2, 77, 128), (2, 3, 130, 64), (1, 1, 1000, 96), (2, 2, 513, 128)]


@pytest.mark.parametrize("shape", QSHAPES, ids=lambda s: "x".join(map(str, s)))
def test_mx_quantize_bitexact(cuda_lib, shape):
    B, H, N, d = shape
    x, _, _ = workloads.make_qkv(B, H, N, d, seed=sum(shape), outliers=("q",))
    codes, sf = gpu_quant(cuda_lib, x)
    c_ref, s_ref = oracle_quant(x)
    assert sf.shape == (B, H, N, d // 32)
    assert np.array_equal(sf.cpu().numpy(), s_ref)
    assert np.array_equal(codes.cpu().numpy(), c_ref)


def edge_rows():
    """Rows of 128 values, one 32-value block per case:
    zero / negative-zero blocks, the bf16 extremes, bf16 subnormals, block
    maxima on exact powers of two, values on E4M3 rounding ties and values that
    saturate at 448 after scaling."""
    rng = np.random.default_rng(11)
    blocks = []
    blocks.append(np.zeros(32))
    blocks.append(-np.zeros(32))
    blocks.append(np.full(32, 3.3895313892515355e38) * np.where(rng.random(32) < 0.5, -1, 1))   # bf16 max
    blocks.append(rng.standard_normal(32) * 1e-39)                                             # bf16 subnormals
    blocks.append(np.array([9.183549615799121e-41] * 32))                                      # smallest bf16 subnormal
    b = rng.standard_normal(32)
    b[0] = 4.0
    blocks.append(b)                                                                           # max exactly 2^2
    # ties: block max 256 (E = 0), values halfway between E4M3 neighbours
    t = np.array([256.0, 1.0625, 1.1875, -2.125, 2.375, 17.0, 19.0, 0.001953125 * 1.5,
                  0.001953125 * 0.5, 0.001953125 * 2.5, 104.0, 120.0, 232.0, 248.0, 464.0 / 2, 3.0] * 2)
    blocks.append(t)
    s = rng.standard_normal(32)
    s[3] = 1.96875 * 2.0 ** 5                                                                  # scaled: 504 -> 448
    s[4] = -1.9 * 2.0 ** 5
    blocks.append(s)
    blocks.append(rng.standard_normal(32) * 2.0 ** -130)
    blocks.append(rng.standard_normal(32) * 2.0 ** 120)
    blocks.append(np.concatenate([[1e30], rng.standard_normal(31) * 1e-10]))                   # far below the max
    blocks.append(rng.standard_normal(32))
    x = np.concatenate(blocks).reshape(-1, 128)
    return torch.from_numpy(x).to(torch.bfloat16).view(1, 1, -1, 128).contiguous()


def test_mx_quantize_edge_blocks(cuda_lib):
    x = edge_rows()
    codes, sf = gpu_quant(cuda_lib, x)
    c_ref, s_ref = oracle_quant(x)
    assert np.array_equal(sf.cpu().numpy(), s_ref)
    assert np.array_equal(codes.cpu().numpy(), c_ref)


def test_mx_quantize_writes_nothing_past_the_end(cuda_lib):
    B, H, N, d = 1, 1, 37, 96                 # 111 blocks: no multiple of the 8 blocks of a warp
    x, _, _ = workloads.make_qkv(B, H, N, d, seed=4)
    xd = x.to(DEV)
    codes = Guarded((B, H, N, d), torch.uint8, 0xAB)
    sf = Guarded((B, H, N, d // 32), torch.uint8, 0xAB)
    st = cuda_lib.attn_quantize_mxfp8(xd.data_ptr(), codes.t.data_ptr(), sf.t.data_ptr(), B, H, N, d,
                                      torch.cuda.current_stream().cuda_stream)
    assert st == cuda_lib.ATTN_OK
    torch.cuda.synchronize()
    assert codes.intact() and sf.intact()
    c_ref, s_ref = oracle_quant(x)
    assert np.array_equal(codes.t.cpu().numpy(), c_ref) and np.array_equal(sf.t.cpu().numpy(), s_ref)


# ---------------------------------------------------------------- attention
SMALL = [(1, 1, 1, 128), (1, 2, 17, 128), (2, 1, 127, 128), (1, 1, 129, 128), (1, 3, 255, 128),
         (2, 2, 256, 128), (1, 2, 300, 128), (1, 1, 640, 128), (1, 2, 1000, 128), (3, 5, 300, 128)]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("causal", [False, True])
def test_mx_small_parity(cuda_lib, shape, causal):
    B, H, N, d = shape
    q, k, v = workloads.make_qkv(B, H, N, d, seed=hash(shape) % 100000 + 7 * causal)
    o, lse = run_mx(cuda_lib, q, k, v, causal)
    o_ref, l_ref = reference(q, k, v, 1 / math.sqrt(d), causal)
    check(o, lse, o_ref, l_ref)


def test_mx_outliers_and_custom_scale(cuda_lib):
    q, k, v = workloads.make_qkv(1, 2, 700, 128, seed=21, outliers=("q", "k", "v"))
    for scale, causal in ((0.02, False), (0.2, True)):
        o, lse = run_mx(cuda_lib, q, k, v, causal, scale=scale)
        o_ref, l_ref = reference(q, k, v, scale, causal)
        check(o, lse, o_ref, l_ref, tol_max=TOL_MAX_OUTLIERS)


def test_mx_block_scale_spread(cuda_lib):
    """Q, K and V whose 32-column blocks differ by many binades: the scores take
    every block's scale inside the MMA and each V column block is widened relative
    to its own largest scale, so every column block keeps its relative accuracy."""
    B, H, N, d = 1, 2, 384, 128
    q, k, v = workloads.make_qkv(B, H, N, d, seed=33)
    qf, kf, vf = q.float(), k.float(), v.float()
    qf[..., 0:32] *= 2.0 ** -6
    kf[..., 32:64] *= 2.0 ** 5
    kf[..., 96:128] *= 2.0 ** -9
    colscale = [2.0 ** -40, 1.0, 2.0 ** 30, 2.0 ** -100]
    for b, c in enumerate(colscale):
        vf[..., 32 * b:32 * b + 32] *= c
    vf[:, :, 200:, 0:32] *= 2.0 ** 12           # one column block with rows 12 binades apart
    q, k, v = (x.to(torch.bfloat16) for x in (qf, kf, vf))
    for causal in (False, True):
        o, lse = run_mx(cuda_lib, q, k, v, causal)
        o_ref, l_ref = reference(q, k, v, 1 / math.sqrt(d), causal)
        assert np.abs(lse - l_ref).max() <= TOL_LSE
        for b in range(4):
            ob, rb = o[..., 32 * b:32 * b + 32], o_ref[..., 32 * b:32 * b + 32]
            mag = np.abs(rb).max()
            assert mag > 0
            rel = np.abs(ob - rb).max() / mag
            assert rel <= 1e-2, (b, rel)


def test_mx_zero_tensors(cuda_lib):
    """All-zero Q (uniform weights: O = mean of the visible V rows) and all-zero V."""
    B, H, N, d = 1, 1, 260, 128
    q, k, v = workloads.make_qkv(B, H, N, d, seed=44)
    zq = torch.zeros_like(q)
    for causal in (False, True):
        o, lse = run_mx(cuda_lib, zq, k, v, causal)
        o_ref, l_ref = reference(zq, k, v, 1 / math.sqrt(d), causal)
        check(o, lse, o_ref, l_ref)
        o, lse = run_mx(cuda_lib, q, k, torch.zeros_like(v), causal)
        assert np.all(o == 0.0)


def test_mx_deterministic(cuda_lib):
    q, k, v = workloads.make_qkv(2, 3, 700, 128, seed=9)
    (q8, qs), (k8, ks), (v8, vs) = (gpu_quant(cuda_lib, x) for x in (q, k, v))
    outs = [cuda_lib.forward_mxfp8(q8, k8, v8, qs, ks, vs, causal=True) for _ in range(4)]
    torch.cuda.synchronize()
    for o, l in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0][0].view(torch.int16))
        assert torch.equal(l.view(torch.int32), outs[0][1].view(torch.int32))


def test_mx_workload_parity(cuda_lib):
    """The MXFP8 workload at full size in the benchmark's launch configuration:
    codes and scales of every tensor bit for bit; O and LSE on sampled rows of
    sampled heads against the oracle on the dequantised values."""
    w = workloads.WORKLOADS["mxfp8_8k"]
    x = workloads.make_workload(w)
    q8, qs = cuda_lib.quantize_mxfp8(x["q"].to(DEV))
    k8, ks = cuda_lib.quantize_mxfp8(x["k"].to(DEV))
    v8, vs = cuda_lib.quantize_mxfp8(x["v"].to(DEV))
    o, lse = cuda_lib.forward_mxfp8(q8, k8, v8, qs, ks, vs, causal=w.causal)
    torch.cuda.synchronize()
    assert cuda_lib.attn_get_device_status(None) == cuda_lib.ATTN_OK
    heads = list(range(0, w.B * w.H, 7))
    rows = workloads.sample_rows(w.N, 96, w.seed)
    BH = w.B * w.H
    deq = {}
    for name, (c8, sb) in (("q", (q8, qs)), ("k", (k8, ks)), ("v", (v8, vs))):
        c_ref, s_ref = oracle_quant(x[name])
        assert np.array_equal(sb.cpu().numpy(), s_ref), name
        assert np.array_equal(c8.cpu().numpy(), c_ref), name
        deq[name] = mx_dequantize(c_ref, s_ref).reshape(BH, w.N, w.d)
    o_gpu = o.float().cpu().numpy().reshape(BH, w.N, w.d)
    l_gpu = lse.cpu().numpy().reshape(BH, w.N)
    errs, lerr = [], 0.0
    for h in heads:
        o_ref, l_ref = attention_fp64(deq["q"][h:h + 1], deq["k"][h:h + 1], deq["v"][h:h + 1], w.scale, w.causal,
                                      rows=rows)
        errs.append(np.abs(o_gpu[h, rows] - o_ref[0]).ravel())
        lerr = max(lerr, float(np.abs(l_gpu[h, rows] - l_ref[0]).max()))
    e = np.concatenate(errs)
    assert e.max() <= TOL_MAX_OUTLIERS, e.max()
    assert e.mean() <= TOL_MEAN, e.mean()
    assert lerr <= TOL_LSE, lerr


def test_mx_every_code_through_pv_exact(cuda_lib):
    """One key per head: P = 1, so O is V itself. V holds every finite E4M3 code
    (0x7F / 0xFF are the format's NaNs, never written by the quantiser) under
    several block scales, and O must equal the oracle's dequantised V bit for bit
    (every such value is a bf16 value): the on-chip widening of V is exact."""
    from oracle.fp8 import e4m3_decode
    B, H, N, d = 1, 2, 1, 128
    codes = np.arange(256, dtype=np.uint8)
    codes[codes == 0x7F] = 0x00
    codes[codes == 0xFF] = 0x80
    v8 = torch.from_numpy(codes.reshape(B, H, N, d).copy())
    sfv = torch.tensor([127, 120, 133, 127, 100, 127, 140, 127], dtype=torch.uint8).view(B, H, N, d // 32)
    q8 = torch.zeros((B, H, N, d), dtype=torch.uint8)
    sfq = torch.full((B, H, N, d // 32), 127, dtype=torch.uint8)
    o, lse = cuda_lib.forward_mxfp8(*(t.to(DEV) for t in (q8, q8, v8, sfq, sfq, sfv)))
    torch.cuda.synchronize()
    assert cuda_lib.attn_get_device_status(None) == cuda_lib.ATTN_OK
    ref = mx_dequantize(v8.numpy(), sfv.numpy())
    assert np.array_equal(ref, torch.from_numpy(ref).to(torch.bfloat16).double().numpy())   # bf16 values
    assert np.array_equal(o.double().cpu().numpy(), ref)
    assert np.all(lse.cpu().numpy() == 0.0)
    assert e4m3_decode(np.array([0x7E], dtype=np.uint8))[0] == 448.0


def test_mx_long_causal_sampled(cuda_lib):
    """A long causal launch (N = 16384: units of 1 to 128 key blocks, heaviest
    first) on sampled rows, including the first and last rows of Q tiles."""
    B, H, N, d = 1, 2, 16384, 128
    q, k, v = workloads.make_qkv(B, H, N, d, seed=55, outliers=("q", "k"))
    (q8, qs), (k8, ks), (v8, vs) = (gpu_quant(cuda_lib, x) for x in (q, k, v))
    o, lse = cuda_lib.forward_mxfp8(q8, k8, v8, qs, ks, vs, causal=True)
    torch.cuda.synchronize()
    assert cuda_lib.attn_get_device_status(None) == cuda_lib.ATTN_OK
    rows = sorted(set([0, 1, 127, 128, 4095, 8191, 8192, 16383] + workloads.sample_rows(N, 40, 9)))
    o_ref, l_ref = reference(q, k, v, 1 / math.sqrt(d), True, rows=rows)
    o_g = o.float().cpu().numpy()[:, :, rows]
    l_g = lse.cpu().numpy()[:, :, rows]
    err = np.abs(o_g - o_ref)
    assert err.max() <= TOL_MAX, err.max()
    assert err.mean() <= TOL_MEAN, err.mean()
    assert np.abs(l_g - l_ref).max() <= TOL_LSE
