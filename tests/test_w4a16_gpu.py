"""GPU parity of the W4A16 GEMM (w4a16_gemm through the C ABI) against the oracle.

Tolerance, from the arithmetic: the dequantised weights are exact fp16 values on
both sides (checked bit for bit with one-hot activations); the products are
exact; the kernel sums them in fp32 on the tensor cores and rounds Y to fp16.
So |Y - Y_ref| <= 2^-11 |Y_ref| (the output rounding) + 2^-16 (|X| |W|) (fp32
accumulation over K, with margin) per element. A single wrong weight moves an
element by |x| |dw|, far above that bound at these scales.
"""
import numpy as np
import pytest
import torch

import workloads
from oracle.w4a16 import dequantize_weights, w4a16_gemm_fp64

pytestmark = pytest.mark.gpu
CANARY = 1024


def run(lib, x, qw, s, z):
    dev = torch.device("cuda:0")
    M, N = x.shape[0], qw.shape[1]
    raw = torch.full((M * N + 2 * CANARY,), float("nan"), dtype=torch.float16, device=dev)
    raw[:CANARY] = 5.0
    raw[-CANARY:] = 5.0
    y = raw[CANARY:CANARY + M * N].view(M, N)
    lib.w4a16_matmul(x.to(dev), qw.to(dev), s.to(dev), z.to(dev), out=y)
    torch.cuda.synchronize()
    assert bool((raw[:CANARY] == 5.0).all()) and bool((raw[-CANARY:] == 5.0).all()), "write outside Y"
    assert lib.attn_get_device_status(None) == lib.ATTN_OK
    return y.float().cpu().numpy()


def check(y, x, qw, s, z, cols=None):
    xn, qn, sn, zn = (t.numpy() for t in (x, qw, s, z))
    if cols is not None:
        qn, sn, zn = qn[:, cols], sn[:, cols], zn[:, cols]
        y = y[:, cols]
    ref = w4a16_gemm_fp64(xn, qn, sn, zn)
    w = dequantize_weights(qn, sn, zn).astype(np.float64)
    bound = 2.0 ** -11 * np.abs(ref) + 2.0 ** -16 * (np.abs(xn.astype(np.float64)) @ np.abs(w)) + 1e-7
    assert np.isfinite(y).all(), "NaN/inf in Y (unwritten element?)"
    err = np.abs(y - ref)
    assert np.all(err <= bound), f"max err {err.max()}, worst ratio {(err / bound).max()}"


@pytest.mark.parametrize("M,K,N", [(1, 128, 128), (16, 256, 256), (5, 1024, 384), (128, 512, 128),
                                   (33, 384, 640), (100, 128, 256)])
def test_w4a16_small_parity(cuda_lib, M, K, N):
    x, qw, s, z = workloads.make_w4a16(M, N, K, seed=M + K + N)
    check(run(cuda_lib, x, qw, s, z), x, qw, s, z)


def test_w4a16_dequantisation_bit_exact(cuda_lib):
    """One-hot activations select weight rows: Y equals the dequantised weights
    bit for bit (a single exact product per output, rounded to fp16 losslessly)."""
    K, N = 512, 256
    _, qw, s, z = workloads.make_w4a16(1, N, K, seed=3)
    ks = [0, 1, 2, 3, 4, 5, 6, 7, 8, 15, 127, 128, 129, 200, 255, 256, 383, 384, 500, 511]
    x = torch.zeros((len(ks), K), dtype=torch.float16)
    for m, k in enumerate(ks):
        x[m, k] = 1.0
    y = run(cuda_lib, x, qw, s, z)
    w = dequantize_weights(qw.numpy(), s.numpy(), z.numpy())
    np.testing.assert_array_equal(y, w[ks].astype(np.float32))


def test_w4a16_workload_parity(cuda_lib):
    """The decode workload at full size in the launch the benchmark times; the
    oracle checks 384 sampled columns (three whole CTAs' worth and scattered ones)."""
    wl = workloads.GEMM_WORKLOADS["w4a16_decode_mlp"]
    x, qw, s, z = workloads.make_w4a16(wl.M, wl.N, wl.K, wl.seed)
    y = run(cuda_lib, x, qw, s, z)
    rng = np.random.default_rng(0)
    cols = sorted(set(range(128)) | set(range(wl.N - 128, wl.N)) | set(rng.integers(0, wl.N, 128).tolist()))
    check(y, x, qw, s, z, cols=cols)


def test_w4a16_deterministic(cuda_lib):
    dev = torch.device("cuda:0")
    x, qw, s, z = (t.to(dev) for t in workloads.make_w4a16(16, 1024, 2048, seed=9))
    outs = [cuda_lib.w4a16_matmul(x, qw, s, z) for _ in range(4)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
