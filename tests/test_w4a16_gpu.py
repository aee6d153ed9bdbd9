"""GPU parity of the W4A16 GEMM (w4a16_gemm and w4a16_gemm_splitk through the C
ABI) against the oracle.

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


def run(lib, x, qw, s, z, split_k=True, workspace=None):
    dev = torch.device("cuda:0")
    M, N = x.shape[0], qw.shape[1]
    raw = torch.full((M * N + 2 * CANARY,), float("nan"), dtype=torch.float16, device=dev)
    raw[:CANARY] = 5.0
    raw[-CANARY:] = 5.0
    y = raw[CANARY:CANARY + M * N].view(M, N)
    lib.w4a16_matmul(x.to(dev), qw.to(dev), s.to(dev), z.to(dev), out=y, split_k=split_k, workspace=workspace)
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


@pytest.mark.parametrize("split_k", [True, False], ids=["splitk", "tile_per_cta"])
@pytest.mark.parametrize("M,K,N", [(1, 128, 128), (16, 256, 256), (5, 1024, 384), (128, 512, 128),
                                   (33, 384, 640), (100, 128, 256)])
def test_w4a16_small_parity(cuda_lib, M, K, N, split_k):
    x, qw, s, z = workloads.make_w4a16(M, N, K, seed=M + K + N)
    check(run(cuda_lib, x, qw, s, z, split_k=split_k), x, qw, s, z)


# Split-K runs: (M, K, N) with 8 slices per CTA cutting tiles into several
# segments, runs that start and end inside tiles (slices per tile not a multiple
# of 8), a run spanning three tiles, and the largest M
SPLIT_SHAPES = [
    (16, 4096, 1024),     # 8 tiles x 32 slices, 32 CTAs: four aligned segments per tile
    (16, 1280, 3072),     # 24 tiles x 10 slices, 30 CTAs: runs straddle tile boundaries
    (3, 2176, 1152),      # 9 tiles x 17 slices, 19 CTAs: ragged segments, M padded to 16
    (128, 2048, 4608),    # 36 tiles x 16 slices, 72 CTAs at M = 128 (two A buffers)
    (40, 384, 38400),     # 300 tiles x 3 slices, 112 CTAs: runs over up to four tiles
    (16, 8192, 57344),    # 448 tiles x 64 slices, 296 CTAs: ~97-slice runs over up to three tiles
]


@pytest.mark.parametrize("M,K,N", SPLIT_SHAPES)
def test_w4a16_splitk_parity_and_tickets(cuda_lib, M, K, N):
    """Split-K against the oracle (every column for the small shapes, sampled
    columns for the largest), with a caller workspace whose tickets must read
    zero again after the call."""
    lib = cuda_lib
    dev = torch.device("cuda:0")
    x, qw, s, z = workloads.make_w4a16(M, N, K, seed=M * 7 + K + N)
    need = lib.w4a16_gemm_splitk_workspace_bytes(M, N, K)
    ws = torch.zeros(need + 4096, dtype=torch.uint8, device=dev)
    ws[need:] = 0xA5                                   # beyond the required size: never written
    y = run(lib, x, qw, s, z, workspace=ws)
    tickets = ws[:16 * (N // 128)]
    assert int(tickets.count_nonzero()) == 0, "tickets not reset"
    assert bool((ws[need:] == 0xA5).all()), "write past the workspace"
    cols = None
    if N > 8192:
        rng = np.random.default_rng(N)
        cols = sorted(set(range(256)) | set(range(N - 256, N)) | set(rng.integers(0, N, 256).tolist()))
    check(y, x, qw, s, z, cols=cols)


def test_w4a16_splitk_and_tile_per_cta_agree(cuda_lib):
    """The two schedules sum in different orders, so they agree to the fp32
    accumulation bound, not bit for bit; the split-K result is the same on every
    call (fixed partial order) and with a fresh workspace."""
    lib = cuda_lib
    dev = torch.device("cuda:0")
    M, K, N = 16, 2176, 3072
    x, qw, s, z = (t.to(dev) for t in workloads.make_w4a16(M, N, K, seed=41))
    plain = lib.w4a16_matmul(x, qw, s, z, split_k=False)
    outs = [lib.w4a16_matmul(x, qw, s, z) for _ in range(5)]
    fresh = torch.zeros(lib.w4a16_gemm_splitk_workspace_bytes(M, N, K), dtype=torch.uint8, device=dev)
    outs.append(lib.w4a16_matmul(x, qw, s, z, workspace=fresh))
    torch.cuda.synchronize()
    assert lib.attn_get_device_status(None) == lib.ATTN_OK
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    a, b = plain.float().cpu().numpy(), outs[0].float().cpu().numpy()
    xa = np.abs(x.float().cpu().numpy().astype(np.float64))
    w = dequantize_weights(qw.cpu().numpy(), s.cpu().numpy(), z.cpu().numpy()).astype(np.float64)
    bound = 2.0 ** -10 * np.abs(a) + 2.0 ** -15 * (xa @ np.abs(w)) + 1e-7
    assert np.all(np.abs(a - b) <= bound)


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


def _scales(kind, shape, seed):
    """fp16 scales of one regime: typical ([0.005, 0.02)), tiny (2^-20 .. 2^-10, where
    s / 16 is mostly not an fp16 value), mixed (typical and tiny columns alternate, so
    every warp holds both), powers (2^-8 .. 2^-24: s / 16 exact down to 2^-20 only)."""
    gen = torch.Generator().manual_seed(seed)
    typical = (torch.rand(shape, generator=gen) * 0.015 + 0.005).to(torch.float16)
    tiny = torch.exp2(-10.0 - 10.0 * torch.rand(shape, generator=gen)).to(torch.float16)
    if kind == "typical":
        return typical
    if kind == "tiny":
        return tiny
    if kind == "mixed":
        out = typical.clone()
        out[:, 1::2] = tiny[:, 1::2]
        return out
    e = torch.randint(8, 25, shape, generator=gen).to(torch.float32)
    return torch.exp2(-e).to(torch.float16)


@pytest.mark.parametrize("split_k", [True, False], ids=["splitk", "tile_per_cta"])
@pytest.mark.parametrize("kind", ["typical", "tiny", "mixed", "powers"])
def test_w4a16_dequantisation_bit_exact_scale_regimes(cuda_lib, kind, split_k):
    """The kernel unpacks odd nibble pairs without a shift (16 (q - z) times s / 16)
    when s / 16 is exact for a whole warp and takes the shifting form otherwise;
    both must give fp16((q - z) s) bit for bit, for every scale regime."""
    K, N = 256, 384
    _, qw, _, z = workloads.make_w4a16(1, N, K, seed=11)
    s = _scales(kind, (K // 128, N), seed=12)
    ks = list(range(0, 16)) + [127, 128, 135, 200, 255]
    x = torch.zeros((len(ks), K), dtype=torch.float16)
    for m, k in enumerate(ks):
        x[m, k] = 1.0
    y = run(cuda_lib, x, qw, s, z, split_k=split_k)
    w = dequantize_weights(qw.numpy(), s.numpy(), z.numpy())
    np.testing.assert_array_equal(y, w[ks].astype(np.float32))


@pytest.mark.parametrize("split_k", [True, False], ids=["splitk", "tile_per_cta"])
def test_w4a16_workload_parity(cuda_lib, split_k):
    """The decode workload at full size (split-K is the launch the benchmark
    times); the oracle checks 384 sampled columns (three whole tiles' worth and
    scattered ones)."""
    wl = workloads.GEMM_WORKLOADS["w4a16_decode_mlp"]
    x, qw, s, z = workloads.make_w4a16(wl.M, wl.N, wl.K, wl.seed)
    y = run(cuda_lib, x, qw, s, z, split_k=split_k)
    rng = np.random.default_rng(0)
    cols = sorted(set(range(128)) | set(range(wl.N - 128, wl.N)) | set(rng.integers(0, wl.N, 128).tolist()))
    check(y, x, qw, s, z, cols=cols)


@pytest.mark.parametrize("split_k", [True, False], ids=["splitk", "tile_per_cta"])
def test_w4a16_deterministic(cuda_lib, split_k):
    dev = torch.device("cuda:0")
    x, qw, s, z = (t.to(dev) for t in workloads.make_w4a16(16, 1024, 2048, seed=9))
    outs = [cuda_lib.w4a16_matmul(x, qw, s, z, split_k=split_k) for _ in range(4)]
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
