"""Seeded synthetic inputs for the attention forward path.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests. It only draws random numbers and lays them out; it holds none of
the attention arithmetic (no scores, no softmax, no rotation, no quantisation).

Workload shapes follow the pages:
  * ViT-B/16: a 224x224 image cut into 16x16 patches gives N = 196 tokens, 12
    heads ("Self-Attention, CUDA kernels and FlashAttention", §1, patch grid and
    multi-head paragraph); head width 64.
  * LLM training and long-sequence shapes with head width 128 and causal masking.
  * MXFP8 shape: the FP8 shape and outliers, quantised in 32-value blocks along d
    ("Efficient MoE training for biological foundation models", the
    low-precision paragraph).
  * FP8 shape: Q, K and V drawn with rare large outliers; Q and K are later
    multiplied by a random orthogonal matrix before block quantisation
    ("FlashAttention scaling, multi-GPU training and weight quantization", §1,
    FlashAttention-3 FP8 bullet: block quantisation and incoherent processing).
    The same shape also runs in BF16 without quantisation (outliers in Q and K).

Recipe (all on the CPU, torch.Generator seeded per workload):
  1. Q, K, V drawn in that order as fp32 iid N(0, 1), shape [B, H, N, d].
  2. Outliers, when the workload asks for them: for each listed tensor in the
     order q, k, v, round(0.001 * numel) distinct flat positions are drawn
     uniformly (randperm prefix) and overwritten with +-20 (sign drawn per
     position, fair coin).
  3. Rounded to bf16 (round-to-nearest-even).
  4. For FP8 workloads, a d x d orthogonal matrix is drawn from the Haar
     measure: G ~ N(0,1) in fp64, G = QR, Q's columns multiplied by the signs of
     diag(R). It is returned in fp64 and rounded to bf16 (the product the
     kernels and the oracle both consume).
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    fp8: bool = False
    mx: bool = False              # MXFP8 inputs (32-value blocks, no rotation)
    outliers: tuple = ()          # subset of ("q", "k", "v")
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def flops(self) -> float:
        """Algorithmic FLOPs: 4*B*H*N^2*d, halved for causal masking."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2.0 if self.causal else f


# The five workloads, in the order the parity tests and the benchmark use.
WORKLOADS = {
    "vit_b16_single": Workload("vit_b16_single", 1, 12, 196, 64, False, seed=1000),
    "vit_b16_batch": Workload("vit_b16_batch", 64, 12, 196, 64, False, seed=1001),
    "llm_train_causal": Workload("llm_train_causal", 4, 32, 4096, 128, True, seed=1002),
    "long_seq_causal": Workload("long_seq_causal", 1, 16, 32768, 128, True,
                                outliers=("q", "k"), seed=1003),
    "fp8_rotated": Workload("fp8_rotated", 2, 32, 8192, 128, False, fp8=True,
                            outliers=("q", "k", "v"), seed=1004),
    # the FP8 workload's shape in BF16 (no quantisation): the non-causal
    # N >= 4096, d = 128 shape of the tensor-core target, with the BF16
    # long-sequence recipe (outliers in Q and K only: with magnitude-20 V
    # entries |O| reaches 20, where one bf16 step of the output is 0.125)
    "noncausal_8k_bf16": Workload("noncausal_8k_bf16", 2, 32, 8192, 128, False,
                                  outliers=("q", "k"), seed=1005),
    # the FP8 workload's shape and outlier recipe, quantised to MXFP8 (one
    # power-of-two scale per 32 values of a row; no rotation)
    "mxfp8_8k": Workload("mxfp8_8k", 2, 32, 8192, 128, False, mx=True,
                         outliers=("q", "k", "v"), seed=1007),
}

OUTLIER_FRACTION = 0.001
OUTLIER_MAGNITUDE = 20.0


def _plant_outliers(x: torch.Tensor, gen: torch.Generator) -> None:
    flat = x.view(-1)
    n = int(round(OUTLIER_FRACTION * flat.numel()))
    if n == 0:
        return
    pos = torch.randperm(flat.numel(), generator=gen)[:n]
    sign = torch.randint(0, 2, (n,), generator=gen).to(torch.float32) * 2.0 - 1.0
    flat[pos] = sign * OUTLIER_MAGNITUDE


def make_qkv(B: int, H: int, N: int, d: int, seed: int, outliers=()):
    """Return bf16 CPU tensors q, k, v of shape [B, H, N, d] (contiguous)."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    out = {}
    for name in ("q", "k", "v"):
        out[name] = torch.randn((B, H, N, d), generator=gen, dtype=torch.float32)
    for name in ("q", "k", "v"):
        if name in outliers:
            _plant_outliers(out[name], gen)
    return tuple(out[n].to(torch.bfloat16).contiguous() for n in ("q", "k", "v"))


def make_rotation(d: int, seed: int):
    """Haar-random orthogonal d x d matrix: (fp64 tensor, its bf16 rounding)."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    g = torch.randn((d, d), generator=gen, dtype=torch.float64)
    qf, rf = torch.linalg.qr(g)
    signs = torch.sign(torch.diagonal(rf))
    signs[signs == 0] = 1.0
    rot = qf * signs.unsqueeze(0)
    return rot.contiguous(), rot.to(torch.bfloat16).contiguous()


def make_workload(w: Workload):
    """Inputs of a named workload: dict with q, k, v (bf16 CPU) and, for FP8
    workloads, rot64 / rot (fp64 and bf16 rotation)."""
    q, k, v = make_qkv(w.B, w.H, w.N, w.d, w.seed, w.outliers)
    res = {"q": q, "k": k, "v": v}
    if w.fp8:
        res["rot64"], res["rot"] = make_rotation(w.d, w.seed + 7919)
    return res


@dataclasses.dataclass(frozen=True)
class GemmWorkload:
    """A W4A16 GEMM: Y[M, N] = X[M, K] W[K, N] with 4-bit weights."""
    name: str
    M: int
    N: int
    K: int
    seed: int = 0

    @property
    def flops(self) -> float:
        return 2.0 * self.M * self.N * self.K


# decode with a 70B-class model: 16 tokens through one MLP projection
# (hidden 8192 -> intermediate 28672), the weight-bandwidth-bound case of the
# pages' quantisation section
GEMM_WORKLOADS = {
    "w4a16_decode_mlp": GemmWorkload("w4a16_decode_mlp", 16, 28672, 8192, seed=1006),
}


def make_w4a16(M: int, N: int, K: int, seed: int):
    """Random W4A16 operands (CPU): x fp16 [M, K] iid N(0, 1); qweight int32
    [K/8, N] uniform random words (every nibble an independent uniform code
    0..15); scales fp16 [K/128, N] uniform in [0.005, 0.02); zeros uint8
    [K/128, N] uniform 0..15."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    x = torch.randn((M, K), generator=gen, dtype=torch.float32).to(torch.float16)
    qweight = torch.randint(-2**31, 2**31, (K // 8, N), generator=gen, dtype=torch.int64).to(torch.int32)
    scales = (torch.rand((K // 128, N), generator=gen) * 0.015 + 0.005).to(torch.float16)
    zeros = torch.randint(0, 16, (K // 128, N), generator=gen, dtype=torch.int64).to(torch.uint8)
    return x, qweight, scales, zeros


def sample_rows(N: int, count: int, seed: int):
    """Sorted distinct query rows to check at full size: the first and last 128
    rows, the rows on either side of every 128-row block boundary that falls in
    them, and `count` seeded random rows."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    rows = set(range(min(N, 128)))
    rows |= set(range(max(0, N - 128), N))
    rnd = torch.randint(0, N, (count,), generator=gen).tolist()
    rows |= set(rnd)
    return sorted(rows)
