"""CPU oracle for the W4A16 on-the-fly dequantisation GEMM.

TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference leg may import or call anything under oracle/.

Method ("FlashAttention scaling, multi-GPU training and weight quantization", §3,
the W4A16 kernels paragraph): weights are stored as 4-bit integers, eight to a
32-bit word; the kernel reads the packed words from HBM, unpacks them in
registers with shifts and masks, turns each into a 16-bit float with the stored
scale and zero point, and multiplies by the 16-bit activations on the tensor
cores without writing the expanded weights back to memory.

Readings (the page fixes none of the numbers; these are this library's
definitions, shared with the CUDA kernel only through this specification):
  * Y[M, N] = X[M, K] W[K, N], X and Y fp16, W the dequantised weights;
  * qweight: int32 [K/8, N]; word (w, n) holds the weights k = 8w .. 8w+7 of
    output column n, the weight k = 8w + PERM[i] in bits 4i .. 4i+3 with
    PERM = (0, 2, 4, 6, 1, 3, 5, 7) (so that one mask of 0x000F000F over the
    word shifted by 4j picks the adjacent pair k = 8w+2j, 8w+2j+1);
  * groups of G = 128 consecutive k share one fp16 scale and one zero point
    (an integer 0..15, one byte) per output column: scales fp16 [K/G, N],
    zeros uint8 [K/G, N];
  * dequantised weight W[k, n] = fp16((q - z) * s): q - z is an exact small
    integer, the product is rounded once to fp16 (round to nearest even);
  * Y = X W exactly (every product of two fp16 values is exact in fp64 and the
    fp64 sums are far below fp16 resolution), rounded once to fp16 by the
    caller of this oracle when it compares.

Pinned by tests/test_w4a16_oracle_pins.py.
"""
from __future__ import annotations

import numpy as np

GROUP = 128
PERM = (0, 2, 4, 6, 1, 3, 5, 7)


def unpack_int4(qweight):
    """int32 [K/8, N] -> uint8 [K, N] weight codes q (0..15)."""
    w = np.asarray(qweight).astype(np.int64) & 0xFFFFFFFF
    KW, N = w.shape
    q = np.empty((KW * 8, N), dtype=np.uint8)
    for i in range(8):
        q[PERM[i]::8] = ((w >> (4 * i)) & 0xF).astype(np.uint8)
    return q


def dequantize_weights(qweight, scales, zeros):
    """fp16 [K, N]: fp16((q - z) * s) with the group's scale and zero point."""
    q = unpack_int4(qweight).astype(np.int32)
    s = np.repeat(np.asarray(scales, dtype=np.float16), GROUP, axis=0)
    z = np.repeat(np.asarray(zeros, dtype=np.int32), GROUP, axis=0)
    # (q - z) is exact in fp16; numpy's fp16 multiply rounds the exact product once
    return (q - z).astype(np.float16) * s


def w4a16_gemm_fp64(x, qweight, scales, zeros):
    """Y = X W in fp64 (exact up to fp64 summation), X fp16 [M, K]."""
    w = dequantize_weights(qweight, scales, zeros).astype(np.float64)
    return np.asarray(x, dtype=np.float16).astype(np.float64) @ w
