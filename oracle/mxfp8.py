"""CPU oracle for MXFP8 quantisation (32-element blocks with a shared power-of-two scale).

TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference leg may import or call anything under oracle/.

Method ("Efficient MoE training for biological foundation models", the low-precision
paragraph: MXFP8, the Blackwell-native 8-bit format with one scale per 32 values,
used with the tensor cores' block-scaled products). Each block of 32 consecutive
values of a row (along the head dimension d) shares one scale X = 2^E stored as an
E8M0 byte (E + 127); each value is stored as an E4M3 code of v / X.

Readings (the page names the format, not its arithmetic; the definitions below are
the OCP Microscaling format's, restated):
  * E = floor(log2(max |v| over the block)) - 8, the exponent of the block's
    largest magnitude minus that of E4M3's largest binade (448 = 1.75 * 2^8), so
    the largest value lands in [256, 512) and is rounded and saturated to E4M3;
    E is clamped to [-127, 127] (E8M0 bytes 0 .. 254);
  * an all-zero block gets E = 0 (byte 127, X = 1) and zero codes;
  * code = E4M3 round-to-nearest-even, saturating to +-448, of v * 2^-E (an exact
    power-of-two scaling: every bf16 input times 2^-E is exact in fp32);
  * dequantised value = decode(code) * 2^E.

Pinned by tests/test_mxfp8_oracle_pins.py.
"""
from __future__ import annotations

import numpy as np

from .fp8 import e4m3_decode, e4m3_encode

BLOCK = 32


def mx_quantize(x):
    """x: [..., d] values (any real dtype, read exactly as fp64), d a multiple of 32.
    Returns (codes uint8 [..., d], scale bytes uint8 [..., d/32])."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    if d % BLOCK:
        raise ValueError("d must be a multiple of 32")
    blocks = x.reshape(x.shape[:-1] + (d // BLOCK, BLOCK))
    amax = np.abs(blocks).max(axis=-1)
    safe = np.where(amax > 0, amax, 1.0)
    _, ex = np.frexp(safe)                   # safe = m * 2^ex, m in [0.5, 1): floor(log2) = ex - 1
    e = np.where(amax > 0, ex - 1 - 8, 0)
    e = np.clip(e, -127, 127)
    scaled = blocks * np.exp2(-e.astype(np.float64))[..., None]
    codes = e4m3_encode(scaled).reshape(x.shape)
    return codes, (e + 127).astype(np.uint8)


def mx_dequantize(codes, scale_bytes):
    """fp64 values decode(code) * 2^(byte - 127)."""
    codes = np.asarray(codes, dtype=np.uint8)
    d = codes.shape[-1]
    vals = e4m3_decode(codes).reshape(codes.shape[:-1] + (d // BLOCK, BLOCK))
    e = np.asarray(scale_bytes, dtype=np.float64) - 127.0
    return (vals * np.exp2(e)[..., None]).reshape(codes.shape)
