"""CPU oracle for the FP8 preparation step: incoherent rotation and block quantisation.

TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference leg may import or call anything under oracle/.

Method ("FlashAttention scaling, multi-GPU training and weight quantization", §1,
FlashAttention-3 FP8 bullet): Q and K are multiplied by a random orthogonal matrix
before quantisation (incoherent processing, which spreads outliers), and every
small tile is quantised with its own scale (block quantisation). V is quantised
without rotation.

Readings (the page gives no numbers, so these are this library's definitions,
shared with the CUDA kernels only through this specification, not through code):
  * tile = 128 consecutive tokens x all d channels of one (batch, head);
  * rotated value y = x R, the plain matrix product: computed here in fp64
    (every product of two bf16 values is exact there, the sums carry errors of
    order 2^-45 relative) and rounded once to fp32. The page fixes "multiply by
    a random orthogonal matrix", not an accumulation order or precision, so a
    tensor-core product with fp32 accumulation is an equally valid computation
    of y: its result differs from this one by fp32 accumulation error only;
  * scale = amax(|y| over the tile) / 448 in fp32 (IEEE division); a tile of all
    zeros gets scale 1;
  * code = E4M3(y * r), r = 1 / scale in fp32 (one IEEE division per tile), the
    product rounded to fp32, then round-to-nearest-even to OCP E4M3 with
    saturation to +-448 (the format's largest finite value);
  * dequantised value = decode(code) * scale, which is what the attention
    oracle consumes.
Where a float decides an integer code, the decision is taken in fp32, the
kernel's precision. Without rotation (V) y = x exactly, so codes and scales are
unique and compare bit for bit; with rotation the kernel's y may differ from
the exact product by its accumulation error, which can move a code by one step
where y * r lies within that error of a rounding boundary (the GPU tests bound
where and how often).

E4M3 (OCP 8-bit floating point, E4M3 variant): 1 sign bit, 4 exponent bits with
bias 7, 3 mantissa bits; exponent field 0 holds subnormals m * 2^-9; the code
S.1111.111 is NaN; there are no infinities; the largest finite value is 448.

Pinned by tests/test_fp8_oracle_pins.py and tests/golden/e4m3_ocp.json.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
TILE = 128


def e4m3_decode(codes):
    """uint8 codes -> fp64 values (NaN codes decode to NaN)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 0xF) & (m == 0x7), np.nan, val)
    return sign * val


def e4m3_encode(x):
    """fp32/fp64 values -> uint8 E4M3 codes, round-to-nearest-even, saturating
    to +-448. Works in fp64, where every step below is exact for fp32 inputs."""
    x = np.asarray(x, dtype=np.float64)
    neg = np.signbit(x)
    a = np.abs(x)
    safe = np.where(a > 0, a, 1.0)
    # binade exponent, clamped to the smallest normal binade (2^-6)
    e = np.floor(np.log2(safe))
    # guard against log2 rounding at exact powers of two
    e = np.where(np.exp2(e) > safe, e - 1, e)
    e = np.where(np.exp2(e + 1) <= safe, e + 1, e)
    e = np.maximum(e, -6.0)
    quantum = np.exp2(e - 3.0)                 # spacing of representable values
    n = np.rint(a / quantum)                   # numpy rint: ties to even
    val = np.minimum(n * quantum, E4M3_MAX)    # saturate
    code = np.zeros(a.shape, dtype=np.int64)
    sub = val < 2.0 ** -6
    code = np.where(sub, np.rint(val / 2.0 ** -9), code)
    safe_v = np.where(sub, 1.0, val)
    ev = np.floor(np.log2(safe_v))
    ev = np.where(np.exp2(ev) > safe_v, ev - 1, ev)
    ev = np.where(np.exp2(ev + 1) <= safe_v, ev + 1, ev)
    mant = np.rint((safe_v / np.exp2(ev) - 1.0) * 8.0)
    code = np.where(sub, code, (ev + 7.0) * 8.0 + mant)
    code = code.astype(np.int64) | np.where(neg & (val > 0), 0x80, 0)
    # negative zero keeps its sign bit like the hardware conversion
    code = np.where(neg & (val == 0), 0x80, code)
    return code.astype(np.uint8)


def rotate(x_bf16_as_f32, rot_bf16_as_f32):
    """y = x R: the exact product (fp64: bf16 products are exact, the sums are
    within ~2^-45 relative) rounded once to fp32.
    x: [..., d] float32 holding bf16 values; rot: [d, d] float32 holding bf16."""
    x = np.asarray(x_bf16_as_f32, dtype=np.float64)
    r = np.asarray(rot_bf16_as_f32, dtype=np.float64)
    return (x @ r).astype(np.float32)


def quantize_tiles(y_f32):
    """Block quantisation of [BH, N, d] fp32 values: tiles of 128 tokens.
    Returns (codes uint8 [BH, N, d], scales float32 [BH, ceil(N/128)])."""
    y = np.asarray(y_f32, dtype=np.float32)
    BH, N, d = y.shape
    T = (N + TILE - 1) // TILE
    codes = np.empty((BH, N, d), dtype=np.uint8)
    scales = np.empty((BH, T), dtype=np.float32)
    for t in range(T):
        blk = y[:, t * TILE:(t + 1) * TILE, :]
        amax = np.abs(blk).reshape(BH, -1).max(axis=1).astype(np.float32)
        sc = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
        scales[:, t] = sc
        inv = (np.float32(1.0) / sc).astype(np.float32)           # fp32 IEEE division, once per tile
        q = (blk * inv[:, None, None]).astype(np.float32)         # fp32 product, rounded once
        codes[:, t * TILE:(t + 1) * TILE, :] = e4m3_encode(q)
    return codes, scales


def prepare_fp8(x_bf16, rot_bf16=None):
    """Rotation (optional) and block quantisation of one tensor.

    x_bf16:   torch bf16 tensor or float array holding bf16 values, [B, H, N, d].
    rot_bf16: [d, d] bf16 values or None (no rotation, as for V).
    Returns (codes uint8 [B,H,N,d], scales float32 [B,H,ceil(N/128)])."""
    x = _to_f32(x_bf16)
    B, H, N, d = x.shape
    x = x.reshape(B * H, N, d)
    y = x if rot_bf16 is None else rotate(x, _to_f32(rot_bf16))
    codes, scales = quantize_tiles(y)
    return codes.reshape(B, H, N, d), scales.reshape(B, H, -1)


def dequantize(codes, scales):
    """fp64 values decode(code) * scale(tile) for [B,H,N,d] codes."""
    B, H, N, d = codes.shape
    vals = e4m3_decode(codes)
    s = np.repeat(np.asarray(scales, dtype=np.float64), TILE, axis=-1)[..., :N]
    return vals * s[..., None]


def _to_f32(t):
    try:
        import torch
        if isinstance(t, torch.Tensor):
            return t.detach().to("cpu").to(torch.float32).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(t, dtype=np.float32)
