"""Where a rotated tensor's FP8 codes may differ from the oracle's.

The rotation y = x R is a dense product; the oracle takes the exact product
rounded once to fp32, the GPU computes it on the tensor cores with fp32
accumulation in an order of its own. Element (i, c) of the GPU's y is then
within B_ic = GAMMA * sum_k |x_ik R_kc| of the exact value (GAMMA covers 128
fp32 roundings of the running sum, doubled in case the accumulator truncates).
That moves the tile's amax, hence its scale and reciprocal, within computable
intervals, and each code may only land between the codes of the smallest and
the largest value y * r can take. `check_rotated` asserts exactly that, plus
that such moved codes stay rare.
"""
import numpy as np

from oracle import e4m3_decode, e4m3_encode, rotate

GAMMA = 2.0 ** -16
TILE = 128


def _ulp32(a):
    a = np.abs(np.asarray(a, dtype=np.float32))
    return (np.nextafter(a, np.float32(np.inf)) - a).astype(np.float64)


def check_rotated(x_bf16, rot_bf16, codes, scales, max_moved_frac=1e-3):
    """x_bf16: torch bf16 [BH, N, d] (CPU); rot_bf16: torch bf16 [d, d];
    codes: uint8 [BH, N, d] and scales: fp32 [BH, T] from the GPU.
    Returns the number of codes that differ from the oracle's."""
    import torch
    x = x_bf16.to(torch.float64).numpy()
    r = rot_bf16.to(torch.float64).numpy()
    BH, N, d = x.shape
    T = (N + TILE - 1) // TILE
    y_o = rotate(x.astype(np.float32), r.astype(np.float32)).astype(np.float64)   # oracle's fp32 y
    bound = GAMMA * (np.abs(x) @ np.abs(r)) + _ulp32(y_o)                          # |y_gpu - y_o|
    moved = 0
    codes = np.asarray(codes)
    scales = np.asarray(scales, dtype=np.float32)
    for t in range(T):
        sl = slice(t * TILE, min(N, (t + 1) * TILE))
        ay, bb = np.abs(y_o[:, sl]), bound[:, sl]
        amax_lo = np.maximum(ay - bb, 0).reshape(BH, -1).max(1)
        amax_hi = (ay + bb).reshape(BH, -1).max(1)
        s = scales[:, t].astype(np.float64)
        # scale = fp32(amax / 448): within one fp32 step of the amax interval / 448
        s_lo = amax_lo / 448.0 * (1 - 2.0 ** -23)
        s_hi = amax_hi / 448.0 * (1 + 2.0 ** -23)
        ok_s = (s >= s_lo) & (s <= s_hi) | ((amax_lo == 0) & (s == 1.0))
        assert ok_s.all(), f"tile {t}: scale outside [{s_lo[~ok_s][:3]}, {s_hi[~ok_s][:3]}]: {s[~ok_s][:3]}"
        inv_lo = 1.0 / s * (1 - 2.0 ** -23)        # fp32(1/s) for this (GPU) scale
        inv_hi = 1.0 / s * (1 + 2.0 ** -23)
        t_lo = np.maximum(ay - bb, 0) * inv_lo[:, None, None] * (1 - 2.0 ** -23)
        t_hi = (ay + bb) * inv_hi[:, None, None] * (1 + 2.0 ** -23)
        c = codes[:, sl]
        mag = np.abs(e4m3_decode(c & 0x7F))
        lo_code = np.abs(e4m3_decode(e4m3_encode(t_lo.astype(np.float32))))
        hi_code = np.abs(e4m3_decode(e4m3_encode(np.minimum(t_hi, 448.0).astype(np.float32))))
        assert np.all(mag >= lo_code) and np.all(mag <= hi_code), "code outside its interval"
        # the sign follows y unless y may be zero
        sign_free = (ay - bb) <= 0
        sign_ok = ((c >> 7) == (y_o[:, sl] < 0)) | sign_free | (mag == 0)
        assert np.all(sign_ok), "code sign"
        # how many codes differ from the oracle's own (with its own scale)
        s_o = np.where(ay.reshape(BH, -1).max(1) > 0, (ay.reshape(BH, -1).max(1).astype(np.float32)
                                                       / np.float32(448.0)), np.float32(1.0)).astype(np.float32)
        inv_o = (np.float32(1.0) / s_o).astype(np.float32)
        c_o = e4m3_encode((y_o[:, sl].astype(np.float32) * inv_o[:, None, None]).astype(np.float32))
        moved += int((c_o != c).sum())
    assert moved <= max_moved_frac * codes.size, f"{moved} of {codes.size} codes moved"
    return moved
