"""Pins for the FP8 preparation oracle (E4M3 coding, rotation, block quantisation).

  * E4M3 codes worked by hand from the OCP definition (tests/golden/e4m3_ocp.json);
  * every finite code round-trips; every midpoint between neighbours rounds to the
    even code;
  * the encoder agrees with torch's float8_e4m3fn conversion (a library routine)
    on random values after clamping to +-448;
  * the rotation equals the exact rational product rounded once to fp32, and is
    exact for a permutation matrix;
  * block scales: amax of the tile maps to 448, zeros give scale 1, dequantised
    values are within half a code step of the input;
  * the quantiser multiplies by the fp32 reciprocal of the tile scale (a value
    worked by hand where dividing instead would give the neighbouring code).
"""
import json
import os

import numpy as np
import pytest
import torch

from fractions import Fraction

from oracle import e4m3_decode, e4m3_encode, prepare_fp8, dequantize, rotate

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_golden_codes():
    g = json.load(open(os.path.join(GOLDEN, "e4m3_ocp.json")))
    for val, code in g["exact"]:
        assert int(e4m3_encode(np.float32(val))) == code, val
        assert e4m3_decode(np.uint8(code)) == val, code
    for row in g["rounded"]:
        val, code = row[0], row[1]
        assert int(e4m3_encode(np.float32(val))) == code, val


def test_all_codes_round_trip_and_midpoints_to_even():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = e4m3_decode(codes)
    back = e4m3_encode(vals.astype(np.float32))
    # +0 and -0 both decode to 0; the sign is kept
    np.testing.assert_array_equal(back, codes)
    pos = np.sort(e4m3_decode(np.arange(0, 127, dtype=np.uint8)))
    assert pos[-1] == 448.0 and pos[1] == 2.0 ** -9
    for a, b in zip(pos[:-1], pos[1:]):
        mid = np.float32((a + b) / 2)
        ca, cb = int(e4m3_encode(np.float32(a))), int(e4m3_encode(np.float32(b)))
        got = int(e4m3_encode(mid))
        assert got == (ca if ca % 2 == 0 else cb), (a, b)


def test_encoder_matches_torch_float8():
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.standard_normal(200000) * 10.0,
        rng.standard_normal(50000) * 1e-3,
        rng.uniform(-500, 500, 50000),
    ]).astype(np.float32)
    xc = np.clip(x, -448.0, 448.0)
    ref = torch.from_numpy(xc).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = e4m3_encode(x)
    np.testing.assert_array_equal(got, ref)


def _fp32_round(v: Fraction) -> float:
    """Exact rational -> nearest fp32 (ties to even), for normal magnitudes."""
    if v == 0:
        return 0.0
    a = abs(v)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    quantum = Fraction(2) ** (e - 23)
    n = round(a / quantum)                 # Fraction.__round__: half to even
    r = float(n * quantum)
    return r if v > 0 else -r


def test_rotation_is_the_exact_product_rounded_once():
    rng = np.random.default_rng(3)
    d = 16
    x = torch.from_numpy(rng.standard_normal((5, d)).astype(np.float32)).to(torch.bfloat16)
    r = torch.from_numpy(rng.standard_normal((d, d)).astype(np.float32) / 4).to(torch.bfloat16)
    y = rotate(x.float().numpy(), r.float().numpy())
    assert y.dtype == np.float32
    # independent restatement: exact rational sum of the (bf16) products, one rounding
    xf, rf = x.double().numpy(), r.double().numpy()
    for i in range(5):
        for c in range(d):
            exact = sum(Fraction(float(xf[i, kk])) * Fraction(float(rf[kk, c])) for kk in range(d))
            assert float(y[i, c]) == _fp32_round(exact), (i, c)
    # a permutation matrix moves values exactly
    perm = np.eye(d, dtype=np.float32)[rng.permutation(d)]
    yp = rotate(x.float().numpy(), perm)
    np.testing.assert_array_equal(yp, x.float().numpy() @ perm)


def test_quantiser_multiplies_by_the_fp32_reciprocal():
    """Worked by hand. A tile whose largest magnitude is 3136 = 7 * 448 has the
    scale 3136 / 448 = 7 exactly; r = fp32(1/7) = 0.142857149... is 4.5e-8 too
    large (relative). The value 10.9375 = 7 * 1.5625 sits, after exact division,
    on the midpoint 1.5625 between the E4M3 values 1.5 (code 0x3C, even mantissa)
    and 1.625 (0x3D), which ties to 0x3C; multiplied by r it becomes
    fp32(1.5625 * (1 + 4.5e-8)) = 1.5625 + 2^-23, above the midpoint: 0x3D."""
    x = torch.zeros(1, 1, 128, 128, dtype=torch.bfloat16)
    x[0, 0, 0, 0] = 3136.0
    x[0, 0, 5, 7] = 10.9375
    x[0, 0, 9, 3] = -10.9375
    codes, scales = prepare_fp8(x, None)
    assert scales[0, 0, 0] == 7.0
    assert codes[0, 0, 0, 0] == 0x7E            # 448
    assert codes[0, 0, 5, 7] == 0x3D
    assert codes[0, 0, 9, 3] == 0xBD


def test_block_quantisation_properties():
    rng = np.random.default_rng(11)
    B, H, N, d = 1, 2, 300, 128
    x = torch.from_numpy(rng.standard_normal((B, H, N, d)).astype(np.float32) * 3).to(torch.bfloat16)
    x[0, 1, 128:256] = 0.0                         # an all-zero tile
    codes, scales = prepare_fp8(x, None)
    assert codes.shape == (B, H, N, d) and scales.shape == (B, H, 3)
    assert scales[0, 1, 1] == 1.0
    xf = x.float().numpy()
    for h in range(H):
        for t in range(3):
            blk = xf[0, h, t * 128:(t + 1) * 128]
            if h == 1 and t == 1:
                continue
            assert scales[0, h, t] == np.float32(np.abs(blk).max()) / np.float32(448.0)
            # the tile's largest magnitude encodes as +-448 (code 0x7E / 0xFE)
            i = np.unravel_index(np.abs(blk).argmax(), blk.shape)
            assert codes[0, h, t * 128 + i[0], i[1]] & 0x7F == 0x7E
    deq = dequantize(codes, scales)
    # half a code step: relative 2^-4 for normals, 2^-10 * scale absolute for subnormals
    s_full = np.repeat(scales, 128, axis=-1)[..., :N][..., None]
    err = np.abs(deq - xf)
    bound = np.maximum(np.abs(xf) * 2.0 ** -4, 2.0 ** -10 * s_full) * (1 + 1e-6)
    assert np.all(err <= bound)


def test_rotation_spreads_outliers():
    """Incoherent processing lowers the tile amax relative to the RMS when a few
    large outliers are present."""
    from workloads import make_rotation
    rng = np.random.default_rng(5)
    x = rng.standard_normal((1, 1, 128, 128)).astype(np.float32)
    x[0, 0, rng.integers(0, 128, 16), rng.integers(0, 128, 16)] = 20.0
    xb = torch.from_numpy(x).to(torch.bfloat16)
    _, rot = make_rotation(128, 1)
    _, s_plain = prepare_fp8(xb, None)
    _, s_rot = prepare_fp8(xb, rot)
    assert s_rot[0, 0, 0] < 0.5 * s_plain[0, 0, 0]


def _quantize_like_gpu(y32):
    """Block quantisation of an fp32 y [BH, N, d] the way the reading defines it
    (fp32 amax / 448, fp32 reciprocal, fp32 product, E4M3)."""
    BH, N, d = y32.shape
    T = (N + 127) // 128
    codes = np.empty(y32.shape, np.uint8)
    scales = np.empty((BH, T), np.float32)
    for t in range(T):
        blk = y32[:, t * 128:(t + 1) * 128]
        amax = np.abs(blk).reshape(BH, -1).max(1)
        s = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
        inv = (np.float32(1.0) / s).astype(np.float32)
        scales[:, t] = s
        codes[:, t * 128:(t + 1) * 128] = e4m3_encode((blk * inv[:, None, None]).astype(np.float32))
    return codes, scales


def test_rotated_code_bounds_admit_fp32_accumulation_and_reject_mistakes():
    """The GPU check for rotated tensors (tests/fp8_bounds.py) accepts the codes of
    any fp32 accumulation order of x R (here: increasing k, decreasing k) and the
    oracle's own, and rejects a transposed rotation and a dropped rotation."""
    from fp8_bounds import check_rotated
    from workloads import make_qkv, make_rotation
    q, _, _ = make_qkv(1, 2, 300, 128, seed=8, outliers=("q",))
    x = q.reshape(2, 300, 128)
    _, rot = make_rotation(128, 3)
    xf, rf = x.float().numpy(), rot.float().numpy()
    codes_o, scales_o = prepare_fp8(x.unsqueeze(0), rot)
    assert check_rotated(x, rot, codes_o[0], scales_o[0]) == 0
    for order in (range(128), range(127, -1, -1)):
        y = np.zeros((2, 300, 128), np.float32)
        for kk in order:
            y = (y + xf[..., kk:kk + 1] * rf[kk:kk + 1, :]).astype(np.float32)
        c, s = _quantize_like_gpu(y)
        check_rotated(x, rot, c, s)
    for wrong in (xf @ rf.T, xf):
        c, s = _quantize_like_gpu(wrong.astype(np.float32))
        with pytest.raises(AssertionError):
            check_rotated(x, rot, c, s)
