"""Pins for the MXFP8 oracle (oracle/mxfp8.py), worked by hand from its definition.

  * a block whose largest magnitude is 1.0 gets E = -8 (byte 119): 1.0 becomes
    2^8 = 256 (code 0x78) and 0.3 becomes 76.8, which rounds to 80 (code 0x6A),
    dequantised 80 * 2^-8 = 0.3125;
  * a block whose largest magnitude is 500 gets E = 0 and saturates to 448;
  * an all-zero block: byte 127, zero codes;
  * scales are powers of two, the largest element of every block lands in
    [256, 512) after scaling, and every dequantised value is within half an E4M3
    step of its input (relative 2^-4, absolute 2^-10 * 2^E at the subnormals),
    except values in [448, 512) * 2^E, which saturate to 448 * 2^E;
  * blocks are 32 consecutive values of a row: changing one value only moves its
    own block's scale.
"""
import numpy as np

from oracle.mxfp8 import mx_dequantize, mx_quantize


def test_hand_worked_block():
    x = np.zeros((1, 64))
    x[0, 0], x[0, 1], x[0, 2] = 1.0, 0.3, -0.5
    x[0, 32:] = 0.0
    codes, sb = mx_quantize(x)
    assert sb.tolist() == [[119, 127]]
    assert codes[0, 0] == 0x78 and codes[0, 1] == 0x6A and codes[0, 2] == 0xF0   # -0.5 -> -128
    assert not codes[0, 32:].any()
    deq = mx_dequantize(codes, sb)
    assert deq[0, 0] == 1.0 and deq[0, 1] == 0.3125 and deq[0, 2] == -0.5


def test_saturation_and_range():
    x = np.full((1, 32), 1.0)
    x[0, 5] = 500.0
    codes, sb = mx_quantize(x)
    assert sb[0, 0] == 127                              # floor(log2 500) = 8, E = 0
    assert codes[0, 5] == 0x7E                          # 448
    assert mx_dequantize(codes, sb)[0, 5] == 448.0


def test_invariants_on_random_rows():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((64, 128)) * np.exp2(rng.integers(-20, 20, size=(64, 1)))
    x[3, 40] = 20.0
    codes, sb = mx_quantize(x)
    assert codes.shape == x.shape and sb.shape == (64, 4)
    deq = mx_dequantize(codes, sb)
    e = sb.astype(np.float64) - 127
    for r in range(64):
        for b in range(4):
            blk = x[r, 32 * b:32 * b + 32]
            top = np.abs(blk).max() * np.exp2(-e[r, b])
            assert 256.0 <= top < 512.0                 # the largest value's binade after scaling
            err = np.abs(deq[r, 32 * b:32 * b + 32] - blk)
            bound = np.maximum(np.abs(blk) * 2.0 ** -4, 2.0 ** -10 * np.exp2(e[r, b])) * (1 + 1e-12)
            # values in [448, 512) after scaling saturate to 448 (the format's choice of E)
            bound = np.maximum(bound, np.abs(blk) - 448.0 * np.exp2(e[r, b]))
            assert np.all(err <= bound)
    y = x.copy()
    y[10, 70] *= 64.0
    _, sb2 = mx_quantize(y)
    changed = np.argwhere(sb2 != sb)
    assert all((r, b) == (10, 2) for r, b in changed)


def test_ties_subnormals_and_exponent_clamps():
    """Worked by hand. A block whose maximum is 256 has E = 0, so its other values
    are encoded as they are: 1.0625 lies halfway between 1.0 (0x38) and 1.125
    (0x39) and goes to the even mantissa, 1.0; 1.1875 lies halfway between 1.125
    and 1.25 (0x3A) and goes to 1.25; 3 * 2^-9 is the subnormal code 3; 2^-10 is
    halfway between 0 and the smallest subnormal 2^-9 and goes to 0; 3 * 2^-10 is
    halfway between codes 1 and 2 and goes to 2. A block whose maximum is 2^-125
    would need E = -133 and is clamped to E = -127 (byte 0), so 2^-125 is encoded
    as 4.0 (0x48); a block whose maximum is 1.5 * 2^127 has E = 119 (byte 246)
    and 384 (0x7C)."""
    x = np.zeros((1, 96))
    x[0, :6] = [256.0, 1.0625, 1.1875, 3 * 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -10]
    x[0, 32] = 2.0 ** -125
    x[0, 64] = 1.5 * 2.0 ** 127
    codes, sb = mx_quantize(x)
    assert sb.tolist() == [[127, 0, 246]]
    assert codes[0, :6].tolist() == [0x78, 0x38, 0x3A, 0x03, 0x00, 0x02]
    assert codes[0, 32] == 0x48 and codes[0, 64] == 0x7C
    deq = mx_dequantize(codes, sb)
    assert deq[0, 32] == 2.0 ** -125 and deq[0, 64] == 1.5 * 2.0 ** 127
