"""Pins for the W4A16 oracle (oracle/w4a16.py), worked by hand from its definition.

  * a packed word worked by hand: nibble slot i holds weight k = PERM[i];
  * dequantisation values worked by hand, including a product that must round
    to nearest even in fp16 (a plain fp32 or an exact product would differ);
  * the GEMM against a pure-Python brute force on a tiny shape;
  * one-hot activations select weight rows exactly;
  * a transposed or un-interleaved unpacking changes the result (the golden
    word catches it).
"""
import math

import numpy as np

from oracle.w4a16 import GROUP, dequantize_weights, unpack_int4, w4a16_gemm_fp64


def test_golden_word():
    # slots 0..7 hold the values 0..7 (0x76543210): weight k = PERM[slot] gets the slot's value,
    # so k = 0..7 read 0, 4, 1, 5, 2, 6, 3, 7
    qw = np.array([[0x76543210]], dtype=np.uint32).view(np.int32)
    assert unpack_int4(qw)[:, 0].tolist() == [0, 4, 1, 5, 2, 6, 3, 7]
    # 0xF in the top slot (k = 7): the sign bit of the int32 word must not leak
    qw = np.array([[0xF0000000]], dtype=np.uint32).view(np.int32)
    assert unpack_int4(qw)[:, 0].tolist() == [0, 0, 0, 0, 0, 0, 0, 15]


def _one_group(q_col, s, z):
    """Pack 128 codes (one group, one column) by hand from the definition."""
    words = []
    for w in range(GROUP // 8):
        v = 0
        for i, k in enumerate((0, 2, 4, 6, 1, 3, 5, 7)):
            v |= int(q_col[8 * w + k]) << (4 * i)
        words.append(v)
    qw = np.array(words, dtype=np.uint32).view(np.int32).reshape(-1, 1)
    return qw, np.array([[s]], dtype=np.float16), np.array([[z]], dtype=np.uint8)


def test_golden_dequantisation():
    q = np.zeros(GROUP, dtype=np.int64)
    q[0], q[1], q[2], q[127] = 9, 0, 11, 15
    w = dequantize_weights(*_one_group(q, 0.5, 8))[:, 0]
    assert w[0] == 0.5 and w[1] == -4.0 and w[2] == 1.5 and w[127] == 3.5
    # s = 1 + 2^-10, q - z = 3: the exact product 3 + 3 * 2^-10 lies halfway between
    # the fp16 neighbours 3 + 2^-9 (odd significand) and 3 + 2^-8 (even): rounds to 3 + 2^-8
    q[5] = 11
    w = dequantize_weights(*_one_group(q, 1.0009765625, 8))[:, 0]
    assert float(w[5]) == 3.00390625
    assert w.dtype == np.float16


def test_gemm_against_brute_force():
    rng = np.random.default_rng(4)
    M, K, N = 3, 256, 5
    q = rng.integers(0, 16, size=(K, N))
    z = rng.integers(0, 16, size=(K // GROUP, N))
    s = (rng.random((K // GROUP, N)) * 0.05 + 0.001).astype(np.float16)
    words = np.zeros((K // 8, N), dtype=np.int64)
    for n in range(N):
        for w in range(K // 8):
            v = 0
            for i, k in enumerate((0, 2, 4, 6, 1, 3, 5, 7)):
                v |= int(q[8 * w + k, n]) << (4 * i)
            words[w, n] = v
    qw = words.astype(np.uint32).view(np.int32)
    x = rng.standard_normal((M, K)).astype(np.float16)
    y = w4a16_gemm_fp64(x, qw, s, z.astype(np.uint8))
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                wk = float(np.float16(float(q[k, n] - z[k // GROUP, n]) * float(s[k // GROUP, n])))
                acc += float(x[m, k]) * wk
            assert math.isclose(y[m, n], acc, rel_tol=0, abs_tol=1e-9), (m, n)


def test_one_hot_rows_select_weights():
    rng = np.random.default_rng(8)
    K, N = 256, 16
    qw = rng.integers(-2**31, 2**31, size=(K // 8, N), dtype=np.int64).astype(np.int32)
    s = (rng.random((K // GROUP, N)) + 0.5).astype(np.float16)
    z = rng.integers(0, 16, size=(K // GROUP, N)).astype(np.uint8)
    x = np.zeros((4, K), dtype=np.float16)
    rows = [0, 7, 128, 255]
    for m, k in enumerate(rows):
        x[m, k] = 1.0
    y = w4a16_gemm_fp64(x, qw, s, z)
    np.testing.assert_array_equal(y, dequantize_weights(qw, s, z)[rows].astype(np.float64))
