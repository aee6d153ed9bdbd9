"""The polynomial 2^x that the kernels evaluate on the FMA pipe (part of the
softmax exponentials): constants equal the Remez fit, and an fp32 emulation of
the kernel's exact steps (round via 1.5*2^23, Horner in fp32 with FMA, exponent
add) stays within the fit's relative-error bound plus fp32 rounding."""
import os
import re
import sys

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "exact_attention_forward_11_b200",
                    "csrc")
sys.path.insert(0, CSRC)
import fit_exp2_poly  # noqa: E402


def kernel_constants():
    text = open(os.path.join(CSRC, "attn_fwd_kernel.cuh")).read()
    return [float(re.search(rf"kExp2C{i} = ([0-9.e+-]+)f;", text).group(1)) for i in range(4)]


def emulate(x):
    """fp32 emulation of exp2_poly_x2 (fma emulated in fp64, exact for fp32 inputs
    up to one final rounding)."""
    f32 = np.float32
    c = [f32(v) for v in kernel_constants()]
    x = np.maximum(x.astype(np.float32), f32(-125.0))
    magic = f32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x.astype(np.float64) - n).astype(np.float32)
    fma = lambda a, b, cc: (a.astype(np.float64) * b + cc).astype(np.float32)  # noqa: E731
    q = fma(f, np.float32(c[3]), np.float32(c[2]))
    q = fma(q, f, np.float32(c[1]))
    q = fma(q, f, np.float32(c[0]))
    bits = q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_constants_match_fit():
    coeffs, bound = fit_exp2_poly.remez()
    assert bound < 8e-5
    np.testing.assert_array_equal(np.float32(kernel_constants()), np.float32(coeffs))


def test_fp32_evaluation_within_bound():
    x = np.concatenate([np.linspace(-124.9, 8.0, 2_000_001), np.arange(-124, 9).astype(np.float64),
                        np.arange(-124, 9) + 0.5]).astype(np.float32)
    got = emulate(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 7.48e-5 + 4e-7, rel.max()


def test_clamp_gives_tiny_normal_for_minus_inf():
    got = emulate(np.array([-np.inf, -1e30, -200.0], dtype=np.float32))
    assert np.all(got > 0) and np.all(got < 1e-37)
    assert np.all(np.isfinite(got))
