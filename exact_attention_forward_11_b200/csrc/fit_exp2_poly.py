"""Fits the polynomial the kernels use to evaluate 2^x on the FMA pipe.

Method: Cody & Waite style argument reduction, x = n + f with n = round(x) and
f in [-1/2, 1/2]; 2^x = 2^n * p(f), where p is the degree-3 polynomial that
minimises the maximum RELATIVE error |p(f) / 2^f - 1| on [-1/2, 1/2], found with
the Remez exchange algorithm (equioscillation on 5 reference points). The scale
2^n is applied by adding n to the exponent field of p(f).

    python fit_exp2_poly.py     # prints the coefficients and the error bound

The coefficients are written into attn_fwd_kernel.cuh (kExp2Poly*); a CPU test
checks that they match this fit and that the fp32 evaluation stays within the
bound.
"""
import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez(degree=DEGREE, iters=30):
    n = degree + 2
    # Chebyshev extrema as the initial reference
    k = np.arange(n)
    ref = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i for coefficients and E
        A = np.zeros((n, n))
        for i, x in enumerate(ref):
            A[i, :degree + 1] = x ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** ref)
        c = sol[:degree + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: extrema of the error, one per sign alternation
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        idx = np.array(idx)
        # keep the n largest alternating extrema
        cand = sorted(idx, key=lambda i: -abs(err[i]))
        chosen = []
        for i in sorted(cand[: 4 * n]):
            if not chosen or np.sign(err[i]) != np.sign(err[chosen[-1]]):
                chosen.append(i)
            elif abs(err[i]) > abs(err[chosen[-1]]):
                chosen[-1] = i
        if len(chosen) < n:
            break
        # choose the contiguous window of n alternating points with the largest minimum
        best = max(range(len(chosen) - n + 1), key=lambda s: min(abs(err[chosen[s:s + n]])))
        ref = grid[chosen[best:best + n]]
    err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    coeffs, bound = remez()
    c32 = np.asarray(coeffs, dtype=np.float32)
    for i, v in enumerate(c32):
        print(f"c{i} = {float(v)!r}  ({float(v).hex()})")
    print(f"max relative error (exact arithmetic): {bound:.3e}")
