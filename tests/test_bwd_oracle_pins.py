"""Pins for the fp64 backward oracle (oracle/attention_bwd.py), independent of its code.

Each check is chosen so that a plausible slip (a dropped scale, D taken from the
wrong rows, dS transposed, a missing causal mask on dS, dK from Q^T dS instead
of dS^T Q) fails at least one of them:
  * central finite differences of the pinned forward oracle (the loss
    L = sum O * G for a fixed G, so dL/dO = G);
  * a pure-Python brute force with explicit loops on tiny shapes;
  * closed forms: one key (dQ = dK = 0, dV = dO), identical keys (dQ = 0),
    causal row 0 (dQ_0 = 0);
  * invariants: sum_j dK_j = 0, sum_j dV_j = sum_i dO_i, linearity in dO, and
    under a causal mask the last key's gradients depend on the last query only.
"""
import math

import numpy as np
import pytest

from oracle import attention_fp64
from oracle.attention_bwd import attention_bwd_fp64

RNG = np.random.default_rng(2718)


def _loss(q, k, v, g, scale, causal):
    o, _ = attention_fp64(q, k, v, scale, causal)
    return float((o * g).sum())


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(1, 3), (5, 3), (7, 4)])
def test_finite_differences(N, d, causal):
    q, k, v, g = (RNG.standard_normal((1, 1, N, d)) for _ in range(4))
    scale = 0.6
    dq, dk, dv = attention_bwd_fp64(q, k, v, g, scale, causal)
    eps = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args = {"q": q, "k": k, "v": v}
            lp = _loss(**{**args, name: xp}, g=g, scale=scale, causal=causal)
            lm = _loss(**{**args, name: xm}, g=g, scale=scale, causal=causal)
            num[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(grad, num, rtol=0, atol=2e-8, err_msg=name)


def brute_force(q, k, v, do, scale, causal):
    """Explicit loops: P row by row, then every gradient entry from its sum."""
    N, d = len(q), len(q[0])
    P = [[0.0] * N for _ in range(N)]
    for i in range(N):
        keys = [j for j in range(N) if (not causal) or j <= i]
        s = {j: scale * sum(q[i][t] * k[j][t] for t in range(d)) for j in keys}
        mx = max(s.values())
        z = sum(math.exp(x - mx) for x in s.values())
        for j in keys:
            P[i][j] = math.exp(s[j] - mx) / z
    O = [[sum(P[i][j] * v[j][c] for j in range(N)) for c in range(d)] for i in range(N)]
    dP = [[sum(do[i][c] * v[j][c] for c in range(d)) for j in range(N)] for i in range(N)]
    D = [sum(do[i][c] * O[i][c] for c in range(d)) for i in range(N)]
    dS = [[P[i][j] * (dP[i][j] - D[i]) for j in range(N)] for i in range(N)]
    dq = [[scale * sum(dS[i][j] * k[j][c] for j in range(N)) for c in range(d)] for i in range(N)]
    dk = [[scale * sum(dS[i][j] * q[i][c] for i in range(N)) for c in range(d)] for j in range(N)]
    dv = [[sum(P[i][j] * do[i][c] for i in range(N)) for c in range(d)] for j in range(N)]
    return np.array(dq), np.array(dk), np.array(dv)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(2, 1), (4, 2), (9, 5), (17, 3)])
def test_brute_force(N, d, causal):
    q, k, v, do = (RNG.standard_normal((N, d)) for _ in range(4))
    scale = 0.45
    got = attention_bwd_fp64(q[None], k[None], v[None], do[None], scale, causal)
    want = brute_force(q.tolist(), k.tolist(), v.tolist(), do.tolist(), scale, causal)
    for g, w in zip(got, want):
        np.testing.assert_allclose(g[0], w, rtol=0, atol=1e-12)


def test_single_key():
    q, k, v, do = (RNG.standard_normal((1, 1, 1, 6)) for _ in range(4))
    dq, dk, dv = attention_bwd_fp64(q, k, v, do, 0.3, False)
    assert np.abs(dq).max() == 0 and np.abs(dk).max() == 0
    np.testing.assert_allclose(dv, do, atol=1e-15)


@pytest.mark.parametrize("causal", [False, True])
def test_identical_keys_give_zero_dq(causal):
    N, d = 12, 4
    q, v, do = (RNG.standard_normal((1, 1, N, d)) for _ in range(3))
    k = np.tile(RNG.standard_normal(d), (1, 1, N, 1))
    dq, _, _ = attention_bwd_fp64(q, k, v, do, 0.8, causal)
    np.testing.assert_allclose(dq, 0.0, atol=1e-13)


def test_causal_row_zero_and_last_key():
    N, d = 10, 3
    q, k, v, do = (RNG.standard_normal((1, 1, N, d)) for _ in range(4))
    dq, dk, dv = attention_bwd_fp64(q, k, v, do, 0.5, True)
    np.testing.assert_allclose(dq[0, 0, 0], 0.0, atol=1e-15)     # row 0 sees key 0 only
    # the last key is seen by the last query only: earlier queries do not move its gradients
    q2, do2 = q.copy(), do.copy()
    q2[0, 0, :N - 1] = RNG.standard_normal((N - 1, d))
    do2[0, 0, :N - 1] = RNG.standard_normal((N - 1, d))
    _, dk2, dv2 = attention_bwd_fp64(q2, k, v, do2, 0.5, True)
    np.testing.assert_allclose(dk2[0, 0, N - 1], dk[0, 0, N - 1], atol=1e-13)
    np.testing.assert_allclose(dv2[0, 0, N - 1], dv[0, 0, N - 1], atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_sum_invariants_and_linearity(causal):
    B, H, N, d = 2, 2, 23, 5
    q, k, v, do, do2 = (RNG.standard_normal((B, H, N, d)) for _ in range(5))
    dq, dk, dv = attention_bwd_fp64(q, k, v, do, 0.4, causal)
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)           # rows of dS sum to 0
    np.testing.assert_allclose(dv.sum(axis=2), do.sum(axis=2), atol=1e-12)  # rows of P sum to 1
    a, b = 0.7, -1.3
    g1 = attention_bwd_fp64(q, k, v, do2, 0.4, causal)
    gl = attention_bwd_fp64(q, k, v, a * do + b * do2, 0.4, causal)
    for x, y, z in zip((dq, dk, dv), g1, gl):
        np.testing.assert_allclose(z, a * x + b * y, atol=1e-12)


def test_row_selection():
    q, k, v, do = (RNG.standard_normal((1, 2, 40, 4)) for _ in range(4))
    dq, dk, dv = attention_bwd_fp64(q, k, v, do, 0.5, True)
    dqs, dks, dvs = attention_bwd_fp64(q, k, v, do, 0.5, True, rows=[0, 7, 39])
    np.testing.assert_array_equal(dqs, dq[:, :, [0, 7, 39]])
    np.testing.assert_array_equal(dks, dk)


def test_given_output_enters_through_d_only():
    """With o = the exact O the result is unchanged; a perturbed o changes only
    D, so dV is untouched and dQ moves by exactly -scale * dD_i * (P K)_i."""
    N, d = 9, 4
    q, k, v, do = (RNG.standard_normal((1, 1, N, d)) for _ in range(4))
    scale = 0.5
    o, _ = attention_fp64(q, k, v, scale, False)
    base = attention_bwd_fp64(q, k, v, do, scale, False)
    same = attention_bwd_fp64(q, k, v, do, scale, False, o=o)
    for a, b in zip(base, same):
        np.testing.assert_allclose(a, b, atol=1e-14)
    delta = RNG.standard_normal(o.shape) * 1e-3
    dq2, _, dv2 = attention_bwd_fp64(q, k, v, do, scale, False, o=o + delta)
    np.testing.assert_allclose(dv2, base[2], atol=1e-15)
    dd = (do * delta).sum(-1)                                    # change of D_i
    pk, _ = attention_fp64(q, k, k, scale, False)                # (P K)_i
    np.testing.assert_allclose(dq2 - base[0], -scale * dd[..., None] * pk, atol=1e-13)
