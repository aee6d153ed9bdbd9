"""Pins for the fp64 attention oracle, independent of the oracle's own code.

Each check is chosen so that a plausible slip in the oracle (a dropped scale, a
wrong sign, a transposed operand, an off-by-one causal mask, log base 2 instead of
e, a missing normalisation) fails at least one of them:
  * hand-derived golden cases (tests/golden/attention_hand.json);
  * a pure-Python brute force with explicit loops and math.exp on tiny shapes;
  * closed forms: one key, identical keys, zero queries;
  * invariants: rows of P sum to 1, convexity, LSE bounds, orthogonal invariance,
    key/value permutation equivariance, linearity in V, one-hot dominance;
  * blocked online softmax (the tiled recurrence of "Self-Attention, CUDA kernels
    and FlashAttention", §3, online-softmax bullet) equals the materialised result.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import attention_fp64, attention_probs_fp64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(12345)


def brute_force(q, k, v, scale, causal):
    """Explicit loops over rows, keys and channels; math.exp; no numpy algebra."""
    N, d = len(q), len(q[0])
    dv = len(v[0])
    O, L = [], []
    for i in range(N):
        keys = [j for j in range(N) if (not causal) or j <= i]
        s = []
        for j in keys:
            acc = 0.0
            for t in range(d):
                acc += q[i][t] * k[j][t]
            s.append(scale * acc)
        mx = max(s)
        w = [math.exp(x - mx) for x in s]
        tot = sum(w)
        row = []
        for c in range(dv):
            acc = 0.0
            for w_j, j in zip(w, keys):
                acc += w_j * v[j][c]
            row.append(acc / tot)
        O.append(row)
        L.append(mx + math.log(tot))
    return np.array(O), np.array(L)


@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLDEN, "attention_hand.json")))["cases"],
                         ids=lambda c: c["name"])
@pytest.mark.parametrize("causal", [False, True])
def test_golden_hand_cases(case, causal):
    q, k, v = (np.array(case[n], dtype=np.float64)[None] for n in ("q", "k", "v"))
    o, lse = attention_fp64(q, k, v, case["scale"], causal=causal)
    exp = case["causal" if causal else "noncausal"]
    np.testing.assert_allclose(o[0], np.array(exp["o"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0], np.array(exp["lse"]), rtol=0, atol=1e-12)


@pytest.mark.parametrize("N", [1, 2, 3, 17, 40])
@pytest.mark.parametrize("d", [1, 4, 9])
@pytest.mark.parametrize("causal", [False, True])
def test_brute_force_tiny(N, d, causal):
    q = RNG.standard_normal((N, d))
    k = RNG.standard_normal((N, d))
    v = RNG.standard_normal((N, d))
    scale = 0.7 / math.sqrt(d)
    o, lse = attention_fp64(q[None], k[None], v[None], scale, causal)
    ob, lb = brute_force(q.tolist(), k.tolist(), v.tolist(), scale, causal)
    np.testing.assert_allclose(o[0], ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0], lb, rtol=0, atol=1e-12)


def test_brute_force_vit_rows():
    """A ViT-sized head (N=196, d=64) against the brute force on a few rows."""
    N, d = 196, 64
    q, k, v = (RNG.standard_normal((N, d)) for _ in range(3))
    scale = 1 / 8
    rows = [0, 1, 127, 128, 195]
    o, lse = attention_fp64(q[None], k[None], v[None], scale, False, rows=rows)
    ob, lb = brute_force(q.tolist(), k.tolist(), v.tolist(), scale, False)
    np.testing.assert_allclose(o[0], ob[rows], atol=1e-12)
    np.testing.assert_allclose(lse[0], lb[rows], atol=1e-12)


def test_single_key_returns_v():
    d = 8
    q, k, v = (RNG.standard_normal((1, 1, d)) for _ in range(3))
    o, lse = attention_fp64(q, k, v, 0.3, False)
    np.testing.assert_allclose(o[0, 0], v[0, 0], atol=1e-15)
    np.testing.assert_allclose(lse[0, 0], 0.3 * float(q[0, 0] @ k[0, 0]), atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_identical_keys_give_mean_of_v(causal):
    N, d = 37, 5
    q = RNG.standard_normal((N, d))
    krow = RNG.standard_normal(d)
    k = np.tile(krow, (N, 1))
    v = RNG.standard_normal((N, d))
    scale = 0.9
    o, lse = attention_fp64(q[None], k[None], v[None], scale, causal)
    for i in range(N):
        cnt = i + 1 if causal else N
        np.testing.assert_allclose(o[0, i], v[:cnt].mean(axis=0), atol=1e-12)
        np.testing.assert_allclose(lse[0, i], scale * q[i] @ krow + math.log(cnt), atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_and_zero_scale(causal):
    N, d = 23, 6
    k, v = RNG.standard_normal((N, d)), RNG.standard_normal((N, d))
    for q, scale in ((np.zeros((N, d)), 0.5), (RNG.standard_normal((N, d)), 0.0)):
        o, lse = attention_fp64(q[None], k[None], v[None], scale, causal)
        for i in range(N):
            cnt = i + 1 if causal else N
            np.testing.assert_allclose(o[0, i], v[:cnt].mean(axis=0), atol=1e-12)
            np.testing.assert_allclose(lse[0, i], math.log(cnt), atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_probability_rows_sum_to_one(causal):
    """Rows of the materialised P sum to 1 ("Self-Attention, CUDA kernels and
    FlashAttention", §1, softmax paragraph), and that P is the one behind the
    oracle's outputs: P V equals attention_fp64's O and ln P_ij + LSE_i equals
    the score S_ij written out with explicit loops (a dropped scale or a
    transposed product in either function fails here)."""
    B, H, N, d = 2, 3, 50, 16
    q, k, v = (RNG.standard_normal((B, H, N, d)) for _ in range(3))
    scale = 0.25
    p = attention_probs_fp64(q, k, scale, causal)
    np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-13)
    assert (p >= 0).all()
    if causal:
        assert np.all(np.triu(p[0, 0], 1) == 0)
    o, lse = attention_fp64(q, k, v, scale, causal)
    np.testing.assert_allclose(np.einsum("bhij,bhjc->bhic", p, v), o, rtol=0, atol=1e-12)
    for b, h, i, j in ((0, 0, 3, 1), (1, 2, 49, 0), (1, 1, 20, 20), (0, 2, 7, 30)):
        if causal and j > i:
            assert p[b, h, i, j] == 0.0
            continue
        s_ij = scale * sum(q[b, h, i, t] * k[b, h, j, t] for t in range(d))
        assert abs(math.log(p[b, h, i, j]) + lse[b, h, i] - s_ij) <= 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_convexity_and_lse_bounds(causal):
    B, H, N, d = 1, 2, 70, 12
    q, k, v = (RNG.standard_normal((B, H, N, d)) * 3 for _ in range(3))
    scale = 1 / math.sqrt(d)
    o, lse = attention_fp64(q, k, v, scale, causal)
    for h in range(H):
        for i in range(N):
            cnt = i + 1 if causal else N
            vis = v[0, h, :cnt]
            assert np.all(o[0, h, i] >= vis.min(0) - 1e-12)
            assert np.all(o[0, h, i] <= vis.max(0) + 1e-12)
            smax = (scale * k[0, h, :cnt] @ q[0, h, i]).max()
            assert smax - 1e-12 <= lse[0, h, i] <= smax + math.log(cnt) + 1e-12


def test_orthogonal_rotation_invariance():
    """(Q R)(K R)^T = Q K^T for orthogonal R, the identity behind incoherent
    processing ("FlashAttention scaling, multi-GPU training and weight
    quantization", §1, FlashAttention-3 FP8 bullet)."""
    from workloads import make_rotation
    d = 32
    rot, _ = make_rotation(d, 5)
    rot = rot.numpy()
    np.testing.assert_allclose(rot @ rot.T, np.eye(d), atol=1e-13)
    q, k, v = (RNG.standard_normal((1, 2, 40, d)) for _ in range(3))
    o1, l1 = attention_fp64(q, k, v, 0.2, False)
    o2, l2 = attention_fp64(q @ rot, k @ rot, v, 0.2, False)
    np.testing.assert_allclose(o1, o2, atol=1e-10)
    np.testing.assert_allclose(l1, l2, atol=1e-10)


def test_permutation_equivariance_and_linearity():
    N, d = 31, 7
    q, k, v, v2 = (RNG.standard_normal((1, 1, N, d)) for _ in range(4))
    perm = RNG.permutation(N)
    o, lse = attention_fp64(q, k, v, 0.4, False)
    op, lp = attention_fp64(q, k[:, :, perm], v[:, :, perm], 0.4, False)
    np.testing.assert_allclose(o, op, atol=1e-12)
    np.testing.assert_allclose(lse, lp, atol=1e-12)
    # permuting queries permutes outputs
    oq, lq = attention_fp64(q[:, :, perm], k, v, 0.4, False)
    np.testing.assert_allclose(oq, o[:, :, perm], atol=1e-12)
    # linear in V
    a, b = 1.7, -0.3
    o2, _ = attention_fp64(q, k, v2, 0.4, False)
    olin, _ = attention_fp64(q, k, a * v + b * v2, 0.4, False)
    np.testing.assert_allclose(olin, a * o + b * o2, atol=1e-12)


def test_one_hot_dominance():
    N, d = 20, 16
    q, k, v = (RNG.standard_normal((N, d)) for _ in range(3))
    i, j = 7, 13
    k[j] = 50.0 * q[i] / np.linalg.norm(q[i])
    o, _ = attention_fp64(q[None], k[None], v[None], 1.0, False)
    np.testing.assert_allclose(o[0, i], v[j], atol=1e-9)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 127, 128, 129, 300])
def test_blocked_online_softmax_equals_materialised(N, causal):
    """Tile-by-tile online softmax with a running max and normaliser and the
    division by the normaliser deferred to the end ("FlashAttention scaling,
    multi-GPU training and weight quantization", §1, FlashAttention-2 bullet on
    non-matmul work) equals the materialised oracle. This pins the recurrence
    the kernels implement before any kernel exists."""
    d, BLK = 16, 128
    q, k, v = (RNG.standard_normal((N, d)) for _ in range(3))
    scale = 0.3
    o_ref, l_ref = attention_fp64(q[None], k[None], v[None], scale, causal)
    o = np.zeros((N, d))
    m = np.full(N, -np.inf)
    l = np.zeros(N)
    for j0 in range(0, N, BLK):
        s = scale * q @ k[j0:j0 + BLK].T
        if causal:
            keys = np.arange(j0, min(N, j0 + BLK))
            s = np.where(keys[None, :] <= np.arange(N)[:, None], s, -np.inf)
        m_new = np.maximum(m, s.max(1))
        alpha = np.exp(m - m_new)
        p = np.exp(s - m_new[:, None])
        l = alpha * l + p.sum(1)
        o = alpha[:, None] * o + p @ v[j0:j0 + BLK]
        m = m_new
    o = o / l[:, None]
    np.testing.assert_allclose(o, o_ref[0], atol=1e-12)
    np.testing.assert_allclose(m + np.log(l), l_ref[0], atol=1e-12)


def test_row_sampling_matches_full():
    q, k, v = (RNG.standard_normal((2, 2, 300, 8)) for _ in range(3))
    o, lse = attention_fp64(q, k, v, 0.5, True)
    rows = [0, 5, 128, 299]
    os_, ls = attention_fp64(q, k, v, 0.5, True, rows=rows, panel=3)
    # the GEMM library may block differently for other panel shapes: fp64 rounding only
    np.testing.assert_allclose(os_, o[:, :, rows], atol=1e-13)
    np.testing.assert_allclose(ls, lse[:, :, rows], atol=1e-13)
