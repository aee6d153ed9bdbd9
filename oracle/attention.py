"""fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference leg may import or call anything under oracle/. The
product path (the CUDA library and its Python binding) never does.

What it computes is the plain definition, written out with the full score matrix
materialised in fp64 (numpy; the matrix products are library GEMMs):

  S_ij  = scale * sum_t Q_it K_jt                 ("Self-Attention, CUDA kernels and
                                                     FlashAttention", §1, eq. Scores)
  causal: S_ij = -inf for j > i                    (reading: square, top-left
                                                     aligned mask; the pages do not
                                                     define the mask)
  P_i   = softmax_j(S_ij), rows sum to 1           (same page, §1, softmax weighting
                                                     paragraph)
  O_i   = sum_j P_ij V_j                           (same page, §1, eq. Attention)
  LSE_i = ln sum_j exp(S_ij)                        (same page, §3, recompute bullet:
                                                     the forward keeps only the small
                                                     per-row normalisation statistics;
                                                     reading: natural log, scale
                                                     included)

Each (batch, head) is independent (same page, §1, multi-head paragraph). Rows are
processed in panels of at most `panel` rows only to bound memory: softmax is
row-wise, so a panel computes exactly the arithmetic the full matrix would for
those rows. `rows=` restricts the computation to chosen query rows (the same
per-row arithmetic), which is how full-size workloads are sampled.

Pinned by tests/test_oracle_pins.py (brute force, closed forms, invariants).
"""
from __future__ import annotations

import numpy as np


def _as_bhnd(x):
    x = np.asarray(x, dtype=np.float64)
    if x.ndim == 3:
        return x[None], True
    if x.ndim != 4:
        raise ValueError("expected [B,H,N,d] or [H,N,d]")
    return x, False


def attention_fp64(q, k, v, scale, causal=False, rows=None, panel=1024):
    """Exact attention forward in fp64.

    q, k, v: arrays [B, H, N, d] (or [H, N, d]); any real dtype, read as fp64.
    scale:   the multiplier of Q K^T (the pages' 1/sqrt(d_k)).
    causal:  key j is visible to query i iff j <= i.
    rows:    optional sorted iterable of query rows; if given, only those rows are
             computed and O has shape [B, H, len(rows), d], LSE [B, H, len(rows)].
    Returns (O, LSE) as fp64 arrays.
    """
    q, squeeze = _as_bhnd(q)
    k, _ = _as_bhnd(k)
    v, _ = _as_bhnd(v)
    B, H, N, d = q.shape
    if k.shape != (B, H, N, d) or v.shape[:3] != (B, H, N):
        raise ValueError("q, k, v shapes disagree")
    row_idx = np.arange(N) if rows is None else np.asarray(list(rows), dtype=np.int64)
    R = row_idx.shape[0]
    dv = v.shape[3]
    out = np.empty((B, H, R, dv), dtype=np.float64)
    lse = np.empty((B, H, R), dtype=np.float64)
    keys = np.arange(N)
    for b in range(B):
        for h in range(H):
            kt = k[b, h].T
            vv = v[b, h]
            for p0 in range(0, R, panel):
                ridx = row_idx[p0:p0 + panel]
                s = scale * (q[b, h, ridx] @ kt)                 # [r, N] scores
                if causal:
                    s = np.where(keys[None, :] <= ridx[:, None], s, -np.inf)
                m = s.max(axis=1, keepdims=True)                 # row max
                e = np.exp(s - m)                                # unnormalised weights
                l = e.sum(axis=1, keepdims=True)                 # row normaliser
                out[b, h, p0:p0 + panel] = (e @ vv) / l
                lse[b, h, p0:p0 + panel] = (m + np.log(l))[:, 0]
    if squeeze:
        return out[0], lse[0]
    return out, lse


def attention_probs_fp64(q, k, scale, causal=False):
    """The materialised probability matrix P = softmax(scale Q K^T) per (b, h),
    shape [..., N, N]. Small inputs only (used to check that rows sum to 1)."""
    q, squeeze = _as_bhnd(q)
    k, _ = _as_bhnd(k)
    N = q.shape[2]
    s = scale * np.einsum("bhid,bhjd->bhij", q, k)
    if causal:
        mask = np.tril(np.ones((N, N), dtype=bool))
        s = np.where(mask, s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    p = e / e.sum(axis=-1, keepdims=True)
    return p[0] if squeeze else p
