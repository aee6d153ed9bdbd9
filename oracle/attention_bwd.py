"""fp64 CPU oracle for the backward pass of exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference leg may import or call anything under oracle/. The
product path (the CUDA library and its Python binding) never does.

The forward keeps only O and the per-row normalisation statistic LSE so that the
backward pass can recompute the attention weights tile by tile instead of storing
the N x N matrix ("Self-Attention, CUDA kernels and FlashAttention", §3,
recompute bullet). What the backward computes is the gradient of a loss L(O)
through O = softmax(S) V, S = scale Q K^T ("Self-Attention, CUDA kernels and
FlashAttention", §1, eq. Scores and eq. Attention), given dO = dL/dO. Written
out with the full matrices in fp64 (numpy; the products are library GEMMs):

  S   = scale Q K^T, causal: S_ij = -inf for j > i
  P   = row-softmax(S)
  O   = P V
  dV  = P^T dO
  dP  = dO V^T
  D_i = sum_c dO_ic O_ic            (= sum_j P_ij dP_ij)
  dS  = P * (dP - D)                (softmax Jacobian applied row by row)
  dQ  = scale dS K
  dK  = scale dS^T Q

Reading: LSE is the statistic the forward saved, not a differentiated output, so
the backward takes dO only (no gradient flows into LSE). D is formed from the
forward output O; the backward receives that O as an input (at the library's
boundary it is the bf16 O the forward wrote), so `o=` lets a caller give the O
that D is taken from, exactly as the method receives it; by default the exact O
is recomputed.

Pinned by tests/test_bwd_oracle_pins.py (central finite differences of the forward
oracle, a pure-Python brute force, closed forms, invariants).
"""
from __future__ import annotations

import numpy as np

from .attention import _as_bhnd


def attention_bwd_fp64(q, k, v, do, scale, causal=False, rows=None, o=None):
    """Gradients (dQ, dK, dV) of L with dL/dO = do, in fp64.

    q, k, v, do: arrays [B, H, N, d] (or [H, N, d]); read as fp64.
    rows: optional iterable of query rows; if given, dQ is computed for those
          rows only (shape [B, H, len(rows), d]); dK and dV need every row and
          are returned in full.
    o:    optional forward output [B, H, N, d] that D_i = dO_i . O_i is taken
          from (default: the exact O recomputed here).
    Returns (dq, dk, dv) as fp64 arrays.
    """
    q, squeeze = _as_bhnd(q)
    k, _ = _as_bhnd(k)
    v, _ = _as_bhnd(v)
    do, _ = _as_bhnd(do)
    o_in = None if o is None else _as_bhnd(o)[0]
    B, H, N, d = q.shape
    if k.shape != (B, H, N, d) or v.shape[:3] != (B, H, N) or do.shape != v.shape:
        raise ValueError("q, k, v, do shapes disagree")
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    keys = np.arange(N)
    for b in range(B):
        for h in range(H):
            s = scale * (q[b, h] @ k[b, h].T)                       # [N, N]
            if causal:
                s = np.where(keys[None, :] <= keys[:, None], s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            p = e / e.sum(axis=1, keepdims=True)                    # rows sum to 1
            o_bh = p @ v[b, h]
            dv[b, h] = p.T @ do[b, h]
            dp = do[b, h] @ v[b, h].T
            o_d = o_bh if o_in is None else o_in[b, h]
            dd = (do[b, h] * o_d).sum(axis=1, keepdims=True)        # D_i
            ds = p * (dp - dd)
            dq[b, h] = scale * (ds @ k[b, h])
            dk[b, h] = scale * (ds.T @ q[b, h])
    if rows is not None:
        dq = dq[:, :, np.asarray(list(rows), dtype=np.int64)]
    if squeeze:
        return dq[0], dk[0], dv[0]
    return dq, dk, dv
