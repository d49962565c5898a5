"""Chunkwise rewrite of the gated delta rule, in float64 numpy — TEST INFRASTRUCTURE ONLY.

This exists for one purpose: to pin the token-by-token recurrence in
``kda_oracle.c`` against an algebraically equivalent blocked form (its
"chunked rewrite" self-check).  It is never used to produce expected values for
the GPU and shares nothing with the CUDA path.

Derivation (per head; chunk of C tokens starting from state S0; i, j index
tokens inside the chunk; every product below is over the key channel c):

    G_i   = sum_{s<=i} g_s                     cumulative log-decay, per channel
    u_i   = beta_i (v_i - (Diag(exp g_i) S_{i-1})^T k_i)
    S_i   = Diag(exp G_i) S0 + sum_{j<=i} Diag(exp(G_i - G_j)) k_j u_j^T

Substituting S_{i-1} into u_i gives the lower-triangular system

    (I + A) U = Diag(beta) (V - (exp(G) * K) S0),
    A[i, j]   = beta_i * sum_c k_i[c] k_j[c] exp(G_i[c] - G_j[c])      (j < i)

so with T = (I + A)^{-1} Diag(beta), W = T (exp(G) * K) and U~ = T V:

    U     = U~ - W S0
    O     = (exp(G) * Q) S0 + P U,   P[i, j] = sum_c q_i[c] k_j[c] exp(G_i[c] - G_j[c])  (j <= i)
    S_C   = Diag(exp G_C) S0 + (exp(G_C - G) * K)^T U

Small inputs only: the pairwise exponentials are formed directly (no
overflow protection), which is fine for the gentle gates the self-check uses.
"""
from __future__ import annotations

import numpy as np


def _chunk_step(q, k, v, g, beta, S0):
    """One chunk for one head.  q, k, g: [C, dk]; v: [C, dv]; beta: [C]; S0: [dk, dv]."""
    C = q.shape[0]
    G = np.cumsum(g, axis=0)                                   # [C, dk]
    diff = G[:, None, :] - G[None, :, :]                       # G_i - G_j, [C, C, dk]
    with np.errstate(over="ignore", invalid="ignore"):
        decay = np.where(np.tril(np.ones((C, C), bool))[:, :, None], np.exp(diff), 0.0)
    A = beta[:, None] * np.einsum("ic,jc,ijc->ij", k, k, decay)
    A = np.tril(A, -1)
    P = np.einsum("ic,jc,ijc->ij", q, k, decay)                # j <= i by construction
    Tm = np.linalg.solve(np.eye(C) + A, np.diag(beta))         # (I + A)^{-1} Diag(beta)
    Gam = np.exp(G)
    W = Tm @ (Gam * k)
    Ut = Tm @ v
    U = Ut - W @ S0
    O = (Gam * q) @ S0 + P @ U
    S = np.exp(G[-1])[:, None] * S0 + (np.exp(G[-1][None, :] - G) * k).T @ U
    return O, S


def chunked(q, k, v, g, beta, s0=None, chunk=64):
    """Same signature and result as ``oracle.recurrent`` (up to rounding), computed chunkwise."""
    q, k, v, g, beta = (np.asarray(a, dtype=np.float64) for a in (q, k, v, g, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    sT = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if s0 is None else np.array(s0[b, h], dtype=np.float64)
            for t0 in range(0, T, chunk):
                t1 = min(T, t0 + chunk)
                O, S = _chunk_step(q[b, t0:t1, h], k[b, t0:t1, h], v[b, t0:t1, h],
                                   g[b, t0:t1, h], beta[b, t0:t1, h], S)
                o[b, t0:t1, h] = O
            sT[b, h] = S
    return o, sT
