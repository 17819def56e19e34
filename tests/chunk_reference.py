"""fp64 numpy chunk form of the KDA recurrence -- test infrastructure (a debug reference).

This is NOT the oracle (the oracle is the sequential loop in ``oracle/kda_oracle.c``).  It writes out
the chunk-parallel algebra that the CUDA path implements, in plain numpy, so that the tests can show
on the CPU that the algebra is an identity (it reproduces the oracle to rounding) before any kernel is
trusted.  It shares no code with the CUDA path.

Per chunk of C tokens (positions r = 0..C-1), with lambda = max(log_alpha, ln 0.0067) and the
chunk-local inclusive cumsum g:
  A[r,s]   = beta_r sum_c k_rc k_sc exp(g_rc - g_sc)      (s < r; strictly lower)
  Aqk[r,s] = sum_c q_rc k_sc exp(g_rc - g_sc)             (s <= r)
  X        = (I + A)^-1                                    (blocked forward substitution, 16x16 tiles)
  W = X diag(beta) (K * exp(g)),  U = X diag(beta) V,  U' = U - W S
  O = (Q * exp(g)) S + Aqk U'
  S <- Diag(exp(g_C)) S + (K * exp(g_C - g))^T U'
The products exp(g_r - g_s) are formed through a 16-token tile anchor b (the cumulative log-decay just
before the row's tile): exp(g_r - b) * exp(b - g_s).  The floor keeps exp(b - g_s) <= exp(-16 ln 0.0067)
inside one tile, which is the fact that lets diagonal tiles use the same dense product as the others
(orkas.ai "Kimi K3 architecture" post, section "GPU 코드 경로 하나를 없앤 하한").
"""
from __future__ import annotations

import math

import numpy as np

LOG_FLOOR = math.log(0.0067)


def blocked_unit_lower_inverse(A: np.ndarray, tile: int = 16) -> np.ndarray:
    """(I + A)^-1 for strictly lower A by blocked forward substitution on tile x tile blocks.

    Diagonal blocks are inverted by row-wise forward substitution; an off-diagonal block is
    X_ij = -X_ii sum_{j <= m < i} A_im X_mj.
    """
    n = A.shape[0]
    nb = (n + tile - 1) // tile
    X = np.zeros((n, n))
    sl = [slice(b * tile, min(n, (b + 1) * tile)) for b in range(nb)]
    for b in range(nb):
        Ab = A[sl[b], sl[b]]
        m = Ab.shape[0]
        Xb = np.zeros((m, m))
        for r in range(m):
            row = np.zeros(m)
            row[r] = 1.0
            for s in range(r):
                row -= Ab[r, s] * Xb[s]
            Xb[r] = row
        X[sl[b], sl[b]] = Xb
    for d in range(1, nb):
        for i in range(d, nb):
            j = i - d
            acc = np.zeros((X[sl[i], sl[i]].shape[0], X[sl[j], sl[j]].shape[0]))
            for m in range(j, i):
                acc += A[sl[i], sl[m]] @ X[sl[m], sl[j]]
            X[sl[i], sl[j]] = -X[sl[i], sl[i]] @ acc
    return X


def chunk_forward(q, k, v, log_alpha, beta, s0=None, C=64, tile=16, want_transition=False):
    q = np.asarray(q, np.float64); k = np.asarray(k, np.float64); v = np.asarray(v, np.float64)
    lam = np.maximum(np.asarray(log_alpha, np.float64), LOG_FLOOR)
    beta = np.asarray(beta, np.float64)
    T, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if s0 is None else np.array(s0, np.float64)
    M = np.eye(dk) if want_transition else None
    O = np.zeros((T, dv))
    for c0 in range(0, T, C):
        c1 = min(T, c0 + C)
        n = c1 - c0
        g = np.cumsum(lam[c0:c1], axis=0)
        Kc, Qc, Vc, Bc = k[c0:c1], q[c0:c1], v[c0:c1], beta[c0:c1]
        A = np.zeros((n, n))
        Aqk = np.zeros((n, n))
        for i0 in range(0, n, tile):
            i1 = min(n, i0 + tile)
            b = g[i0 - 1] if i0 > 0 else np.zeros(dk)
            left_k = Kc[i0:i1] * np.exp(g[i0:i1] - b)
            left_q = Qc[i0:i1] * np.exp(g[i0:i1] - b)
            right = Kc[:i1] * np.exp(b - g[:i1])     # <= exp(80.09) inside the row's own tile
            A[i0:i1, :i1] = left_k @ right.T
            Aqk[i0:i1, :i1] = left_q @ right.T
        A = np.tril(A, -1) * Bc[:, None]
        Aqk = np.tril(Aqk, 0)
        X = blocked_unit_lower_inverse(A, tile)
        W = X @ (Bc[:, None] * Kc * np.exp(g))
        U = X @ (Bc[:, None] * Vc)
        Up = U - W @ S
        O[c0:c1] = (Qc * np.exp(g)) @ S + Aqk @ Up
        Kdec = Kc * np.exp(g[-1] - g)
        S = np.exp(g[-1])[:, None] * S + Kdec.T @ Up
        if M is not None:
            M = np.exp(g[-1])[:, None] * M - Kdec.T @ (W @ M)
    return (O, S, M) if want_transition else (O, S)
