"""fp64 numpy restatement of the chunkwise (64-token) algebra of the gated delta rule.

Test infrastructure: it is NOT the oracle (the oracle is the token-by-token recurrence in
oracle/gdn_oracle.cpp) and NOT the CUDA path.  It exists to pin, on the CPU, the exact
reassociation that the CUDA kernels implement (per chunk: A, T=(I+A)^-1, W, U~, the state
scan, the output, and every backward term) against the oracle, before any kernel runs.

Per chunk (tokens i=0..63, zero-padded past the sequence end with g=0, beta=0):
  G = inclusive cumsum of g;  Gam_ij = exp(G_i - G_j) for i >= j else 0
  A = strict_lower(diag(beta) (K K^T * Gam));   T = (I + A)^-1
  W = T diag(beta e^G) K;   U~ = T diag(beta) V;   U = U~ - W S^T
  O = scale (diag(e^G) Q S^T + (Q K^T * Gam) U)
  S' = e^{G_C} S + U^T diag(e^{G_C - G}) K           (G_C = G at the last position)
The backward mirrors these products term by term.

With affine=True the passes over the chunks take the form the sequential CUDA passes use:
the chunk step is affine in the state, so with D = diag(e^{G_C - G}) (zero past the chunk's
last token), N = W^T D K and B = U~^T D K (neither depends on the state):
  S' = e^{G_C} S + B - S N
  dS = e^{G_C} dS' - (W^T dU_loc - scale Q^T diag(e^G) dO + N dS'^T)^T,  dU_loc = scale P^T dO
"""
from __future__ import annotations

import numpy as np

C = 64


def _pad(x, n):
    out = np.zeros((C,) + x.shape[1:], dtype=np.float64)
    out[:n] = x
    return out


def _chunk_terms(Q, K, V, g, b):
    G = np.cumsum(g)
    idx = np.arange(C)
    low_incl = idx[:, None] >= idx[None, :]
    low_strict = idx[:, None] > idx[None, :]
    Gam = np.where(low_incl, np.exp(np.where(low_incl, G[:, None] - G[None, :], 0.0)), 0.0)
    KK = K @ K.T
    A = np.where(low_strict, b[:, None] * KK * Gam, 0.0)
    T = np.linalg.inv(np.eye(C) + A)
    X = (b * np.exp(G))[:, None] * K
    Y = b[:, None] * V
    W = T @ X
    Ut = T @ Y
    return G, Gam, A, T, X, Y, W, Ut, low_incl, low_strict


def fwd_unit(q, k, v, g, beta, S0, scale, affine=False):
    """q,k [L,K]; v [L,V]; g, beta [L]; S0 [V,K] (S orientation).  Returns o [L,V], S_final."""
    L = len(g)
    S = S0.copy()
    o = np.zeros((L, v.shape[1]))
    for c0 in range(0, L, C):
        n = min(C, L - c0)
        Q, K, V = _pad(q[c0:c0 + n], n), _pad(k[c0:c0 + n], n), _pad(v[c0:c0 + n], n)
        gg, bb = _pad(g[c0:c0 + n], n), _pad(beta[c0:c0 + n], n)
        G, Gam, A, T, X, Y, W, Ut, li, ls = _chunk_terms(Q, K, V, gg, bb)
        U = Ut - W @ S.T
        P = (Q @ K.T) * Gam
        O = scale * (np.exp(G)[:, None] * (Q @ S.T) + P @ U)
        o[c0:c0 + n] = O[:n]
        GC = G[-1]
        if affine:
            Dk = (np.exp(GC - G) * (np.arange(C) < n))[:, None] * K
            S = np.exp(GC) * S + Ut.T @ Dk - S @ (W.T @ Dk)
        else:
            S = np.exp(GC) * S + (U * np.exp(GC - G)[:, None]).T @ K
    return o, S


def bwd_unit(q, k, v, g, beta, S0, dO, dSfin, scale, affine=False):
    """Chunkwise backward.  Returns dq, dk, dv, dg, dbeta, dS0 for one (sequence, head)."""
    L = len(g)
    nck = (L + C - 1) // C
    # forward recompute: states entering each chunk
    S = S0.copy()
    saved = []
    for c in range(nck):
        c0 = c * C
        n = min(C, L - c0)
        Q, K, V = _pad(q[c0:c0 + n], n), _pad(k[c0:c0 + n], n), _pad(v[c0:c0 + n], n)
        gg, bb = _pad(g[c0:c0 + n], n), _pad(beta[c0:c0 + n], n)
        G, Gam, A, T, X, Y, W, Ut, li, ls = _chunk_terms(Q, K, V, gg, bb)
        U = Ut - W @ S.T
        saved.append((c0, n, Q, K, V, bb, G, Gam, A, T, X, Y, W, U, S.copy(), ls))
        GC = G[-1]
        S = np.exp(GC) * S + (U * np.exp(GC - G)[:, None]).T @ K
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dg = np.zeros_like(g)
    db = np.zeros_like(beta)
    dSn = dSfin.copy()
    for c in reversed(range(nck)):
        c0, n, Q, K, V, bb, G, Gam, A, T, X, Y, W, U, Sc, ls = saved[c]
        dOc = _pad(dO[c0:c0 + n], n)
        GC = G[-1]
        D = np.exp(GC - G)
        P = (Q @ K.T) * Gam
        # dv_local and the output-path terms
        dU = scale * P.T @ dOc + D[:, None] * (K @ dSn.T)
        dP = np.where(Gam > 0, scale * dOc @ U.T, 0.0) * (np.arange(C)[:, None] >= np.arange(C)[None, :])
        dPG = dP * Gam
        dQ = scale * np.exp(G)[:, None] * (dOc @ Sc) + dPG @ K
        dKc = dPG.T @ Q + D[:, None] * (U @ dSn)
        dW = -dU @ Sc
        dG = (dP * P).sum(1) - (dP * P).sum(0)
        dG += scale * np.exp(G) * ((dOc @ Sc) * Q).sum(1)
        r = ((U @ dSn) * K).sum(1) * D
        dG -= r
        dG[-1] += np.exp(GC) * (dSn * Sc).sum() + r.sum()
        # state chain
        if affine:
            live = (np.arange(C) < n)
            Dk = (D * live)[:, None] * K
            acc = W.T @ (scale * P.T @ dOc) + Q.T @ (-scale * (np.exp(G) * live)[:, None] * dOc) \
                + (W.T @ Dk) @ dSn.T
            dS = np.exp(GC) * dSn - acc.T
        else:
            dS = np.exp(GC) * dSn + scale * (np.exp(G)[:, None] * dOc).T @ Q - dU.T @ W
        # WY backward
        dT = dU @ Y.T + dW @ X.T
        dX = T.T @ dW
        dY = T.T @ dU
        dA = np.where(ls, -(T.T @ dT @ T.T), 0.0)
        dVc = bb[:, None] * dY
        dbc = (dY * V).sum(1) + np.exp(G) * (dX * K).sum(1) + (dA * Gam * (K @ K.T)).sum(1)
        dAs = dA * Gam * bb[:, None]
        dKc += (bb * np.exp(G))[:, None] * dX + dAs @ K + dAs.T @ K
        dG += bb * np.exp(G) * (dX * K).sum(1) + (dA * A).sum(1) - (dA * A).sum(0)
        dgc = np.cumsum(dG[::-1])[::-1]
        dq[c0:c0 + n] = dQ[:n]
        dk[c0:c0 + n] = dKc[:n]
        dv[c0:c0 + n] = dVc[:n]
        dg[c0:c0 + n] = dgc[:n]
        db[c0:c0 + n] = dbc[:n]
        dSn = dS
    return dq, dk, dv, dg, db, dSn
