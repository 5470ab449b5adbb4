"""fp64 numpy restatement of the chunkwise (64-token) algebra of the KDA delta rule (a decay per
key channel), in the sub-chunk form the CUDA kernels implement.

Test infrastructure: it is NOT the oracle (that is the token-by-token recurrence in
oracle/kda.py) and NOT the CUDA path.  It pins, on the CPU, the reassociation the kernels use.

Per chunk (tokens i = 0..63, padded past the sequence end with yg = 0, beta = 0), for one value
head with state S (V x K) entering the chunk:
  Gam_i = inclusive cumsum of yg_i over the chunk (a K-vector per token, <= 0, decreasing)
  Kt_i = k_i * e^{Gam_i},  Qt_i = q_i * e^{Gam_i},  Kh_i = k_i * e^{Gam_C - Gam_i}     (all factors <= 1)
  A_ij = beta_i sum_c k_i[c] k_j[c] e^{Gam_i[c] - Gam_j[c]}   (j < i),   T = (I + A)^-1
  P_ij =        sum_c q_i[c] k_j[c] e^{Gam_i[c] - Gam_j[c]}   (j <= i)
  W = T diag(beta) Kt,  U~ = T diag(beta) V,  U = U~ - W S^T
  O = scale (Qt S^T + P U),   S' = S Diag(e^{Gam_C}) + U^T Kh
A and P are taken in 16-token sub-chunks: for i in sub-chunk a and j in an earlier sub-chunk,
e^{Gam_i - Gam_j} = e^{Gam_i - Gam_r} e^{Gam_r - Gam_j} with r the last token before sub-chunk a,
both factors <= 1, so the block is a plain product of two rescaled key/query tiles; inside a
sub-chunk the per-channel exponentials of differences are summed directly (a factored form
would need e^{-Gam_j}, which overflows fp32 within a few tokens at strong decay).
"""
from __future__ import annotations

import numpy as np

C = 64
SUB = 16


def _gate(g, A_log, dt_bias):
    x = g + (0.0 if dt_bias is None else dt_bias)
    sp = np.where(x > 20, x, np.log1p(np.exp(np.minimum(x, 20.0))))
    return -np.exp(A_log) * sp


def intra(Qc, Kc, Gam, b):
    """A (strict lower) and P (lower incl. diagonal) of one chunk, sub-chunk form."""
    A = np.zeros((C, C))
    P = np.zeros((C, C))
    for a in range(C // SUB):
        ia = slice(a * SUB, (a + 1) * SUB)
        if a > 0:
            r = a * SUB - 1
            left_k = Kc[ia] * np.exp(Gam[ia] - Gam[r])
            left_q = Qc[ia] * np.exp(Gam[ia] - Gam[r])
            right = Kc[:a * SUB] * np.exp(Gam[r] - Gam[:a * SUB])
            A[ia, :a * SUB] = b[ia, None] * (left_k @ right.T)
            P[ia, :a * SUB] = left_q @ right.T
        for i in range(a * SUB, (a + 1) * SUB):
            for j in range(a * SUB, i + 1):
                e = np.exp(Gam[i] - Gam[j])
                if j < i:
                    A[i, j] = b[i] * np.sum(Kc[i] * Kc[j] * e)
                P[i, j] = np.sum(Qc[i] * Kc[j] * e)
    return A, P


def fwd_unit(Qc, Kc, Vc, ygc, b, S, scale):
    """One chunk: returns (O [C,V], S_next [V,K], U [C,V])."""
    Gam = np.cumsum(ygc, axis=0)
    A, P = intra(Qc, Kc, Gam, b)
    T = np.linalg.inv(np.eye(C) + A)
    W = T @ (b[:, None] * Kc * np.exp(Gam))
    Ut = T @ (b[:, None] * Vc)
    U = Ut - W @ S.T
    O = scale * ((Qc * np.exp(Gam)) @ S.T + P @ U)
    Sn = S * np.exp(Gam[-1])[None, :] + U.T @ (Kc * np.exp(Gam[-1] - Gam))
    return O, Sn, U


def forward(q, k, v, g_raw, A_log, dt_bias, beta, scale=None, h0=None):
    """Dense batch only: q, k [B,T,H,K], v [B,T,HV,V], g_raw [B,T,HV,K]; states [B,HV,K,V]."""
    q, k, v, g_raw, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g_raw, beta))
    A_log = np.asarray(A_log, dtype=np.float64)
    B, T, H, K = q.shape
    HV, V = v.shape[2], v.shape[3]
    G = HV // H
    if scale is None:
        scale = K ** -0.5
    dtb = None if dt_bias is None else np.asarray(dt_bias, dtype=np.float64).reshape(HV, K)
    o = np.zeros((B, T, HV, V))
    ht = np.zeros((B, HV, K, V))
    for bb in range(B):
        for hv in range(HV):
            S = np.zeros((V, K)) if h0 is None else np.asarray(h0[bb, hv], dtype=np.float64).T.copy()
            yg = _gate(g_raw[bb, :, hv], A_log[hv], None if dtb is None else dtb[hv])
            for c0 in range(0, T, C):
                n = min(C, T - c0)
                pad = lambda x: np.concatenate([x, np.zeros((C - n,) + x.shape[1:])]) if n < C else x
                Qc, Kc = pad(q[bb, c0:c0 + n, hv // G]), pad(k[bb, c0:c0 + n, hv // G])
                Vc, ygc, b = pad(v[bb, c0:c0 + n, hv]), pad(yg[c0:c0 + n]), pad(beta[bb, c0:c0 + n, hv])
                O, S, _ = fwd_unit(Qc, Kc, Vc, ygc, b, S, scale)
                o[bb, c0:c0 + n, hv] = O[:n]
            ht[bb, hv] = S.T
    return o, ht


def gated_rows(Wt, R, Gam):
    """F_i = sum_{j <= i} Wt_ij R_j e^{Gam_i - Gam_j}  (per channel), sub-chunk form."""
    F = np.zeros_like(R)
    for a in range(C // SUB):
        ia = slice(a * SUB, (a + 1) * SUB)
        if a > 0:
            r = a * SUB - 1
            RT = R[:a * SUB] * np.exp(Gam[r] - Gam[:a * SUB])
            F[ia] += np.exp(Gam[ia] - Gam[r]) * (Wt[ia, :a * SUB] @ RT)
        for i in range(a * SUB, (a + 1) * SUB):
            for j in range(a * SUB, i + 1):
                F[i] += Wt[i, j] * R[j] * np.exp(Gam[i] - Gam[j])
    return F


def gated_cols(Wt, L, Gam):
    """G_j = sum_{i >= j} Wt_ij L_i e^{Gam_i - Gam_j}  (per channel), sub-chunk form."""
    Gm = np.zeros_like(L)
    for a in range(C // SUB):
        ia = slice(a * SUB, (a + 1) * SUB)
        if a > 0:
            r = a * SUB - 1
            Ls = L[ia] * np.exp(Gam[ia] - Gam[r])
            Gm[:a * SUB] += np.exp(Gam[r] - Gam[:a * SUB]) * (Wt[ia, :a * SUB].T @ Ls)
        for i in range(a * SUB, (a + 1) * SUB):
            for j in range(a * SUB, i + 1):
                Gm[j] += Wt[i, j] * L[i] * np.exp(Gam[i] - Gam[j])
    return Gm


def bwd_unit(Qc, Kc, Vc, ygc, b, S, dO, dSn, scale):
    """One chunk backward: returns (dQ, dK, dV, db, dyg, dS_entering) for loss
    sum(dO * O) + sum(dSn * S_next), S (V x K) the state entering the chunk."""
    Gam = np.cumsum(ygc, axis=0)
    A, P = intra(Qc, Kc, Gam, b)
    T = np.linalg.inv(np.eye(C) + A)
    eG, eC = np.exp(Gam), np.exp(Gam[-1])
    Kt, Qt, Kh = Kc * eG, Qc * eG, Kc * np.exp(Gam[-1] - Gam)
    X, Y = b[:, None] * Kt, b[:, None] * Vc
    W, Ut = T @ X, T @ Y
    U = Ut - W @ S.T
    # scan part
    dU = scale * P.T @ dO + Kh @ dSn.T
    dS = dSn * eC[None, :] + scale * dO.T @ Qt - dU.T @ W
    # output and state products
    dQt = scale * dO @ S
    dP = np.tril(scale * dO @ U.T)
    dKh = U @ dSn
    dW = -dU @ S
    dGam = dQt * Qt - dKh * Kh
    dGamC = np.sum(dKh * Kh, axis=0) + np.sum(dSn * S, axis=0) * eC
    dQ = dQt * eG
    dK = dKh * np.exp(Gam[-1] - Gam)
    # P_ij = sum_c q_i k_j e^{Gam_i - Gam_j}
    F2 = gated_rows(dP, Kc, Gam)
    G2 = gated_cols(dP, Qc, Gam)
    dQ += F2
    dK += G2
    dGam += Qc * F2 - Kc * G2
    # WY part
    dT = dW @ X.T + dU @ Y.T
    dX, dY = T.T @ dW, T.T @ dU
    dV = b[:, None] * dY
    db = np.sum(dY * Vc, axis=1) + np.sum(dX * Kt, axis=1)
    dKt = b[:, None] * dX
    dK += dKt * eG
    dGam += dKt * Kt
    dA = np.tril(-T.T @ dT @ T.T, -1)
    # A_ij = b_i sum_c k_i k_j e^{Gam_i - Gam_j}
    F1 = gated_rows(dA, Kc, Gam)              # without b
    G1 = gated_cols(b[:, None] * dA, Kc, Gam)
    db += np.sum(Kc * F1, axis=1)
    dK += b[:, None] * F1 + G1
    dGam += b[:, None] * Kc * F1 - Kc * G1
    dGam[-1] += dGamC
    dyg = np.cumsum(dGam[::-1], axis=0)[::-1]
    return dQ, dK, dV, db, dyg, dS


def backward(q, k, v, g_raw, A_log, dt_bias, beta, dO, scale=None, h0=None, dht=None):
    """Dense batch: dq, dk, dv, dbeta, dyg (dL/dlog-decay, [B,T,HV,K]), dh0."""
    q, k, v, g_raw, beta, dO = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g_raw, beta, dO))
    A_log = np.asarray(A_log, dtype=np.float64)
    B, T, H, K = q.shape
    HV, V = v.shape[2], v.shape[3]
    G = HV // H
    if scale is None:
        scale = K ** -0.5
    dtb = None if dt_bias is None else np.asarray(dt_bias, dtype=np.float64).reshape(HV, K)
    out = dict(dq=np.zeros((B, T, H, K)), dk=np.zeros((B, T, H, K)), dv=np.zeros((B, T, HV, V)),
               dbeta=np.zeros((B, T, HV)), dg=np.zeros((B, T, HV, K)), dh0=np.zeros((B, HV, K, V)))
    for bb in range(B):
        for hv in range(HV):
            yg = _gate(g_raw[bb, :, hv], A_log[hv], None if dtb is None else dtb[hv])
            S = np.zeros((V, K)) if h0 is None else np.asarray(h0[bb, hv], dtype=np.float64).T.copy()
            chunks, states = [], []
            for c0 in range(0, T, C):
                n = min(C, T - c0)
                pad = lambda x, n=n: np.concatenate([x, np.zeros((C - n,) + x.shape[1:])]) if n < C else x
                ch = (pad(q[bb, c0:c0 + n, hv // G]), pad(k[bb, c0:c0 + n, hv // G]),
                      pad(v[bb, c0:c0 + n, hv]), pad(yg[c0:c0 + n]), pad(beta[bb, c0:c0 + n, hv]),
                      pad(dO[bb, c0:c0 + n, hv]), c0, n)
                chunks.append(ch)
                states.append(S)
                _, S, _ = fwd_unit(ch[0], ch[1], ch[2], ch[3], ch[4], S, scale)
            dS = np.zeros((V, K)) if dht is None else np.asarray(dht[bb, hv], dtype=np.float64).T.copy()
            for (Qc, Kc, Vc, ygc, bc, dOc, c0, n), S0 in zip(chunks[::-1], states[::-1]):
                dQ, dK, dV, db, dyg, dS = bwd_unit(Qc, Kc, Vc, ygc, bc, S0, dOc, dS, scale)
                out["dq"][bb, c0:c0 + n, hv // G] += dQ[:n]
                out["dk"][bb, c0:c0 + n, hv // G] += dK[:n]
                out["dv"][bb, c0:c0 + n, hv] = dV[:n]
                out["dbeta"][bb, c0:c0 + n, hv] = db[:n]
                out["dg"][bb, c0:c0 + n, hv] = dyg[:n]
            out["dh0"][bb, hv] = dS.T
    return out
