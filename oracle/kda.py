"""fp64 oracle of the KDA (per-channel gated) delta rule, token by token.

TEST INFRASTRUCTURE ONLY: the tests and the bench's CPU leg call it; the product path never
does.  It imports nothing from the CUDA library package.

The pages give the KDA gate only (MindSpeed-Ops "KDA gate" task: yg = -exp(A_log[h]) *
softplus(g + dt_bias), per (token, head, channel)) and name the KDA chunk kernels beside the
Gated DeltaNet ones (the G_T_CONTIG article lists the KDA chunk backward among the kernels that
read the gate along time).  The recurrence is taken as the Gated DeltaNet one with the scalar
decay of each value head replaced by that head's per-key-channel decay (the plainest reading
the pages support): for the state S (V x K) of value head hv,

    S_t = S_{t-1} Diag(exp(yg_t)) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,   o_t = scale S_t q_t,

yg_t[c] = -exp(A_log[hv]) softplus(g_t[hv, c] + dt_bias[hv*K + c]) for key channel c, the decay
applied before the erase as in the Gated DeltaNet path.  With a gate that is the same on every
channel it is exactly the Gated DeltaNet recurrence.

Layouts match the library's: q, k [B,T,H,K]; v, o [B,T,HV,V]; g_raw [B,T,HV,K]; beta [B,T,HV];
A_log [HV]; dt_bias [HV*K] or None; states [Nst,HV,K,V] with h[k][v] = S[v][k].

The backward (recurrent_bwd) is the plain reverse-mode derivative of that recurrence for
L = sum(dO * o) + sum(dht * h_final), taken token by token backwards over the stored states:
with S_d = S_{t-1} Diag(alpha_t), alpha_t = e^{yg_t}, e = S_d k_t, u = beta_t (v_t - e), S_t = S_d + u k_t^T,
    dS_t += scale dO_t q_t^T,   dq_t = scale S_t^T dO_t,
    du = dS_t k_t,   dk_t = dS_t^T u + S_d^T de,   dbeta_t = du . (v_t - e),   dv_t = beta_t du,
    de = -beta_t du,   dS_d = dS_t + de k_t^T,
    dyg_t[c] = alpha_t[c] sum_v dS_d[v, c] S_{t-1}[v, c],   dS_{t-1} = dS_d Diag(alpha_t),
and the gate chain of the KDA gate (oracle/kda_gate.bwd) from dyg to g_raw, A_log and dt_bias.
"""
from __future__ import annotations

import numpy as np

from . import kda_gate


def _f64(x):
    return kda_gate._f64(x)


def recurrent_fwd(q, k, v, g_raw, A_log, dt_bias, beta, scale=None, cu_seqlens=None, h0=None):
    """Returns (o [B,T,HV,V], h_final [Nst,HV,K,V]) in float64."""
    q, k, v, g_raw, A_log, dt_bias, beta, h0 = map(_f64, (q, k, v, g_raw, A_log, dt_bias, beta, h0))
    B, T, H, K = q.shape
    HV, V = v.shape[2], v.shape[3]
    G = HV // H
    if scale is None:
        scale = K ** -0.5
    yg = kda_gate.fwd(g_raw, A_log, dt_bias)  # [B,T,HV,K] log-decay per key channel
    if cu_seqlens is not None:
        cu = [int(x) for x in np.asarray(cu_seqlens)]
        spans = [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]
    else:
        spans = [(b, 0, T) for b in range(B)]
    o = np.zeros((B, T, HV, V))
    ht = np.zeros((len(spans), HV, K, V))
    kh = np.arange(HV) // G  # key head of each value head
    for n, (b, t0, t1) in enumerate(spans):
        S = np.zeros((HV, V, K)) if h0 is None else np.transpose(h0[n], (0, 2, 1)).copy()
        for t in range(t0, t1):
            kk, qq = k[b, t][kh], q[b, t][kh]                     # [HV, K]
            S *= np.exp(yg[b, t])[:, None, :]                     # decay column c of S
            e = np.einsum("hvk,hk->hv", S, kk)                    # S k
            S += (beta[b, t][:, None] * (v[b, t] - e))[:, :, None] * kk[:, None, :]
            o[b, t] = scale * np.einsum("hvk,hk->hv", S, qq)
        ht[n] = np.transpose(S, (0, 2, 1))
    return o, ht


def recurrent_bwd(q, k, v, g_raw, A_log, dt_bias, beta, dO, scale=None, cu_seqlens=None, h0=None,
                  dht=None):
    """Backward of L = sum(dO*o) + sum(dht*h_final).  Returns a dict (float64) with dq, dk
    [B,T,H,K]; dv [B,T,HV,V]; dbeta [B,T,HV]; dg (dL/dyg, the log-decay) and dg_raw [B,T,HV,K];
    dh0 [Nst,HV,K,V]; dA_log [HV]; ddt_bias [HV*K] (or None without dt_bias)."""
    q, k, v, g_raw, A_log, dt_bias, beta, dO, h0, dht = map(
        _f64, (q, k, v, g_raw, A_log, dt_bias, beta, dO, h0, dht))
    B, T, H, K = q.shape
    HV, V = v.shape[2], v.shape[3]
    G = HV // H
    if scale is None:
        scale = K ** -0.5
    yg = kda_gate.fwd(g_raw, A_log, dt_bias)
    alpha = np.exp(yg)
    if cu_seqlens is not None:
        cu = [int(x) for x in np.asarray(cu_seqlens)]
        spans = [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]
    else:
        spans = [(b, 0, T) for b in range(B)]
    kh = np.arange(HV) // G
    dq = np.zeros((B, T, H, K))
    dk = np.zeros((B, T, H, K))
    dv = np.zeros((B, T, HV, V))
    dbeta = np.zeros((B, T, HV))
    dyg = np.zeros((B, T, HV, K))
    dh0 = np.zeros((len(spans), HV, K, V))
    for n, (b, t0, t1) in enumerate(spans):
        S = np.zeros((HV, V, K)) if h0 is None else np.transpose(h0[n], (0, 2, 1)).copy()
        prev, dec, es = [], [], []
        for t in range(t0, t1):  # forward, keeping S_{t-1}, S_d and e of every token
            kk = k[b, t][kh]
            prev.append(S.copy())
            S = S * alpha[b, t][:, None, :]
            dec.append(S.copy())
            e = np.einsum("hvk,hk->hv", S, kk)
            es.append(e)
            S = S + (beta[b, t][:, None] * (v[b, t] - e))[:, :, None] * kk[:, None, :]
        dS = np.zeros((HV, V, K)) if dht is None else np.transpose(dht[n], (0, 2, 1)).copy()
        for idx in range(t1 - t0 - 1, -1, -1):
            t = t0 + idx
            kk, qq = k[b, t][kh], q[b, t][kh]
            Sd, Sp, e = dec[idx], prev[idx], es[idx]
            bt = beta[b, t]
            u = bt[:, None] * (v[b, t] - e)
            St = Sd + u[:, :, None] * kk[:, None, :]
            dS = dS + scale * dO[b, t][:, :, None] * qq[:, None, :]
            dqh = scale * np.einsum("hvk,hv->hk", St, dO[b, t])
            du = np.einsum("hvk,hk->hv", dS, kk)
            dkh = np.einsum("hvk,hv->hk", dS, u)
            dbeta[b, t] = np.sum(du * (v[b, t] - e), axis=1)
            dv[b, t] = bt[:, None] * du
            de = -bt[:, None] * du
            dkh = dkh + np.einsum("hvk,hv->hk", Sd, de)
            dSd = dS + de[:, :, None] * kk[:, None, :]
            dyg[b, t] = alpha[b, t] * np.sum(dSd * Sp, axis=1)
            dS = dSd * alpha[b, t][:, None, :]
            np.add.at(dq[b, t], kh, dqh)
            np.add.at(dk[b, t], kh, dkh)
        dh0[n] = np.transpose(dS, (0, 2, 1))
    dg_raw, dA_log, ddt = kda_gate.bwd(g_raw, A_log, dyg, dt_bias)
    return dict(dq=dq, dk=dk, dv=dv, dbeta=dbeta, dg=dyg, dg_raw=dg_raw, dh0=dh0, dA_log=dA_log,
                ddt_bias=ddt)
