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
