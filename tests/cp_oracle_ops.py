"""Test infrastructure: the per-rank computations of the context-parallel module done by the
fp64 oracle on the CPU (float64 torch tensors), so the exchange and fold logic can be run on
CPU ranks.  Not a product path."""
from __future__ import annotations

import numpy as np
import torch

from oracle import oracle


def _t(x):
    return torch.from_numpy(np.ascontiguousarray(x))


class OracleOps:
    def fwd(self, q, k, v, g_raw, A_log, dt_bias, beta, h0, workspace=None):
        o, ht, _ = oracle.fwd(q, k, v, g_raw, A_log, dt_bias, beta, h0=h0)
        return _t(o), _t(ht)

    def bwd(self, q, k, v, g_raw, A_log, dt_bias, beta, h0, d_o, dht, workspace):
        g = oracle.bwd(q, k, v, g_raw, A_log, dt_bias, beta, d_o, h0=h0, dht=dht)
        g["dg_raw"] = g.pop("da")
        return {k_: _t(v_) for k_, v_ in g.items()}

    def affine(self, A, X, B=None, transpose=False):
        A = A.transpose(-1, -2) if transpose else A
        out = torch.matmul(A.double(), X.double())
        return out + B.double() if B is not None else out

    def workspace(self, q, v):
        return None
