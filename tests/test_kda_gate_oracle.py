"""CPU pins of the KDA-gate oracle (oracle/kda_gate.py), each against something other than
the oracle's own formula: closed-form softplus values, the Gated DeltaNet gate of the C++
oracle (an independent implementation of the same per-element map), torch's softplus with
threshold 20 (a library routine), and central finite differences for the backward."""
from __future__ import annotations

import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import kda_gate, oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "gate_softplus.txt")


def _golden():
    rows = [l.split() for l in open(GOLDEN) if l.strip() and not l.startswith("#")]
    return np.array([[float(a), float(b)] for a, b in rows])


def test_softplus_closed_forms():
    xs, sp = _golden().T
    np.testing.assert_allclose(kda_gate.softplus20(xs), sp, rtol=1e-15, atol=0)


def test_forward_matches_gdn_gate_of_the_cpp_oracle():
    """With D = 1 the KDA gate of head h is the Gated DeltaNet gate of value head h."""
    rng = np.random.default_rng(5)
    T, H = 37, 6
    a = rng.standard_normal((1, T, H)) * 8.0
    A_log = np.log(rng.uniform(1, 16, H))
    dt_bias = rng.standard_normal(H) * 0.5
    got = kda_gate.fwd(a.reshape(T, H, 1), A_log, dt_bias).reshape(T, H)
    for h in range(H):
        ref = oracle.gate(a[0, :, h], float(A_log[h]), float(dt_bias[h]))
        np.testing.assert_allclose(got[:, h], ref, rtol=1e-14, atol=1e-300)


def test_forward_matches_torch_softplus_threshold_20():
    rng = np.random.default_rng(6)
    g = rng.standard_normal((9, 4, 24)) * 15.0
    A_log = rng.standard_normal(4)
    dt_bias = rng.standard_normal(4 * 24)
    ref = (-torch.tensor(A_log).exp().view(4, 1)
           * F.softplus(torch.tensor(g) + torch.tensor(dt_bias).view(4, 24), threshold=20.0))
    np.testing.assert_allclose(kda_gate.fwd(g, A_log, dt_bias), ref.numpy(), rtol=1e-13, atol=1e-300)
    # no bias
    ref0 = -torch.tensor(A_log).exp().view(4, 1) * F.softplus(torch.tensor(g), threshold=20.0)
    np.testing.assert_allclose(kda_gate.fwd(g, A_log), ref0.numpy(), rtol=1e-13, atol=1e-300)


@pytest.mark.parametrize("with_bias", [True, False])
def test_backward_matches_central_differences(with_bias):
    rng = np.random.default_rng(7)
    T, H, D = 5, 3, 4
    g = rng.standard_normal((T, H, D)) * 6.0
    g[0, 0, :2] = [20.5, 30.0]  # the pass-through branch
    A_log = rng.standard_normal(H)
    dt_bias = rng.standard_normal(H * D) if with_bias else None
    w = rng.standard_normal((T, H, D))  # L = sum(w * yg)
    dg, dA, ddt = kda_gate.bwd(g, A_log, w, dt_bias)
    L = lambda gg, AA, bb: float((w * kda_gate.fwd(gg, AA, bb)).sum())
    eps = 1e-6
    for idx in [(0, 0, 0), (0, 0, 2), (3, 2, 1), (4, 1, 3)]:
        gp, gm = g.copy(), g.copy()
        gp[idx] += eps
        gm[idx] -= eps
        fd = (L(gp, A_log, dt_bias) - L(gm, A_log, dt_bias)) / (2 * eps)
        assert abs(fd - dg[idx]) <= 1e-6 * max(1.0, abs(fd)), (idx, fd, dg[idx])
    for h in range(H):
        ap, am = A_log.copy(), A_log.copy()
        ap[h] += eps
        am[h] -= eps
        fd = (L(g, ap, dt_bias) - L(g, am, dt_bias)) / (2 * eps)
        assert abs(fd - dA[h]) <= 1e-6 * max(1.0, abs(fd)), (h, fd, dA[h])
    if with_bias:
        for c in [0, 5, H * D - 1]:
            bp, bm = dt_bias.copy(), dt_bias.copy()
            bp[c] += eps
            bm[c] -= eps
            fd = (L(g, A_log, bp) - L(g, A_log, bm)) / (2 * eps)
            assert abs(fd - ddt[c]) <= 1e-6 * max(1.0, abs(fd)), (c, fd, ddt[c])
    else:
        assert ddt is None
