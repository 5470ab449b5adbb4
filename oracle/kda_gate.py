"""fp64 oracle of the KDA gate (per-channel gate) and of its backward.

TEST INFRASTRUCTURE ONLY: the tests and the bench's CPU leg call it; the product path never
does.  It imports nothing from the CUDA library package.

The operation, as the "KDA gate" task of the MindSpeed-Ops issue tracker defines it
(sections on the formula and the computation flow): for g [..., H, D], A_log [H] and an
optional dt_bias [H*D] (viewed as [H, D]),
    yg = -exp(A_log[h]) * softplus(g + dt_bias[h, d]),   softplus(x) = x if x > 20 else log(1 + e^x).
The backward is its plain derivative for a loss L(yg) with dyg = dL/dyg:
    dg        = dyg * (-exp(A_log[h])) * (x > 20 ? 1 : sigmoid(x)),   x = g + dt_bias
    dA_log[h] = sum over every element of head h of dyg * yg          (d(-e^A)/dA = -e^A)
    ddt_bias  = sum over the leading (token) dims of dg.
Everything in float64 numpy; inputs of any float dtype are widened exactly.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def softplus20(x):
    """Stable softplus with the strict x > 20 pass-through."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 20.0, x, np.log1p(np.exp(np.minimum(x, 20.0))))


def fwd(g, A_log, dt_bias=None):
    """yg (float64, the shape of g)."""
    g, A_log, dt_bias = _f64(g), _f64(A_log), _f64(dt_bias)
    H, D = g.shape[-2:]
    x = g + (dt_bias.reshape(H, D) if dt_bias is not None else 0.0)
    return -np.exp(A_log).reshape(H, 1) * softplus20(x)


def bwd(g, A_log, dyg, dt_bias=None):
    """(dg, dA_log, ddt_bias or None), float64."""
    g, A_log, dyg, dt_bias = _f64(g), _f64(A_log), _f64(dyg), _f64(dt_bias)
    H, D = g.shape[-2:]
    x = g + (dt_bias.reshape(H, D) if dt_bias is not None else 0.0)
    nexp = -np.exp(A_log).reshape(H, 1)
    dsp = np.where(x > 20.0, 1.0, 1.0 / (1.0 + np.exp(-np.minimum(x, 50.0))))
    dg = dyg * nexp * dsp
    yg = nexp * softplus20(x)
    lead = tuple(range(g.ndim - 2))
    dA = (dyg * yg).sum(axis=lead).sum(axis=-1)
    ddt = dg.sum(axis=lead).reshape(H * D) if dt_bias is not None else None
    return dg, dA, ddt
