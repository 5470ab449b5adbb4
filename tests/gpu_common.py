"""Helpers of the GPU parity tests: run a seeded case through the C-ABI binding and
through the fp64 oracle, and compare with the tolerances of the workloads:
  fp32 tensors: max abs error <= 1e-4 on every output;
  bf16 tensors (fp32 accumulation): o and final state relative L2 <= 5e-3 and
  max abs <= 2e-2; every gradient relative L2 <= 1e-2   (rel L2 = |x-ref|_2 / |ref|_2).
The two parameter gradients that are sums over all tokens, dA_log = sum_t dg_t g_t and
ddt_bias = sum_t dg_t c_t (c_t = -exp(A_log) softplus'(x_t)), inherit their bf16 bound
from dg's by Cauchy-Schwarz: |error| <= 1e-2 |dg|_2 |w|_2 per value head (w = g or c).
These sums cancel heavily on the workloads (sum|dg g| / |sum dg g| ~ 500), so a relative
bound of their own would ask dg for ~2e-5 accuracy.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import oracle
from gated_deltanet_chunkwise_chunk_b200 import synth

FP32_MAX_ABS = 1e-4
BF16_OUT_REL_L2 = 5e-3
BF16_OUT_MAX_ABS = 2e-2
BF16_GRAD_REL_L2 = 1e-2

GRADS = ("dq", "dk", "dv", "dg", "dbeta", "dh0", "dg_raw", "dA_log", "ddt_bias")


def to_dev(case: synth.Case, dev="cuda"):
    t = lambda x: None if x is None else x.to(dev).contiguous()
    return dict(q=t(case.q), k=t(case.k), v=t(case.v), g_raw=t(case.a), A_log=t(case.A_log),
                dt_bias=t(case.dt_bias), beta=t(case.beta), cu_seqlens=t(case.cu_seqlens),
                initial_state=t(case.h0))


def run_gpu(case: synth.Case, backward=True):
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    d = to_dev(case)
    o, ht = gdn.gdn_chunk_fwd(**d)
    out = dict(o=o, ht=ht)
    if backward:
        g = gdn.gdn_chunk_bwd(**d, d_o=case.dO.cuda(), dht=None if case.dht is None else case.dht.cuda())
        out.update(g)
    torch.cuda.synchronize()
    return {k: v.detach().double().cpu().numpy() for k, v in out.items() if v is not None}


def run_oracle(case: synth.Case, backward=True):
    cu = None if case.cu_seqlens is None else case.cu_seqlens.numpy()
    o, ht, g = oracle.fwd(case.q, case.k, case.v, case.a, case.A_log, case.dt_bias, case.beta,
                          cu_seqlens=cu, h0=case.h0)
    out = dict(o=o, ht=ht, _g=g)
    x = case.a.double().numpy() + case.dt_bias.double().numpy()
    sp1 = np.where(x > 20, 1.0, 1.0 / (1.0 + np.exp(-np.minimum(x, 50.0))))
    out["_c"] = -np.exp(case.A_log.double().numpy()) * sp1
    if backward:
        g = oracle.bwd(case.q, case.k, case.v, case.a, case.A_log, case.dt_bias, case.beta,
                       case.dO, cu_seqlens=cu, h0=case.h0, dht=case.dht)
        g["dg_raw"] = g.pop("da")
        out.update(g)
    return out


def rel_l2(x, ref):
    n = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / n) if n > 0 else float(np.linalg.norm(x))


def compare(gpu: dict, ref: dict, dtype: str, select=None, keys=None):
    """Returns a list of failures (empty = parity).  ``select`` maps output name -> index
    function applied to the GPU result before comparing (for sampled heads)."""
    fails, report = [], {}
    for k in (keys or ref.keys()):
        if k not in gpu or k.startswith("_"):
            continue
        x = gpu[k] if select is None or k not in select else select[k](gpu[k])
        r = ref[k]
        assert x.shape == r.shape, (k, x.shape, r.shape)
        mx = float(np.abs(x - r).max()) if r.size else 0.0
        rl = rel_l2(x, r)
        report[k] = (mx, rl)
        if not np.isfinite(x).all():
            fails.append(f"{k}: non-finite values")
        elif dtype == "fp32":
            if mx > FP32_MAX_ABS:
                fails.append(f"{k}: max abs {mx:.3e} > {FP32_MAX_ABS}")
        elif k in ("o", "ht"):
            if rl > BF16_OUT_REL_L2 or mx > BF16_OUT_MAX_ABS:
                fails.append(f"{k}: rel L2 {rl:.3e} / max abs {mx:.3e}")
        elif k in ("dA_log", "ddt_bias") and "dg" in ref:
            wt = ref["_g"] if k == "dA_log" else ref["_c"]
            dg = ref["dg"]
            HV = dg.shape[-1]
            bound = np.array([BF16_GRAD_REL_L2 * np.linalg.norm(dg[..., h]) * np.linalg.norm(wt[..., h])
                              for h in range(HV)])
            if (np.abs(x - r) > bound).any():
                fails.append(f"{k}: |err| {np.abs(x - r)} > dg-derived bound {bound}")
        else:
            if rl > BF16_GRAD_REL_L2:
                fails.append(f"{k}: rel L2 {rl:.3e} > {BF16_GRAD_REL_L2}")
    return fails, report


def head_select(case: synth.Case, kheads):
    """Index functions picking the sampled heads out of full-size GPU outputs."""
    G = case.HV // case.H
    vh = [h * G + j for h in kheads for j in range(G)]
    return dict(o=lambda x: x[:, :, vh], ht=lambda x: x[:, vh], dh0=lambda x: x[:, vh],
                dq=lambda x: x[:, :, kheads], dk=lambda x: x[:, :, kheads], dv=lambda x: x[:, :, vh],
                dg=lambda x: x[:, :, vh], dbeta=lambda x: x[:, :, vh], dg_raw=lambda x: x[:, :, vh],
                dA_log=lambda x: x[vh], ddt_bias=lambda x: x[vh])
