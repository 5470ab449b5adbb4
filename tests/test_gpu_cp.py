"""Context parallelism on one GPU: gdn_state_affine against an fp64 product, and the ranks'
computations (segment summaries, folds, segment forward and backward on the library's kernels)
run one after another, the exchange replaced by Python lists, against the oracle over the whole
sequences (the Gated DeltaNet tolerances of gpu_common)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from gated_deltanet_chunkwise_chunk_b200 import cp, synth

from .gpu_common import compare, run_oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("K,V,transpose", [(128, 128, False), (128, 128, True), (64, 128, True), (64, 64, False)])
def test_state_affine(K, V, transpose):
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    g = torch.Generator().manual_seed(K + V)
    A = torch.randn(3, 5, K, K, generator=g)
    X = torch.randn(3, 5, K, V, generator=g)
    B = torch.randn(3, 5, K, V, generator=g)
    ref = (A.double().transpose(-1, -2) if transpose else A.double()) @ X.double() + B.double()
    out = gdn.state_affine(A.cuda(), X.cuda(), B.cuda(), transpose=transpose)
    Xc = X.cuda()
    gdn.state_affine(A.cuda(), Xc, B.cuda(), transpose=transpose, out=Xc)  # in place
    torch.cuda.synchronize()
    bound = 1e-5 * (A.double().abs().transpose(-1, -2) if transpose else A.double().abs()) @ X.double().abs() + 1e-6
    assert ((out.cpu().double() - ref).abs() <= bound).all()
    assert torch.equal(Xc.cpu(), out.cpu())


def _emulate(case, bounds, dO):
    ops = cp.Ops()
    dev = lambda x: None if x is None else x.cuda().contiguous()
    segs = [tuple(dev(x) for x in (case.q[:, a:b], case.k[:, a:b], case.v[:, a:b], case.a[:, a:b],
                                   case.A_log, case.dt_bias, case.beta[:, a:b]))
            for a, b in zip(bounds[:-1], bounds[1:])]
    h0, dht = dev(case.h0), dev(case.dht)
    sums = [cp.segment_summary(ops, *s) for s in segs]
    Mts, Bhs = [s[0] for s in sums], [s[1] for s in sums]
    starts, outs, wss = [], [], []
    for r, s in enumerate(segs):
        h = cp.start_state(ops, Mts, Bhs, r, h0)
        ws = ops.workspace(s[0], s[2])
        starts.append(h)
        wss.append(ws)
        outs.append(ops.fwd(*s, h, workspace=ws))
    dOs = [dev(dO[:, a:b]) for a, b in zip(bounds[:-1], bounds[1:])]
    Ds = [ops.bwd(*s, starts[r], dOs[r], None, wss[r])["dh0"] for r, s in enumerate(segs)]
    grads = [ops.bwd(*s, starts[r], dOs[r], cp.end_gradient(ops, Mts, Ds, r, dht), wss[r])
             for r, s in enumerate(segs)]
    torch.cuda.synchronize()
    cat = lambda key: torch.cat([g[key] for g in grads], dim=1).double().cpu().numpy()
    res = {"o": torch.cat([o for o, _ in outs], dim=1).double().cpu().numpy(),
           "ht": outs[-1][1].double().cpu().numpy(),
           "dh0": grads[0]["dh0"].double().cpu().numpy()}
    for key in ("dq", "dk", "dv", "dg", "dbeta", "dg_raw"):
        res[key] = cat(key)
    for key in ("dA_log", "ddt_bias"):
        res[key] = sum(g[key].double() for g in grads).cpu().numpy()
    return res


@pytest.mark.parametrize("bounds,long_memory", [([0, 200, 512], False), ([0, 64, 130, 300, 512], False),
                                                ([0, 150, 333, 700], True), ([0, 0, 200, 512], True)])
def test_segments_equal_the_whole_sequence(bounds, long_memory):
    T = bounds[-1]
    case = synth.make_case(B=1, T=T, H=2, HV=4, K=128, V=128, dtype="bf16", seed=700 + T, h0=True,
                           dht=True, long_memory=long_memory, name=f"cp_{len(bounds) - 1}x")
    gpu = _emulate(case, bounds, case.dO)
    ref = run_oracle(case)
    fails, report = compare(gpu, ref, "bf16")
    assert not fails, (case.name, fails, report)
