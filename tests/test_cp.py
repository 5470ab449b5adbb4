"""Context parallelism over T on CPU: the fold algebra with the fp64 oracle as the per-rank
computation (one process, 1-4 segments), and the real exchange (torch.distributed all-gather and
all-reduce) with two gloo ranks, both against the oracle run over the whole sequences."""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from gated_deltanet_chunkwise_chunk_b200 import cp, synth
from oracle import oracle

from .cp_oracle_ops import OracleOps


def _case(T, seed):
    c = synth.make_case(B=2, T=T, H=2, HV=4, K=16, V=16, dtype="fp32", seed=seed, h0=True, dht=True)
    dO = torch.from_numpy(np.random.default_rng(seed).standard_normal((2, T, 4, 16)))
    return c, dO


def _seg(c, a, b):
    return (c.q[:, a:b], c.k[:, a:b], c.v[:, a:b], c.a[:, a:b], c.A_log, c.dt_bias, c.beta[:, a:b])


@pytest.mark.parametrize("bounds,with_dht", [([0, 37], True), ([0, 20, 37], True), ([0, 1, 15, 36, 37], True),
                                             ([0, 0, 30, 37], True), ([0, 11, 25, 37], False)])
def test_fold_algebra_matches_the_whole_sequence(bounds, with_dht):
    c, dO = _case(37, 71)
    if not with_dht:
        c.dht = None
    ops = OracleOps()
    segs = [_seg(c, a, b) for a, b in zip(bounds[:-1], bounds[1:])]
    sums = [cp.segment_summary(ops, *s) for s in segs]
    Mts, Bhs = [s[0] for s in sums], [s[1] for s in sums]
    o_ref, ht_ref, _ = oracle.fwd(c.q, c.k, c.v, c.a, c.A_log, c.dt_bias, c.beta, h0=c.h0)
    g_ref = oracle.bwd(c.q, c.k, c.v, c.a, c.A_log, c.dt_bias, c.beta, dO, h0=c.h0, dht=c.dht)
    starts, outs = [], []
    for r, s in enumerate(segs):
        h = cp.start_state(ops, Mts, Bhs, r, c.h0)
        starts.append(h)
        outs.append(ops.fwd(*s, h))
    o = torch.cat([x[0] for x in outs], dim=1).numpy()
    np.testing.assert_allclose(o, o_ref, rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(outs[-1][1].numpy(), ht_ref, rtol=1e-9, atol=1e-10)
    Ds = [ops.bwd(*s, starts[r], dO[:, a:b], None, None)["dh0"]
          for r, (s, a, b) in enumerate(zip(segs, bounds[:-1], bounds[1:]))]
    grads = []
    for r, (s, a, b) in enumerate(zip(segs, bounds[:-1], bounds[1:])):
        g_end = cp.end_gradient(ops, Mts, Ds, r, c.dht)
        grads.append(ops.bwd(*s, starts[r], dO[:, a:b], g_end, None))
    for key in ("dq", "dk", "dv", "dg", "dbeta", "dg_raw"):
        got = torch.cat([g[key] for g in grads], dim=1).numpy()
        np.testing.assert_allclose(got, g_ref[key if key != "dg_raw" else "da"], rtol=1e-8, atol=1e-10,
                                   err_msg=key)
    np.testing.assert_allclose(grads[0]["dh0"].numpy(), g_ref["dh0"], rtol=1e-8, atol=1e-10)
    for key in ("dA_log", "ddt_bias"):
        np.testing.assert_allclose(sum(g[key] for g in grads).numpy(), g_ref[key], rtol=1e-8, atol=1e-9)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, bounds, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        c, dO = _case(37, 72)
        a, b = bounds[rank], bounds[rank + 1]
        s = _seg(c, a, b)
        ex = cp.DistExchange()
        ops = OracleOps()
        o, ht, ctx = cp.cp_forward(*s, c.h0, ex, ops=ops)
        g = cp.cp_backward(*s, dO[:, a:b], c.dht, ctx, ex, ops=ops)
        q.put((rank, o.numpy(), ht.numpy(), {k_: v_.numpy() for k_, v_ in g.items()}))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_exchange():
    bounds = [0, 22, 37]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, bounds, q)) for r in range(2)]
    for p_ in procs:
        p_.start()
    res = dict()
    for _ in range(2):
        r, o, ht, g = q.get(timeout=120)
        res[r] = (o, ht, g)
    for p_ in procs:
        p_.join(timeout=60)
        assert p_.exitcode == 0
    c, dO = _case(37, 72)
    o_ref, ht_ref, _ = oracle.fwd(c.q, c.k, c.v, c.a, c.A_log, c.dt_bias, c.beta, h0=c.h0)
    g_ref = oracle.bwd(c.q, c.k, c.v, c.a, c.A_log, c.dt_bias, c.beta, dO, h0=c.h0, dht=c.dht)
    np.testing.assert_allclose(np.concatenate([res[0][0], res[1][0]], axis=1), o_ref, rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(res[1][1], ht_ref, rtol=1e-9, atol=1e-10)
    for key in ("dq", "dk", "dv", "dbeta"):
        got = np.concatenate([res[0][2][key], res[1][2][key]], axis=1)
        np.testing.assert_allclose(got, g_ref[key], rtol=1e-8, atol=1e-10, err_msg=key)
    np.testing.assert_allclose(res[0][2]["dh0"], g_ref["dh0"], rtol=1e-8, atol=1e-10)
    for key in ("dA_log", "ddt_bias"):  # all-reduced: every rank holds the total
        for r in (0, 1):
            np.testing.assert_allclose(res[r][2][key], g_ref[key], rtol=1e-8, atol=1e-9)


def test_segment_summary_needs_square_states():
    c = synth.make_case(B=1, T=5, H=1, HV=1, K=16, V=8, dtype="fp32", seed=1, h0=True)
    with pytest.raises(ValueError):
        cp.segment_summary(OracleOps(), *_seg(c, 0, 5))
