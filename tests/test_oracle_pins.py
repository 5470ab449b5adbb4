"""Pins of the fp64 oracle to facts other than itself (CPU only).

Each test ties the token-by-token oracle to a closed form, a brute-force sum, an
invariant of the recurrence, a library routine or finite differences, chosen so that a
dropped term, a wrong sign, a wrong index or a transposed operand fails at least one.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import oracle
from gated_deltanet_chunkwise_chunk_b200 import synth

from . import chunk_algebra

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
pytestmark = pytest.mark.filterwarnings("ignore")


def _rng(seed):
    return np.random.default_rng(seed)


def _case(T, K=8, V=8, H=1, HV=1, seed=0, h0=True):
    r = _rng(seed)
    q = r.standard_normal((1, T, H, K))
    k = r.standard_normal((1, T, H, K))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = r.standard_normal((1, T, HV, V))
    a = r.standard_normal((1, T, HV))
    beta = 1 / (1 + np.exp(-r.standard_normal((1, T, HV))))
    A_log = np.log(r.uniform(1, 16, HV))
    dt_bias = r.standard_normal(HV) * 0.5
    S0 = r.standard_normal((1, HV, K, V)) * 0.5 if h0 else None
    return dict(q=q, k=k, v=v, a=a, A_log=A_log, dt_bias=dt_bias, beta=beta, h0=S0)


def _gate_lib(a, A_log, dt_bias):
    """The gate through torch's softplus (threshold 20: returns x when x > 20)."""
    x = torch.as_tensor(a, dtype=torch.float64) + torch.as_tensor(dt_bias, dtype=torch.float64)
    return (-torch.exp(torch.as_tensor(A_log, dtype=torch.float64)) *
            torch.nn.functional.softplus(x, beta=1.0, threshold=20.0)).numpy()


# ---------------------------------------------------------------- gate
def test_gate_golden_closed_forms():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "gate_softplus.txt")) if l.strip()
            and not l.startswith("#")]
    for xs, sps in rows:
        x, sp = float(xs), float(sps)
        # A_log = 0 -> g = -softplus(x)
        got = oracle.gate([x], 0.0, 0.0)[0]
        assert got == pytest.approx(-sp, rel=1e-15, abs=1e-300), (x, got, sp)
    # scale by exp(A_log) and shift by dt_bias
    assert oracle.gate([1.0], math.log(3.0), -1.0)[0] == pytest.approx(-3 * math.log(2.0), rel=1e-15)


def test_gate_matches_library_softplus():
    r = _rng(1)
    a = np.concatenate([r.standard_normal(4000) * 8, r.uniform(19.0, 21.0, 500),
                        r.uniform(-45, -20, 100), r.uniform(20.5, 40, 100)])
    for A_log, dtb in [(0.3, 0.1), (math.log(15.9), -0.7), (-2.0, 1.5)]:
        ref = _gate_lib(a, A_log, dtb)
        got = oracle.gate(a, A_log, dtb)
        np.testing.assert_allclose(got, ref, rtol=1e-14, atol=0)


def test_gate_branch_is_strict_at_20():
    # x = 20 exactly takes the log branch, just above passes x through
    assert oracle.gate([20.0], 0.0, 0.0)[0] == pytest.approx(-math.log1p(math.exp(20.0)), rel=1e-16)
    assert oracle.gate([20.0 + 1e-9], 0.0, 0.0)[0] == -(20.0 + 1e-9)


# ---------------------------------------------------------------- forward pins
def test_beta0_gives_decayed_initial_state_readout():
    """With beta = 0 the delta rule never writes: o_t = scale exp(G_t) S_0 q_t
    (the literal 'beta = 0' and 'g = 0, beta = 0' checks, with a random S_0 so they are
    not trivially zero)."""
    c = _case(23, K=8, V=6, seed=2)
    c["beta"][:] = 0.0
    scale = 0.37
    o, ht, g = oracle.fwd(**c, scale=scale)
    G = np.cumsum(_gate_lib(c["a"][0, :, 0], c["A_log"][0], c["dt_bias"][0]))
    S0 = c["h0"][0, 0].T  # V x K
    ref = scale * np.exp(G)[:, None] * (c["q"][0, :, 0] @ S0.T)
    np.testing.assert_allclose(o[0, :, 0], ref, rtol=1e-12, atol=1e-14)
    # g = 0 as well: constant state
    c["A_log"][:] = -np.inf
    o, ht, g = oracle.fwd(**c, scale=scale)
    np.testing.assert_allclose(o[0, :, 0], scale * c["q"][0, :, 0] @ S0.T, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(ht[0, 0], c["h0"][0, 0], rtol=0, atol=0)


@pytest.mark.parametrize("gated", [False, True])
def test_orthonormal_keys_reduce_to_brute_force_linear_attention(gated):
    """T <= K mutually orthonormal keys and S_0 = 0: S_{t-1} k_t = 0, so the delta rule is
    exactly beta-weighted (gated) causal linear attention, checked against the O(T^2) sum
    o_t = scale sum_{s<=t} beta_s e^{G_t - G_s} (k_s . q_t) v_s."""
    T, K, V = 12, 16, 5
    r = _rng(3)
    Qo, _ = np.linalg.qr(r.standard_normal((K, K)))
    c = _case(T, K=K, V=V, seed=4, h0=False)
    c["k"][0, :, 0] = Qo[:T]
    if not gated:
        c["A_log"][:] = -np.inf
    scale = 0.5
    o, ht, g = oracle.fwd(**c, scale=scale)
    gg = np.zeros(T) if not gated else _gate_lib(c["a"][0, :, 0], c["A_log"][0], c["dt_bias"][0])
    G = np.cumsum(gg)
    qs, ks, vs, b = c["q"][0, :, 0], c["k"][0, :, 0], c["v"][0, :, 0], c["beta"][0, :, 0]
    ref = np.zeros((T, V))
    for t in range(T):
        for s in range(t + 1):
            ref[t] += scale * b[s] * math.exp(G[t] - G[s]) * (ks[s] @ qs[t]) * vs[s]
    np.testing.assert_allclose(o[0, :, 0], ref, rtol=1e-11, atol=1e-13)


def test_no_erase_flag_matches_brute_force_gated_quadratic_form():
    """General keys with the erase term switched off equal the gated quadratic form
    o_t = scale (e^{G_t} S_0 q_t + sum_{s<=t} beta_s e^{G_t-G_s} (k_s.q_t) v_s)."""
    T, K, V = 30, 8, 7
    c = _case(T, K=K, V=V, seed=5)
    scale = 0.3
    o, ht, g = oracle.fwd(**c, scale=scale, flags=oracle.FLAG_NO_ERASE)
    G = np.cumsum(_gate_lib(c["a"][0, :, 0], c["A_log"][0], c["dt_bias"][0]))
    qs, ks, vs, b = c["q"][0, :, 0], c["k"][0, :, 0], c["v"][0, :, 0], c["beta"][0, :, 0]
    S0 = c["h0"][0, 0].T
    ref = np.zeros((T, V))
    for t in range(T):
        ref[t] = scale * math.exp(G[t]) * (S0 @ qs[t])
        for s in range(t + 1):
            ref[t] += scale * b[s] * math.exp(G[t] - G[s]) * (ks[s] @ qs[t]) * vs[s]
    np.testing.assert_allclose(o[0, :, 0], ref, rtol=1e-11, atol=1e-13)
    # and the delta rule proper differs from it
    o2, _, _ = oracle.fwd(**c, scale=scale)
    assert np.abs(o2 - o).max() > 1e-3


@pytest.mark.parametrize("gated", [False, True])
def test_exact_write_invariant(gated):
    """beta = 1 and unit keys: the rule overwrites the value stored under k_t, so
    S_t k_t = v_t for every t, whatever the decay (it only scales the erased part)."""
    T, K, V = 10, 8, 6
    c = _case(T, K=K, V=V, seed=6)
    c["beta"][:] = 1.0
    c["A_log"][:] = -np.inf if not gated else c["A_log"]
    if gated:  # moderate decays so the state is far from zero
        c["A_log"][:] = np.log(0.05)
    for t in range(1, T + 1):
        sub = {kk: (vv[:, :t] if kk in ("q", "k", "v", "a", "beta") else vv) for kk, vv in c.items()}
        _, ht, _ = oracle.fwd(**sub)
        S = ht[0, 0].T  # V x K
        np.testing.assert_allclose(S @ c["k"][0, t - 1, 0], c["v"][0, t - 1, 0], rtol=0, atol=1e-12)


def test_single_token_closed_form():
    """T = 1: o = scale (e^g S_0 (I - beta k k^T) + beta v k^T) q."""
    K, V = 8, 5
    c = _case(1, K=K, V=V, seed=7)
    scale = 0.41
    o, ht, _ = oracle.fwd(**c, scale=scale)
    g = _gate_lib(c["a"][0, 0, 0], c["A_log"][0], c["dt_bias"][0])
    k, q, v, b = c["k"][0, 0, 0], c["q"][0, 0, 0], c["v"][0, 0, 0], c["beta"][0, 0, 0]
    S0 = c["h0"][0, 0].T
    S1 = math.exp(g) * S0 @ (np.eye(K) - b * np.outer(k, k)) + b * np.outer(v, k)
    np.testing.assert_allclose(o[0, 0, 0], scale * S1 @ q, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(ht[0, 0], S1.T, rtol=1e-13, atol=1e-15)


def test_varlen_equals_independent_runs():
    """Packing sequences with cu_seqlens equals running each alone (bit-exact)."""
    lens = [5, 1, 70, 64, 17]
    case = synth.make_case(H=2, HV=4, K=8, V=8, lengths=lens, seed=8, h0=True, dht=True)
    cu = case.cu_seqlens.numpy()
    args = dict(A_log=case.A_log, dt_bias=case.dt_bias)
    o, ht, _ = oracle.fwd(case.q, case.k, case.v, case.a, beta=case.beta, cu_seqlens=cu, h0=case.h0, **args)
    gr = oracle.bwd(case.q, case.k, case.v, case.a, beta=case.beta, dO=case.dO, cu_seqlens=cu,
                    h0=case.h0, dht=case.dht, **args)
    for n in range(len(lens)):
        s = slice(cu[n], cu[n + 1])
        sub = lambda t: t[:, s]
        o1, ht1, _ = oracle.fwd(sub(case.q), sub(case.k), sub(case.v), sub(case.a), beta=sub(case.beta),
                                h0=case.h0[n:n + 1], **args)
        assert np.array_equal(o1, o[:, s]) and np.array_equal(ht1, ht[n:n + 1])
        g1 = oracle.bwd(sub(case.q), sub(case.k), sub(case.v), sub(case.a), beta=sub(case.beta),
                        dO=sub(case.dO), h0=case.h0[n:n + 1], dht=case.dht[n:n + 1], **args)
        for key in ("dq", "dk", "dv", "dg", "dbeta", "da"):
            assert np.array_equal(g1[key], gr[key][:, s]), key
        assert np.array_equal(g1["dh0"], gr["dh0"][n:n + 1])


def test_grouped_heads_equal_repeated_keys():
    """HV = 2H equals H' = HV with q,k repeated per group; dq, dk are the group sums."""
    case = synth.make_case(B=2, T=37, H=2, HV=4, K=8, V=8, seed=9, h0=True, dht=True)
    o, ht, _ = oracle.fwd(case.q, case.k, case.v, case.a, case.A_log, case.dt_bias, case.beta, h0=case.h0)
    rep = lambda t: t.repeat_interleave(2, dim=2)
    o2, ht2, _ = oracle.fwd(rep(case.q), rep(case.k), case.v, case.a, case.A_log, case.dt_bias,
                            case.beta, scale=8 ** -0.5, h0=case.h0)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(ht, ht2)
    g1 = oracle.bwd(case.q, case.k, case.v, case.a, case.A_log, case.dt_bias, case.beta, case.dO,
                    h0=case.h0, dht=case.dht)
    g2 = oracle.bwd(rep(case.q), rep(case.k), case.v, case.a, case.A_log, case.dt_bias, case.beta,
                    case.dO, h0=case.h0, dht=case.dht)
    for key in ("dq", "dk"):
        summed = g2[key].reshape(2, 37, 2, 2, 8).sum(3)
        np.testing.assert_allclose(g1[key], summed, rtol=1e-13, atol=1e-15)
    for key in ("dv", "dg", "dbeta", "dh0"):
        np.testing.assert_allclose(g1[key], g2[key], rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- backward: finite differences
def _loss(c, dO, dht, scale):
    o, ht, _ = oracle.fwd(**c, scale=scale)
    return float((o * dO).sum() + (ht * dht).sum())


@pytest.mark.parametrize("T", [1, 5, 37])
def test_backward_matches_central_differences(T):
    """Every gradient of L = sum(dO o) + sum(dht h_T) against central differences
    (fp64, step 1e-6) on tiny inputs with grouped heads, a random initial state, and gate
    inputs on both sides of the softplus pass-through threshold."""
    K = V = 8
    c = _case(T, K=K, V=V, H=1, HV=2, seed=10 + T)
    c["a"][0, ::3, 1] = 23.0 + np.arange(len(c["a"][0, ::3, 1]))  # x > 20 branch (dt_bias small)
    r = _rng(100 + T)
    dO = r.standard_normal((1, T, 2, V))
    dht = r.standard_normal((1, 2, K, V))
    scale = K ** -0.5
    gr = oracle.bwd(**c, dO=dO, dht=dht, scale=scale)
    h = 1e-6
    names = {"q": "dq", "k": "dk", "v": "dv", "beta": "dbeta", "a": "da", "h0": "dh0",
             "A_log": "dA_log", "dt_bias": "ddt_bias"}
    for name, gname in names.items():
        x = c[name]
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            x0 = x[idx]
            x[idx] = x0 + h
            lp = _loss(c, dO, dht, scale)
            x[idx] = x0 - h
            lm = _loss(c, dO, dht, scale)
            x[idx] = x0
            fd[idx] = (lp - lm) / (2 * h)
        an = gr[gname]
        err = np.linalg.norm(fd - an) / max(np.linalg.norm(an), 1e-30)
        assert err <= 1e-6, (name, err)
    # dg (w.r.t. the gate value itself): perturb g through A_log-free route:
    # dL/da = dg * dg/da, so dg = da / (dg/da) where dg/da = -exp(A_log) * softplus'(x).
    x = c["a"][0, :, :] + c["dt_bias"][None, :]
    sp1 = np.where(x > 20, 1.0, 1 / (1 + np.exp(-x)))
    dgda = -np.exp(c["A_log"])[None, :] * sp1
    np.testing.assert_allclose(gr["dg"][0] * dgda, gr["da"][0], rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- the chunk algebra
@pytest.mark.parametrize("affine", [False, True])
@pytest.mark.parametrize("L", [1, 63, 64, 65, 150])
def test_chunk_algebra_equals_token_recurrence(L, affine):
    """The 64-token chunk reassociation the CUDA kernels implement (A, (I+A)^-1, W, U~,
    state scan, output, and every backward term) equals the token-level oracle; with
    affine=True the passes over the chunks take the affine form S' = e^{G_C} S + B - S N the
    sequential kernels use (and its adjoint)."""
    K, V = 16, 12
    c = _case(L, K=K, V=V, seed=20 + L)
    r = _rng(200 + L)
    dO = r.standard_normal((1, L, 1, V))
    dht = r.standard_normal((1, 1, K, V))
    scale = K ** -0.5
    o, ht, g = oracle.fwd(**c, scale=scale)
    gr = oracle.bwd(**c, dO=dO, dht=dht, scale=scale)
    args = (c["q"][0, :, 0], c["k"][0, :, 0], c["v"][0, :, 0], g[0, :, 0], c["beta"][0, :, 0],
            c["h0"][0, 0].T)
    oc, Sc = chunk_algebra.fwd_unit(*args, scale, affine=affine)
    np.testing.assert_allclose(oc, o[0, :, 0], rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(Sc.T, ht[0, 0], rtol=1e-9, atol=1e-11)
    dq, dk, dv, dg, db, dS0 = chunk_algebra.bwd_unit(*args, dO[0, :, 0], dht[0, 0].T, scale,
                                                     affine=affine)
    for got, ref in [(dq, gr["dq"][0, :, 0]), (dk, gr["dk"][0, :, 0]), (dv, gr["dv"][0, :, 0]),
                     (dg, gr["dg"][0, :, 0]), (db, gr["dbeta"][0, :, 0]), (dS0.T, gr["dh0"][0, 0])]:
        np.testing.assert_allclose(got, ref, rtol=1e-8, atol=1e-10)


@pytest.mark.parametrize("affine", [False, True])
def test_chunk_algebra_long_memory_decay(affine):
    """Same equality when the decay is weak, so the state crosses many chunks."""
    L, K, V = 200, 8, 8
    c = _case(L, K=K, V=V, seed=31)
    c["A_log"][:] = np.log(0.02)
    c["dt_bias"][:] = -4.0
    o, ht, g = oracle.fwd(**c)
    assert np.abs(g).max() < 0.05
    oc, Sc = chunk_algebra.fwd_unit(c["q"][0, :, 0], c["k"][0, :, 0], c["v"][0, :, 0], g[0, :, 0],
                                    c["beta"][0, :, 0], c["h0"][0, 0].T, K ** -0.5, affine=affine)
    np.testing.assert_allclose(oc, o[0, :, 0], rtol=1e-9, atol=1e-11)
