"""GPU parity of the KDA gate (gdn_kda_gate_fwd / gdn_kda_gate_bwd) against the fp64 oracle,
on the shapes of the pages' test list (T, H, D), their block-edge sequence lengths, fp32 / fp16
/ bf16 in and out, with and without dt_bias, the x > 20 branch, and a D that is not a multiple
of 8 (the scalar path).

The pages accept |out - ref| <= 1e-3 + 1e-3 |ref| against an fp32 reference; the bounds here
are far tighter, derived from the kernel's fp32 arithmetic, in units u = 2^-24 relative:
x = g + dt_bias rounds once (|x| u; softplus and sigmoid have |d log f / dx| <= 1); the fast
exponential e = exp(-|x|) has the documented error 2 + 1.173|x| ulp (<= (4 + 2.35|x|) u); the two
approximate divisions 2 ulp each; the artanh series for log1p, expf(A_log) and the products a
few u more.  Hence (4|x| + 24) u on top of the output rounding 2^-p (p = 24, 11, 8 for fp32,
fp16, bf16), plus half the subnormal spacing of fp16 and a 1e-35 floor for the flushed range.
The two parameter-gradient sums are fp32 accumulations along fixed chains of length L (rows
per block lane, up to 256 lanes, 8 strands of blocks, 8 in a strand's tail, the tree), so their bound is
(L + per-term bound) u times the sum of the absolute terms."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import kda_gate as okda

pytestmark = pytest.mark.gpu

SHAPES = [(1, 4, 64), (16, 8, 128), (64, 16, 64), (128, 12, 96), (1024, 8, 128), (4096, 16, 256)]
ULP = {torch.float32: 2.0 ** -24, torch.float16: 2.0 ** -11, torch.bfloat16: 2.0 ** -8}


def _inputs(T, H, D, dtype, with_bias, seed):
    gen = torch.Generator().manual_seed(seed)
    g = torch.randn(T, H, D, generator=gen).to(dtype)
    A_log = torch.randn(H, generator=gen)
    dt_bias = torch.randn(H * D, generator=gen) if with_bias else None
    return g, A_log, dt_bias


FLOOR = {torch.float32: 1e-35, torch.float16: 2.0 ** -25, torch.bfloat16: 1e-35}


def _x(g, dt_bias):
    H, D = g.shape[-2:]
    x = g.double().numpy()
    return x + (dt_bias.double().numpy().reshape(H, D) if dt_bias is not None else 0.0)


def _close(got, ref, x, dtype):
    got = got.double().cpu().numpy()
    err = np.abs(got - ref)
    bound = (ULP[dtype] + (4.0 * np.abs(x) + 24.0) * 2.0 ** -24) * np.abs(ref) + FLOOR[dtype]
    assert (err <= bound).all(), f"max excess {float((err - bound).max()):.3e}"


@pytest.mark.parametrize("with_bias", [True, False])
@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("T,H,D", SHAPES)
def test_forward(T, H, D, dtype, with_bias):
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    g, A_log, dt_bias = _inputs(T, H, D, dtype, with_bias, seed=T * 31 + D)
    dev = lambda x: None if x is None else x.cuda()
    yg = gdn.kda_gate_fwd(dev(g), dev(A_log), dev(dt_bias), output_dtype=dtype)
    torch.cuda.synchronize()
    ref, x = okda.fwd(g, A_log, dt_bias), _x(g, dt_bias)
    _close(yg, ref, x, dtype)
    if dtype != torch.float32:  # fp32 output of a low-precision input
        y32 = gdn.kda_gate_fwd(dev(g), dev(A_log), dev(dt_bias), output_dtype=torch.float32)
        _close(y32, ref, x, torch.float32)


@pytest.mark.parametrize("with_bias", [True, False])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("T,H,D", [(1, 4, 64), (128, 12, 96), (4096, 16, 256)])
def test_backward(T, H, D, dtype, with_bias):
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    g, A_log, dt_bias = _inputs(T, H, D, dtype, with_bias, seed=T * 17 + H)
    g[0, 0, :3] = torch.tensor([20.5, 35.0, -40.0]).to(dtype)  # both softplus branches
    dyg = torch.randn(T, H, D, generator=torch.Generator().manual_seed(9))
    dev = lambda x: None if x is None else x.cuda()
    dg, dA, ddt = gdn.kda_gate_bwd(dev(g), dev(A_log), dev(dyg), dev(dt_bias))
    torch.cuda.synchronize()
    rdg, rdA, rddt = okda.bwd(g, A_log, dyg, dt_bias)
    x = _x(g, dt_bias)
    _close(dg, rdg, x, dtype)
    # the sums: a block lane's rows, the lanes, 8 strands of blocks, the strand sum, the tree
    L = T + 256 + 296 + 8 + -(-D // 256) + 8
    per = L + 4.0 * float(np.abs(x).max()) + 24.0
    yg = okda.fwd(g, A_log, dt_bias)
    scaleA = np.abs(dyg.double().numpy() * yg).sum(axis=(0, 2))
    assert (np.abs(dA.double().cpu().numpy() - rdA) <= per * 2.0 ** -24 * scaleA).all()
    if with_bias:
        scaleB = np.abs(rdg).sum(axis=0).reshape(-1)
        assert (np.abs(ddt.double().cpu().numpy() - rddt) <= per * 2.0 ** -24 * scaleB).all()
    else:
        assert ddt is None


EDGE_T = [1, 16, 31, 32, 33, 63, 64, 65, 127, 128, 129, 512, 1024, 2048, 4096]
EDGE_HD = [(4, 64), (8, 96), (12, 128), (16, 256), (32, 64)]


@pytest.mark.parametrize("T", EDGE_T)
def test_block_edges_forward_and_backward(T):
    """The pages' sequence lengths around block boundaries, each with one (H, D) of theirs."""
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    H, D = EDGE_HD[EDGE_T.index(T) % len(EDGE_HD)]
    for dtype in (torch.float32, torch.float16, torch.bfloat16):
        for with_bias in (True, False):
            g, A_log, dt_bias = _inputs(T, H, D, dtype, with_bias, seed=T + 1000 * D)
            dev = lambda x: None if x is None else x.cuda()
            x = _x(g, dt_bias)
            yg = gdn.kda_gate_fwd(dev(g), dev(A_log), dev(dt_bias), output_dtype=dtype)
            torch.cuda.synchronize()
            _close(yg, okda.fwd(g, A_log, dt_bias), x, dtype)
    g, A_log, dt_bias = _inputs(T, H, D, torch.bfloat16, True, seed=T + 7)
    dyg = torch.randn(T, H, D, generator=torch.Generator().manual_seed(T)).to(torch.bfloat16)
    dg, dA, ddt = gdn.kda_gate_bwd(g.cuda(), A_log.cuda(), dyg.cuda(), dt_bias.cuda())
    torch.cuda.synchronize()
    rdg, rdA, rddt = okda.bwd(g, A_log, dyg, dt_bias)
    x = _x(g, dt_bias)
    _close(dg, rdg, x, torch.bfloat16)
    per = (T + 256 + 296 + 8 + 1 + 8) + 4.0 * float(np.abs(x).max()) + 24.0
    scaleA = np.abs(dyg.double().numpy() * okda.fwd(g, A_log, dt_bias)).sum(axis=(0, 2))
    assert (np.abs(dA.double().cpu().numpy() - rdA) <= per * 2.0 ** -24 * scaleA).all()
    scaleB = np.abs(rdg).sum(axis=0).reshape(-1)
    assert (np.abs(ddt.double().cpu().numpy() - rddt) <= per * 2.0 ** -24 * scaleB).all()


@pytest.mark.parametrize("T,H,D", [(33, 3, 20), (129, 5, 3), (1, 1, 1), (300, 2, 12)])
def test_head_dim_not_a_multiple_of_8(T, H, D):
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    g, A_log, dt_bias = _inputs(T, H, D, torch.float16, True, seed=D)
    dyg = torch.randn(T, H, D, generator=torch.Generator().manual_seed(1))
    yg = gdn.kda_gate_fwd(g.cuda(), A_log.cuda(), dt_bias.cuda(), output_dtype=torch.float32)
    dg, dA, ddt = gdn.kda_gate_bwd(g.cuda(), A_log.cuda(), dyg.cuda(), dt_bias.cuda())
    torch.cuda.synchronize()
    x = _x(g, dt_bias)
    _close(yg, okda.fwd(g, A_log, dt_bias), x, torch.float32)
    rdg, rdA, rddt = okda.bwd(g, A_log, dyg, dt_bias)
    _close(dg, rdg, x, torch.float16)
    per = (T + 256 + 296 + 8 + 1 + 8) + 4.0 * float(np.abs(x).max()) + 24.0
    scaleA = np.abs(dyg.double().numpy() * okda.fwd(g, A_log, dt_bias)).sum(axis=(0, 2))
    assert (np.abs(dA.double().cpu().numpy() - rdA) <= per * 2.0 ** -24 * scaleA).all()
    scaleB = np.abs(rdg).sum(axis=0).reshape(-1)
    assert (np.abs(ddt.double().cpu().numpy() - rddt) <= per * 2.0 ** -24 * scaleB).all()


def test_backward_is_deterministic_and_empty_input_is_a_no_op():
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    g, A_log, dt_bias = _inputs(1000, 8, 128, torch.bfloat16, True, seed=3)
    dyg = torch.randn(1000, 8, 128).to(torch.bfloat16)
    dev = lambda x: x.cuda()
    a = gdn.kda_gate_bwd(dev(g), dev(A_log), dev(dyg), dev(dt_bias))
    b = gdn.kda_gate_bwd(dev(g), dev(A_log), dev(dyg), dev(dt_bias))
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    e = torch.empty(0, 8, 128, dtype=torch.bfloat16, device="cuda")
    assert gdn.kda_gate_fwd(e, dev(A_log), dev(dt_bias), output_dtype=torch.float32).numel() == 0
    dg, dA, ddt = gdn.kda_gate_bwd(e, dev(A_log), e, dev(dt_bias))
    torch.cuda.synchronize()
    assert dg.numel() == 0 and torch.all(dA == 0) and torch.all(ddt == 0)
