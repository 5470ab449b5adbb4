"""GPU parity of the KDA gate (gdn_kda_gate_fwd / gdn_kda_gate_bwd) against the fp64 oracle,
on the shapes and dtypes of the pages' own test list (T, H, D) x {fp32, fp16, bf16} x {bias,
no bias}, plus the x > 20 branch.  The kernel computes in fp32 and rounds once to the output
dtype.  Error bound per element, derived from that arithmetic: x = g + dt_bias is rounded
once in fp32 (|dx| <= 2^-24 |x|), and softplus and sigmoid both have a relative sensitivity
|d log f / dx| <= 1, so x's rounding costs at most 2^-24 |x| relative; expf, log1pf, the
reciprocal and the products add a few fp32 ulps (8 allowed); the output rounding adds 2^-p
(p = 24, 11, 8 for fp32, fp16, bf16; half an ulp is at most 2^-p relative), plus half the
subnormal spacing for fp16.  The two parameter-gradient sums are fp32 accumulations along
fixed chains of length L (rows per block, then blocks, then the tree), so their bound is
(L + per-term bound) * 2^-24 times the sum of the absolute terms."""
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


SUBNORMAL_HALF = {torch.float32: 2.0 ** -150, torch.float16: 2.0 ** -25, torch.bfloat16: 2.0 ** -134}


def _x(g, dt_bias):
    H, D = g.shape[-2:]
    x = g.double().numpy()
    return x + (dt_bias.double().numpy().reshape(H, D) if dt_bias is not None else 0.0)


def _close(got, ref, x, dtype):
    got = got.double().cpu().numpy()
    err = np.abs(got - ref)
    bound = (ULP[dtype] + (np.abs(x) + 8.0) * 2.0 ** -24) * np.abs(ref) + SUBNORMAL_HALF[dtype]
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
    # the sums: chains of T/128 rows, 128 blocks, then D/256 + 8 tree levels
    L = -(-T // 128) + 128 + -(-D // 256) + 8
    per = L + float(np.abs(x).max()) + 8.0
    yg = okda.fwd(g, A_log, dt_bias)
    scaleA = np.abs(dyg.double().numpy() * yg).sum(axis=(0, 2))
    assert (np.abs(dA.double().cpu().numpy() - rdA) <= per * 2.0 ** -24 * scaleA).all()
    if with_bias:
        scaleB = np.abs(rdg).sum(axis=0).reshape(-1)
        assert (np.abs(ddt.double().cpu().numpy() - rddt) <= per * 2.0 ** -24 * scaleB).all()
    else:
        assert ddt is None


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
