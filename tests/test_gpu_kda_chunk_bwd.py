"""GPU parity of the chunkwise KDA backward (gdn_kda_chunk_bwd) against the fp64 KDA oracle
backward.  Tolerances as for the Gated DeltaNet path: fp32 max abs <= 1e-4 on every output;
bf16 gradients rel L2 <= 1e-2, and for dA_log and ddt_bias (sums over every token, and channel,
that can cancel) the rel-L2 bound of their summands carried through Cauchy-Schwarz:
|err(dA_log[h])| <= 1e-2 ||dyg[h]|| ||yg[h]||,  |err(ddt_bias[h,c])| <= 1e-2 ||dg_raw[h,c]|| sqrt(T)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from gated_deltanet_chunkwise_chunk_b200 import synth
from oracle import kda as okda
from oracle import kda_gate as okg

from .gpu_common import BF16_GRAD_REL_L2, FP32_MAX_ABS, compare, to_dev

pytestmark = pytest.mark.gpu


def _run(case, seed, with_bias=True, long_memory=False, dht=True, strong=False):
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    g_raw, A_log, dt_bias = synth.kda_gate_inputs(case, seed, with_bias, long_memory)
    if strong:  # most gate inputs past the softplus pass-through (x > 20), decays of -1 .. -100
        g_raw = 8.0 * g_raw + 14.0
    rng = np.random.default_rng(seed + 1)
    dO = torch.from_numpy(rng.standard_normal((case.B, case.T, case.HV, case.V)).astype(np.float32))
    dO = dO.to(case.q.dtype)
    dht_t = torch.from_numpy((0.1 * rng.standard_normal((case.N, case.HV, case.K, case.V))).astype(np.float32)) \
        if dht else None
    d = to_dev(case)
    d["g_raw"], d["A_log"] = g_raw.cuda(), A_log.cuda()
    d["dt_bias"] = None if dt_bias is None else dt_bias.cuda()
    dims = gdn.make_dims(d["q"], d["v"], d["cu_seqlens"])
    ws = torch.empty(gdn.kda_chunk_workspace_bytes(dims, case.cu_seqlens is not None, True),
                     dtype=torch.uint8, device="cuda")
    gdn.gdn_kda_chunk_fwd(**d, workspace=ws)
    d.pop("initial_state")
    out = gdn.gdn_kda_chunk_bwd(**d, d_o=dO.cuda(), workspace=ws,
                                dht=None if dht_t is None else dht_t.cuda())
    torch.cuda.synchronize()
    gpu = {k: v.double().cpu().numpy() for k, v in out.items() if v is not None}
    cu = None if case.cu_seqlens is None else case.cu_seqlens.numpy()
    ref = okda.recurrent_bwd(case.q, case.k, case.v, g_raw, A_log, dt_bias, case.beta, dO,
                             cu_seqlens=cu, h0=case.h0, dht=dht_t)
    fails, report = compare(gpu, {k: v for k, v in ref.items() if k not in ("dA_log", "ddt_bias")},
                            case.dtype)
    fp32 = case.dtype == "fp32"
    yg = okg.fwd(g_raw, A_log, dt_bias)
    for h in range(case.HV):
        bound = FP32_MAX_ABS if fp32 else \
            BF16_GRAD_REL_L2 * np.linalg.norm(ref["dg"][:, :, h]) * np.linalg.norm(yg[:, :, h]) + 1e-6
        err = abs(gpu["dA_log"][h] - ref["dA_log"][h])
        if err > bound:
            fails.append(f"dA_log[{h}]: {err:.3e} > {bound:.3e}")
    if with_bias:
        K = case.K
        ntok = case.B * case.T
        for h in range(case.HV):
            for c in range(K):
                bound = FP32_MAX_ABS if fp32 else \
                    BF16_GRAD_REL_L2 * np.linalg.norm(ref["dg_raw"][:, :, h, c]) * np.sqrt(ntok) + 1e-6
                err = abs(gpu["ddt_bias"][h * K + c] - ref["ddt_bias"][h * K + c])
                if err > bound:
                    fails.append(f"ddt_bias[{h},{c}]: {err:.3e} > {bound:.3e}")
                    break
    else:
        assert "ddt_bias" not in gpu
    assert not fails, (case.name, fails[:6], report)
    return report


@pytest.mark.parametrize("T", [1, 17, 64, 65, 150])
def test_bf16_block_edges(T):
    case = synth.make_case(B=2, T=T, H=2, HV=4, K=128, V=128, dtype="bf16", seed=600 + T, h0=True,
                           name=f"kda_bwd_T{T}")
    _run(case, seed=T)


@pytest.mark.parametrize("K,V", [(64, 64), (64, 128), (128, 64)])
def test_fp32(K, V):
    case = synth.make_case(B=2, T=100, H=2, HV=4, K=K, V=V, dtype="fp32", seed=610 + K + V, h0=True,
                           name=f"kda_bwd_fp32_{K}_{V}")
    _run(case, seed=611)


def test_no_bias_no_dht():
    case = synth.make_case(B=1, T=80, H=1, HV=2, K=128, V=128, dtype="bf16", seed=620, h0=True,
                           name="kda_bwd_nobias")
    _run(case, seed=621, with_bias=False, dht=False)


def test_varlen_ragged_with_empty_sequences():
    case = synth.make_case(H=2, HV=4, K=128, V=128, dtype="bf16", seed=630,
                           lengths=[1, 0, 7, 64, 0, 33, 130, 16], h0=True, name="kda_bwd_varlen")
    _run(case, seed=631)


def test_long_memory():
    case = synth.make_case(B=1, T=300, H=2, HV=4, K=128, V=128, dtype="bf16", seed=640, h0=True,
                           name="kda_bwd_long_memory")
    _run(case, seed=641, long_memory=True)


def test_layer_heads_1024_tokens():
    case = synth.make_case(B=1, T=1024, H=16, HV=32, K=128, V=128, dtype="bf16", seed=650, h0=True,
                           name="kda_bwd_layer")
    _run(case, seed=651)


def test_empty_input_passes_the_gradient_through():
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    case = synth.make_case(B=2, T=0, H=1, HV=2, K=64, V=64, dtype="bf16", seed=660, h0=True, dht=True,
                           name="kda_bwd_T0")
    g_raw, A_log, dt_bias = synth.kda_gate_inputs(case, 661)
    d = to_dev(case)
    d["g_raw"], d["A_log"], d["dt_bias"] = g_raw.cuda(), A_log.cuda(), dt_bias.cuda()
    dims = gdn.make_dims(d["q"], d["v"])
    ws = torch.empty(gdn.kda_chunk_workspace_bytes(dims, False, True), dtype=torch.uint8, device="cuda")
    o, ht = gdn.gdn_kda_chunk_fwd(**d, workspace=ws)
    d.pop("initial_state")
    d_o = torch.empty(2, 0, 2, 64, dtype=torch.bfloat16, device="cuda")
    out = gdn.gdn_kda_chunk_bwd(**d, d_o=d_o, dht=case.dht.cuda(), workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(ht.cpu(), case.h0) and torch.equal(out["dh0"].cpu(), case.dht)
    assert torch.all(out["dA_log"] == 0) and torch.all(out["ddt_bias"] == 0)


def test_bf16_128_runs_the_tensor_core_kernels():
    """bf16 with 128-wide heads takes the tcgen05 KDA kernels for every chunk step of the
    forward and the backward (the per-launch profile names them, and none of the CUDA-core
    ones) and still matches the oracle; fp32 and 64-wide heads keep the CUDA-core kernels."""
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    case = synth.make_case(H=2, HV=4, K=128, V=128, dtype="bf16", seed=670,
                           lengths=[130, 0, 64, 5], h0=True, name="kda_tc_path")
    gdn.profile(True)
    try:
        _run(case, seed=671)
        torch.cuda.synchronize()
        names = set(gdn.profile_read())
    finally:
        gdn.profile(False)
    steps = ("wy", "scan", "out", "bwd_scan", "bwd_dqk", "bwd_wy")
    for k in steps:
        assert f"kda_tc_{k}" in names, (k, names)
        assert f"kda_{k}" not in names, (k, names)


def test_strong_gates_bf16():
    """The backward with gate inputs mostly past softplus's pass-through and per-token
    log-decays down to about -100 (in-chunk exponentials underflow inside a sub-chunk)."""
    case = synth.make_case(B=2, T=150, H=2, HV=4, K=128, V=128, dtype="bf16", seed=680, h0=True,
                           name="kda_bwd_strong_gates")
    _run(case, seed=681, strong=True)


def test_long_sequence_8192_tokens():
    """The backward through 128 chunks per sequence (the reverse tensor-core state pass), weak decay."""
    case = synth.make_case(B=1, T=8192, H=2, HV=4, K=128, V=128, dtype="bf16", seed=690, h0=True,
                           name="kda_bwd_T8192")
    _run(case, seed=691, long_memory=True)
