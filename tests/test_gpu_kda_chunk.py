"""GPU parity of the chunkwise KDA forward (gdn_kda_chunk_fwd) against the fp64 token-by-token
KDA oracle, with the Gated DeltaNet path's tolerances (fp32: max abs 1e-4; bf16: o and final
state rel L2 5e-3 and max abs 2e-2): block-edge lengths around the 16-token sub-chunks and
64-token chunks, ragged varlen with empty sequences, weak and strong per-channel decay, no
dt_bias, K != V, and the layer's heads at 2048 tokens."""
from __future__ import annotations

import pytest
import torch

from gated_deltanet_chunkwise_chunk_b200 import synth
from oracle import kda as okda

from .gpu_common import compare, to_dev

pytestmark = pytest.mark.gpu


def _parity(case, seed, with_bias=True, long_memory=False, strong=False):
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    g_raw, A_log, dt_bias = synth.kda_gate_inputs(case, seed, with_bias, long_memory)
    if strong:  # most gate inputs past the softplus pass-through (x > 20), decays of -1 .. -100
        g_raw = 8.0 * g_raw + 14.0
    d = to_dev(case)
    d["g_raw"], d["A_log"] = g_raw.cuda(), A_log.cuda()
    d["dt_bias"] = None if dt_bias is None else dt_bias.cuda()
    o, ht = gdn.gdn_kda_chunk_fwd(**d)
    torch.cuda.synchronize()
    gpu = {"o": o.double().cpu().numpy(), "ht": ht.double().cpu().numpy()}
    cu = None if case.cu_seqlens is None else case.cu_seqlens.numpy()
    ro, rht = okda.recurrent_fwd(case.q, case.k, case.v, g_raw, A_log, dt_bias, case.beta,
                                 cu_seqlens=cu, h0=case.h0)
    fails, report = compare(gpu, {"o": ro, "ht": rht}, case.dtype)
    assert not fails, (case.name, fails, report)
    return report


@pytest.mark.parametrize("T", [1, 15, 16, 17, 63, 64, 65, 130, 200])
def test_block_edges_bf16(T):
    case = synth.make_case(B=2, T=T, H=2, HV=4, K=128, V=128, dtype="bf16", seed=500 + T, h0=True,
                           name=f"kda_chunk_T{T}")
    _parity(case, seed=T)


@pytest.mark.parametrize("K,V", [(64, 64), (64, 128), (128, 64)])
def test_fp32(K, V):
    case = synth.make_case(B=2, T=150, H=2, HV=4, K=K, V=V, dtype="fp32", seed=510 + K + V, h0=True,
                           name=f"kda_chunk_fp32_{K}_{V}")
    _parity(case, seed=511)


def test_no_bias_no_initial_state():
    case = synth.make_case(B=1, T=97, H=1, HV=2, K=128, V=128, dtype="bf16", seed=520, h0=False,
                           name="kda_chunk_nobias")
    _parity(case, seed=521, with_bias=False)


def test_varlen_ragged_with_empty_sequences():
    case = synth.make_case(H=2, HV=4, K=128, V=128, dtype="bf16", seed=530,
                           lengths=[1, 0, 7, 64, 0, 33, 130, 16], h0=True, name="kda_chunk_varlen")
    _parity(case, seed=531)


def test_long_memory():
    """Weak decay (A_log = log U(0.01, 0.1), dt_bias = -4): the state carries across chunks."""
    case = synth.make_case(B=1, T=700, H=2, HV=4, K=128, V=128, dtype="bf16", seed=540, h0=True,
                           name="kda_chunk_long_memory")
    _parity(case, seed=541, long_memory=True)


def test_layer_heads_2048_tokens():
    case = synth.make_case(B=1, T=2048, H=16, HV=32, K=128, V=128, dtype="bf16", seed=550, h0=True,
                           name="kda_chunk_layer")
    _parity(case, seed=551)


def test_empty_input_returns_the_initial_state():
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    case = synth.make_case(B=2, T=0, H=1, HV=2, K=64, V=64, dtype="fp32", seed=560, h0=True, name="kda_chunk_empty")
    g_raw, A_log, dt_bias = synth.kda_gate_inputs(case, 561)
    d = to_dev(case)
    d["g_raw"], d["A_log"], d["dt_bias"] = g_raw.cuda(), A_log.cuda(), dt_bias.cuda()
    o, ht = gdn.gdn_kda_chunk_fwd(**d)
    torch.cuda.synchronize()
    assert o.numel() == 0 and torch.equal(ht.cpu(), case.h0)


def test_strong_gates_bf16():
    """Gate inputs mostly past softplus's pass-through (x > 20) and per-token log-decays down to
    about -100: the in-chunk exponentials underflow to zero inside a 16-token sub-chunk, and the
    output and final state must still match the oracle (no overflow, no NaN)."""
    case = synth.make_case(B=2, T=150, H=2, HV=4, K=128, V=128, dtype="bf16", seed=560, h0=True,
                           name="kda_chunk_strong_gates")
    _parity(case, seed=561, strong=True)


def test_long_sequence_8192_tokens():
    """128 chunks per sequence through the tensor-core state pass (compensated bf16 pairs carried
    along the whole chain), weak decay so the state keeps its history."""
    case = synth.make_case(B=1, T=8192, H=2, HV=4, K=128, V=128, dtype="bf16", seed=570, h0=True,
                           name="kda_chunk_T8192")
    _parity(case, seed=571, long_memory=True)
