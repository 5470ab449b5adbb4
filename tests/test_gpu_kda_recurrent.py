"""GPU parity of the KDA token-by-token forward (gdn_kda_recurrent_fwd: per-key-channel gate,
decode steps and short prefills) against the fp64 KDA oracle, with the tolerances of the
Gated DeltaNet path (fp32: max abs 1e-4; bf16: o and final state rel L2 5e-3, max abs 2e-2),
and bitwise against gdn_recurrent_fwd when every channel carries the same gate."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from gated_deltanet_chunkwise_chunk_b200 import synth
from oracle import kda as okda

from .gpu_common import compare, to_dev

pytestmark = pytest.mark.gpu


def _run(case, g_raw, A_log, dt_bias, in_place=False):
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    d = to_dev(case)
    d["g_raw"], d["A_log"] = g_raw.cuda(), A_log.cuda()
    d["dt_bias"] = None if dt_bias is None else dt_bias.cuda()
    if in_place:
        st = d["initial_state"]
        o, ht = gdn.gdn_kda_recurrent_fwd(**d, final_state=st)
        assert ht.data_ptr() == st.data_ptr()
    else:
        o, ht = gdn.gdn_kda_recurrent_fwd(**d)
    torch.cuda.synchronize()
    return {"o": o.double().cpu().numpy(), "ht": ht.double().cpu().numpy()}


def _parity(case, seed, with_bias=True, long_memory=False):
    g_raw, A_log, dt_bias = synth.kda_gate_inputs(case, seed, with_bias, long_memory)
    gpu = _run(case, g_raw, A_log, dt_bias)
    cu = None if case.cu_seqlens is None else case.cu_seqlens.numpy()
    o, ht = okda.recurrent_fwd(case.q, case.k, case.v, g_raw, A_log, dt_bias, case.beta,
                               cu_seqlens=cu, h0=case.h0)
    fails, report = compare(gpu, {"o": o, "ht": ht}, case.dtype)
    assert not fails, (case.name, fails, report)
    return report


@pytest.mark.parametrize("with_bias", [True, False])
@pytest.mark.parametrize("dtype,KV", [("bf16", 128), ("fp32", 64), ("fp32", 128), ("bf16", 64)])
def test_decode_step(dtype, KV, with_bias):
    case = synth.make_case(B=8, T=1, H=2, HV=4, K=KV, V=KV, dtype=dtype, seed=400 + KV, h0=True,
                           name=f"kda_decode_{dtype}_{KV}")
    _parity(case, seed=401, with_bias=with_bias)


@pytest.mark.parametrize("dtype,KV", [("bf16", 128), ("fp32", 64), ("bf16", 64)])
def test_decode_batch_pipelined(dtype, KV):
    """A KDA decode step over enough items (>= 1024) to take the persistent pipelined kernel."""
    case = synth.make_case(B=64, T=1, H=4, HV=8, K=KV, V=KV, dtype=dtype, seed=460 + KV, h0=True,
                           name=f"kda_decode_pipe_{dtype}_{KV}")
    _parity(case, seed=461)


@pytest.mark.parametrize("T", [2, 17, 64, 65, 200])
def test_short_prefill(T):
    case = synth.make_case(B=2, T=T, H=2, HV=4, K=128, V=128, dtype="bf16", seed=410 + T, h0=True,
                           name=f"kda_prefill{T}")
    _parity(case, seed=T)


def test_prefill_fp32_no_initial_state_and_long_memory():
    case = synth.make_case(B=3, T=50, H=1, HV=2, K=64, V=64, dtype="fp32", seed=420, h0=False,
                           name="kda_prefill_fp32")
    _parity(case, seed=421)
    case = synth.make_case(B=1, T=300, H=2, HV=4, K=128, V=128, dtype="bf16", seed=422, h0=True,
                           name="kda_long_memory")
    _parity(case, seed=423, long_memory=True)


def test_varlen_ragged_with_empty_sequences():
    case = synth.make_case(H=2, HV=4, K=128, V=128, dtype="bf16", seed=430,
                           lengths=[1, 0, 7, 64, 0, 33, 2], h0=True, name="kda_varlen")
    _parity(case, seed=431)


def test_in_place_state():
    case = synth.make_case(B=4, T=3, H=2, HV=4, K=128, V=128, dtype="bf16", seed=440, h0=True,
                           name="kda_in_place")
    g_raw, A_log, dt_bias = synth.kda_gate_inputs(case, 441)
    a = _run(case, g_raw, A_log, dt_bias)
    b = _run(case, g_raw, A_log, dt_bias, in_place=True)
    assert np.array_equal(a["o"], b["o"]) and np.array_equal(a["ht"], b["ht"])


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_channel_constant_gate_equals_gated_deltanet_bitwise(dtype):
    """Same per-token decay on every channel: the same fp32 operations as the scalar-gate kernel."""
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    case = synth.make_case(B=3, T=40, H=2, HV=4, K=128, V=128, dtype=dtype, seed=450, h0=True,
                           name="kda_vs_gdn")
    d = to_dev(case)
    o1, h1 = gdn.gdn_recurrent_fwd(**d)
    d2 = dict(d)
    d2["g_raw"] = d["g_raw"][..., None].expand(-1, -1, -1, case.K).contiguous()
    d2["dt_bias"] = d["dt_bias"][:, None].expand(-1, case.K).contiguous().view(-1)
    o2, h2 = gdn.gdn_kda_recurrent_fwd(**d2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(h1, h2)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_channel_constant_gate_equals_gated_deltanet_bitwise_pipelined(dtype):
    """The same bitwise equality on a decode batch large enough for the pipelined kernel."""
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    case = synth.make_case(B=64, T=1, H=4, HV=8, K=128, V=128, dtype=dtype, seed=470, h0=True,
                           name="kda_vs_gdn_pipe")
    d = to_dev(case)
    o1, h1 = gdn.gdn_recurrent_fwd(**d)
    d2 = dict(d)
    d2["g_raw"] = d["g_raw"][..., None].expand(-1, -1, -1, case.K).contiguous()
    d2["dt_bias"] = d["dt_bias"][:, None].expand(-1, case.K).contiguous().view(-1)
    o2, h2 = gdn.gdn_kda_recurrent_fwd(**d2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(h1, h2)
