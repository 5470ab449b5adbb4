"""GPU parity of the token-by-token forward (gdn_recurrent_fwd: decode steps and short
prefills) against the fp64 oracle, with the tolerances of gpu_common (fp32: max abs 1e-4;
bf16: o and final state rel L2 5e-3 and max abs 2e-2)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from gated_deltanet_chunkwise_chunk_b200 import synth

from .gpu_common import compare, run_oracle, to_dev

pytestmark = pytest.mark.gpu


def run_recurrent(case, in_place=False):
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    d = to_dev(case)
    if in_place:
        st = d["initial_state"]
        if st is None:
            st = torch.zeros((case.N, case.HV, case.K, case.V), dtype=torch.float32, device="cuda")
            d["initial_state"] = st
        o, ht = gdn.gdn_recurrent_fwd(**d, final_state=st)
        assert ht.data_ptr() == st.data_ptr()
    else:
        o, ht = gdn.gdn_recurrent_fwd(**d)
    torch.cuda.synchronize()
    return {"o": o.double().cpu().numpy(), "ht": ht.double().cpu().numpy()}


def _assert_parity(case, **kw):
    gpu = run_recurrent(case, **kw)
    ref = run_oracle(case, backward=False)
    fails, report = compare(gpu, ref, case.dtype)
    assert not fails, (case.name, fails, report)


@pytest.mark.parametrize("dtype,KV", [("bf16", 128), ("fp32", 64), ("fp32", 128), ("bf16", 64)])
def test_decode_step(dtype, KV):
    """T = 1 per sequence, a random state in: the decode step."""
    case = synth.make_case(B=8, T=1, H=2, HV=4, K=KV, V=KV, dtype=dtype, seed=300 + KV, h0=True,
                           name=f"decode_{dtype}_{KV}")
    _assert_parity(case)


@pytest.mark.parametrize("in_place", [False, True])
@pytest.mark.parametrize("dtype,KV", [("bf16", 128), ("fp32", 64), ("fp32", 128), ("bf16", 64)])
def test_decode_batch_pipelined(dtype, KV, in_place):
    """A decode step over enough (sequence, value head, 32-row slice) items (>= 1024) to take the
    persistent pipelined kernel, out of place and with the state updated in place."""
    case = synth.make_case(B=64, T=1, H=4, HV=8, K=KV, V=KV, dtype=dtype, seed=330 + KV, h0=True,
                           name=f"decode_pipe_{dtype}_{KV}")
    _assert_parity(case, in_place=in_place)


@pytest.mark.parametrize("T", [2, 5, 37, 64, 65, 200])
def test_short_prefill(T):
    case = synth.make_case(B=2, T=T, H=2, HV=4, K=128, V=128, dtype="bf16", seed=310 + T, h0=True,
                           name=f"prefill{T}")
    _assert_parity(case)


def test_prefill_fp32_no_initial_state():
    case = synth.make_case(B=3, T=50, H=1, HV=2, K=64, V=64, dtype="fp32", seed=320, h0=False,
                           name="prefill_fp32")
    _assert_parity(case)


def test_varlen_ragged_with_empty_sequences():
    case = synth.make_case(H=2, HV=4, K=128, V=128, dtype="bf16", seed=321,
                           lengths=[1, 0, 7, 64, 0, 33, 2], h0=True, name="recurrent_varlen")
    _assert_parity(case)


def test_softplus_branch_and_long_memory():
    case = synth.make_case(B=2, T=96, H=2, HV=4, K=128, V=128, dtype="bf16", seed=322, h0=True,
                           big_a=True, name="recurrent_big_a")
    _assert_parity(case)
    case = synth.make_case(B=1, T=300, H=2, HV=4, K=128, V=128, dtype="bf16", seed=323, h0=True,
                           long_memory=True, name="recurrent_long_memory")
    _assert_parity(case)


def test_in_place_state_update_matches_out_of_place():
    case = synth.make_case(B=4, T=3, H=2, HV=4, K=128, V=128, dtype="bf16", seed=324, h0=True,
                           name="recurrent_in_place")
    a = run_recurrent(case)
    b = run_recurrent(case, in_place=True)
    assert np.array_equal(a["o"], b["o"]) and np.array_equal(a["ht"], b["ht"])


def test_decode_steps_chain_to_the_chunked_forward():
    """T single-token steps carried through the state equal one chunked forward over T."""
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    case = synth.make_case(B=2, T=20, H=2, HV=4, K=128, V=128, dtype="bf16", seed=325, h0=True,
                           name="recurrent_chain")
    d = to_dev(case)
    o_chunk, ht_chunk = gdn.gdn_chunk_fwd(**d)
    st = d["initial_state"].clone()
    outs = []
    for t in range(case.T):
        step = {k: (v[:, t:t + 1].contiguous() if k in ("q", "k", "v", "g_raw", "beta") else v)
                for k, v in d.items()}
        step["initial_state"] = st
        o, _ = gdn.gdn_recurrent_fwd(**step, final_state=st)
        outs.append(o)
    o_steps = torch.cat(outs, dim=1)
    torch.cuda.synchronize()
    ref = run_oracle(case, backward=False)
    for got in ({"o": o_steps, "ht": st}, {"o": o_chunk, "ht": ht_chunk}):
        fails, report = compare({k: v.double().cpu().numpy() for k, v in got.items()}, ref, "bf16")
        assert not fails, (fails, report)


def test_invalid_cu_seqlens_sets_device_status():
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    case = synth.make_case(H=1, HV=1, K=64, V=64, dtype="bf16", seed=326, lengths=[10, 20])
    d = to_dev(case)
    d["cu_seqlens"] = torch.tensor([0, 25, 20], dtype=torch.int64, device="cuda")  # not monotone
    ws = torch.empty(gdn.recurrent_workspace_bytes(), dtype=torch.uint8, device="cuda")
    gdn.gdn_recurrent_fwd(**d, workspace=ws)
    assert gdn.gdn_device_status(ws) == gdn.binding.GDN_ERR_INVALID_ARG
    d["cu_seqlens"] = case.cu_seqlens.cuda()
    gdn.gdn_recurrent_fwd(**d, workspace=ws)
    assert gdn.gdn_device_status(ws) == gdn.binding.GDN_OK
