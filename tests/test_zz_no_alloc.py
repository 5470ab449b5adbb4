"""The allocation-free forward entry point (gdn_chunk_fwd_noalloc).

It serves callers that cannot allocate device memory or hand the library a workspace of
their own; it runs the forward in the library's own fixed device array.  Collected last on
purpose: if it fails, a run that stops at the first failure has already run every other
test.  It must pass alone in a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

from gated_deltanet_chunkwise_chunk_b200 import synth

from .gpu_common import compare, run_oracle

pytestmark = pytest.mark.gpu


def _inputs(case):
    d = lambda x: None if x is None else x.cuda()
    return dict(q=d(case.q), k=d(case.k), v=d(case.v), g_raw=d(case.a), A_log=d(case.A_log),
                dt_bias=d(case.dt_bias), beta=d(case.beta), cu_seqlens=d(case.cu_seqlens),
                initial_state=d(case.h0))


def _scribble():
    """A call of another shape, dtype and varlen layout: it leaves unrelated data (and its own
    chunk tables) in the shared array before the next checked call."""
    from gated_deltanet_chunkwise_chunk_b200 import binding
    case = synth.make_case(T=0, H=1, HV=2, K=64, V=64, dtype="fp32", seed=33,
                           lengths=[129, 7, 0, 250], h0=True, name="noalloc_scribble")
    binding.gdn_chunk_fwd_noalloc(**_inputs(case))


@pytest.mark.parametrize("dtype,lengths", [("bf16", None), ("fp32", None), ("bf16", [300, 1, 64, 17])])
def test_noalloc_forward_matches_workspace_forward_twice(dtype, lengths):
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    from gated_deltanet_chunkwise_chunk_b200 import binding
    case = synth.make_case(B=1 if lengths else 2, T=333, H=2, HV=4, K=128, V=128, dtype=dtype,
                           seed=31, lengths=lengths, h0=True, dht=True, name="noalloc")
    x = _inputs(case)
    ref_o, ref_ht = gdn.gdn_chunk_fwd(**x)
    oracle_ref = run_oracle(case, backward=False)
    for call in range(2):
        if call == 1:
            _scribble()  # the second checked call starts from another call's leftovers
        o, ht = binding.gdn_chunk_fwd_noalloc(**x)
        assert binding.noalloc_device_status() == binding.GDN_OK
        got = dict(o=o.double().cpu().numpy(), ht=ht.double().cpu().numpy())
        want = dict(o=ref_o.double().cpu().numpy(), ht=ref_ht.double().cpu().numpy())
        fails, rep = compare(got, want, case.dtype)
        assert not fails, (call, fails, rep)
        fails, rep = compare(got, oracle_ref, case.dtype, keys=["o", "ht"])
        assert not fails, (call, fails, rep)


def test_noalloc_call_allocates_no_device_memory():
    from gated_deltanet_chunkwise_chunk_b200 import binding
    case = synth.make_case(B=1, T=500, H=2, HV=4, K=128, V=128, dtype="bf16", seed=34, h0=True)
    x = _inputs(case)
    o = torch.empty_like(x["v"])
    ht = torch.empty_like(x["initial_state"])
    binding.gdn_chunk_fwd_noalloc(**x, out=o, final_state=ht)  # loads the module, warms up
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        binding.gdn_chunk_fwd_noalloc(**x, out=o, final_state=ht)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0


def test_noalloc_reports_invalid_cu_seqlens():
    from gated_deltanet_chunkwise_chunk_b200 import binding
    case = synth.make_case(H=1, HV=1, K=64, V=64, dtype="bf16", seed=35, lengths=[10, 20])
    x = _inputs(case)
    bad = torch.tensor([0, 25, 20], dtype=torch.int64, device="cuda")  # decreasing
    o = torch.full_like(x["v"], 7.0)
    ht = torch.full((2, 1, 64, 64), 7.0, dtype=torch.float32, device="cuda")
    binding.gdn_chunk_fwd_noalloc(**{**x, "cu_seqlens": bad}, out=o, final_state=ht)
    assert binding.noalloc_device_status() == binding.GDN_ERR_INVALID_ARG
    assert torch.all(o == 7.0)  # no kernel wrote past the failed check
    binding.gdn_chunk_fwd_noalloc(**x, out=o, final_state=ht)
    assert binding.noalloc_device_status() == binding.GDN_OK
    assert not torch.all(o == 7.0)


def test_noalloc_rejects_sizes_beyond_its_array():
    from gated_deltanet_chunkwise_chunk_b200 import binding
    cap = binding.noalloc_scratch_bytes()
    assert cap == 32 << 20
    case = synth.make_case(B=1, T=16384, H=2, HV=8, K=128, V=128, dtype="bf16", seed=32)
    x = _inputs(case)
    dims = binding.make_dims(x["q"], x["v"])
    assert binding.workspace_bytes(dims, False, False) > cap
    o = torch.full_like(x["v"], 3.0)
    with pytest.raises(binding.GDNError) as ei:
        binding.gdn_chunk_fwd_noalloc(**x, out=o)
    assert ei.value.status == binding.GDN_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(o == 3.0)
