"""The device-side failure path, exercised without faulting or hanging the GPU: a test-only
flag makes the forward's sequential pass withhold one tensor-core product, so the bounded
wait for it runs out.  The call must report GDN_ERR_TIMEOUT through the status word, leave
its outputs unwritten, free what it held, and the next call on the same workspace must run
normally and match the oracle."""
import numpy as np
import pytest
import torch

from gated_deltanet_chunkwise_chunk_b200 import synth

from .gpu_common import compare, run_oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("lengths", [None, [200, 0, 65]])
def test_bounded_wait_runs_out_then_the_next_call_recovers(lengths):
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    from gated_deltanet_chunkwise_chunk_b200 import binding
    case = synth.make_case(B=1, T=300, H=2, HV=4, K=128, V=128, dtype="bf16", seed=71,
                           lengths=lengths, h0=True, name="timeout")
    d = lambda x: None if x is None else x.cuda()
    x = dict(q=d(case.q), k=d(case.k), v=d(case.v), g_raw=d(case.a), A_log=d(case.A_log),
             dt_bias=d(case.dt_bias), beta=d(case.beta), cu_seqlens=d(case.cu_seqlens),
             initial_state=d(case.h0))
    dims = gdn.make_dims(x["q"], x["v"], x["cu_seqlens"])
    ws = torch.empty(gdn.workspace_bytes(dims, lengths is not None, False), dtype=torch.uint8,
                     device="cuda")
    o = torch.full_like(x["v"], 7.0)
    gdn.gdn_chunk_fwd(**x, workspace=ws, out=o, output_final_state=False,
                      flags=binding.GDN_FLAG_TEST_WAIT_TIMEOUT)
    assert gdn.gdn_device_status(ws) == binding.GDN_ERR_TIMEOUT
    assert torch.all(o == 7.0)  # the output kernel skipped its work
    # the same workspace, no flag: a normal call with correct results
    o2, ht = gdn.gdn_chunk_fwd(**x, workspace=ws)
    assert gdn.gdn_device_status(ws) == binding.GDN_OK
    got = dict(o=o2.double().cpu().numpy(), ht=ht.double().cpu().numpy())
    fails, rep = compare(got, run_oracle(case, backward=False), case.dtype, keys=["o", "ht"])
    assert not fails, rep
