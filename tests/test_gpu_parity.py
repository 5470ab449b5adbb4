"""GPU parity: the CUDA path through the C ABI against the fp64 oracle, element by element,
on the same seeded inputs (the five workloads, block-edge lengths, ragged varlen tails,
long-memory decay) plus the device chunk table, the device status word, determinism and
degenerate cases."""
import os

import numpy as np
import pytest
import torch

from gated_deltanet_chunkwise_chunk_b200 import synth

from .gpu_common import compare, head_select, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _edge_lengths(limit):
    vals = [int(x) for l in open(os.path.join(GOLDEN, "edge_lengths.txt"))
            if not l.startswith("#") for x in l.split()]
    return [v for v in vals if v <= limit]


def _assert_parity(case, gpu=None, ref=None, select=None):
    gpu = run_gpu(case) if gpu is None else gpu
    ref = run_oracle(case) if ref is None else ref
    fails, report = compare(gpu, ref, case.dtype, select=select)
    assert not fails, f"{case.name}: {fails}\n{report}"
    return report


def test_config0_fp32_full():
    _assert_parity(synth.config_case(0))


def test_config1_bf16_full():
    _assert_parity(synth.config_case(1))


@pytest.mark.parametrize("cfg,kheads", [(2, [0, 15]), (3, [5]), (4, [3])])
def test_full_size_sampled_heads(cfg, kheads):
    """Full-size run in the bench's launch configuration; the oracle recomputes a sample of
    k-heads (with their value heads), which are independent problems."""
    case = synth.config_case(cfg)
    gpu = run_gpu(case)
    sub = synth.subset_heads(case, kheads)
    ref = run_oracle(sub)
    _assert_parity(sub, gpu=gpu, ref=ref, select=head_select(case, kheads))


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("T", _edge_lengths(300) + [257])
def test_block_edge_lengths(dtype, T):
    case = synth.make_case(B=2, T=T, H=1, HV=2, K=128, V=128, dtype=dtype, seed=50 + T, h0=True,
                           dht=True, name=f"edge{T}")
    _assert_parity(case)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("KV", [(64, 64), (64, 128), (128, 64)])
def test_head_dims(dtype, KV):
    K, V = KV
    case = synth.make_case(B=1, T=200, H=2, HV=4, K=K, V=V, dtype=dtype, seed=7, h0=True, dht=True,
                           name=f"K{K}V{V}")
    _assert_parity(case)


@pytest.mark.parametrize("H,HV,lengths", [(2, 2, None), (1, 4, None), (2, 8, [70, 0, 129, 5]),
                                           (1, 8, [300])])
def test_value_head_groups_bf16(H, HV, lengths):
    """G = HV/H value heads share a k-head: dq and dk are sums over the group, which the
    tensor-core backward forms inside its kernels (G = 1, 4, 8)."""
    case = synth.make_case(B=1 if lengths else 2, T=300, H=H, HV=HV, K=128, V=128, dtype="bf16",
                           seed=90 + HV, lengths=lengths, h0=True, dht=True, name=f"H{H}HV{HV}")
    _assert_parity(case)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_varlen_ragged(dtype):
    lens = [1, 63, 64, 65, 127, 128, 129, 300, 0, 17]
    case = synth.make_case(H=2, HV=4, K=128, V=128, dtype=dtype, seed=11, lengths=lens, h0=True,
                           dht=True, name="varlen_ragged")
    _assert_parity(case)


def test_long_memory_decay_bf16():
    """Weak decay (g ~ -1e-3 per token): the state carries information across all chunks."""
    case = synth.make_case(B=1, T=1024, H=2, HV=4, K=128, V=128, dtype="bf16", seed=12,
                           long_memory=True, h0=True, dht=True, name="long_memory")
    _assert_parity(case)


def test_long_memory_decay_fp32():
    case = synth.make_case(B=1, T=1024, H=2, HV=4, K=64, V=64, dtype="fp32", seed=13,
                           long_memory=True, h0=True, dht=True, name="long_memory32")
    _assert_parity(case)


def test_softplus_passthrough_branch():
    case = synth.make_case(B=1, T=256, H=2, HV=2, K=64, V=64, dtype="fp32", seed=14, big_a=True,
                           h0=True, dht=True, name="big_a")
    a = case.a.numpy()
    assert (a > 20.5).any() and (a < -20.5).any()
    _assert_parity(case)


def test_empty_input_passes_state_through():
    case = synth.make_case(B=2, T=0, H=1, HV=2, K=64, V=64, dtype="bf16", seed=15, h0=True,
                           dht=True, name="T0")
    gpu = run_gpu(case)
    np.testing.assert_array_equal(gpu["ht"], case.h0.double().numpy())
    np.testing.assert_array_equal(gpu["dh0"], case.dht.double().numpy())
    assert gpu["o"].size == 0 and np.all(gpu["dA_log"] == 0)


def test_varlen_with_empty_sequences():
    case = synth.make_case(H=1, HV=2, K=64, V=64, dtype="fp32", seed=16, lengths=[0, 70, 0, 5],
                           h0=True, dht=True, name="varlen_empty")
    rep = _assert_parity(case)
    gpu = run_gpu(case)
    np.testing.assert_array_equal(gpu["ht"][0], case.h0[0].double().numpy())


def test_device_chunk_table_bit_exact():
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    for lens in ([5, 1, 70, 64, 17], [4095, 257, 1000], [0, 64, 0], [1]):
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
        d = gdn.gdn_dims(1, int(cu[-1]), 1, 1, 64, 64, len(lens), 1, 0.0)
        cap = gdn.max_chunks(d, True)
        table, count = gdn.gdn_chunk_table_device(d, torch.from_numpy(cu).cuda(), cap)
        host = gdn.gdn_build_chunk_indices(d, cu)
        assert count == len(host)
        t = table.cpu().numpy()
        assert np.array_equal(t[:count], host)
        assert (t[count:] == np.array([-1, -1, 0, 0])).all()
    for B, T in ((2, 200), (1, 32768)):
        d = gdn.gdn_dims(B, T, 1, 1, 64, 64, B, 1, 0.0)
        table, count = gdn.gdn_chunk_table_device(d, None)
        assert np.array_equal(table.cpu().numpy()[:count], gdn.gdn_build_chunk_indices(d, None))


def test_invalid_cu_seqlens_sets_device_status():
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    case = synth.make_case(H=1, HV=1, K=64, V=64, dtype="bf16", seed=17, lengths=[10, 20])
    d = {k: (v.cuda() if v is not None else None) for k, v in dict(
        q=case.q, k=case.k, v=case.v, g_raw=case.a, A_log=case.A_log, dt_bias=case.dt_bias,
        beta=case.beta).items()}
    bad = torch.tensor([0, 25, 20], dtype=torch.int64, device="cuda")  # decreasing
    dims = gdn.make_dims(d["q"], d["v"], bad)
    ws = torch.zeros(gdn.workspace_bytes(dims, True, False), dtype=torch.uint8, device="cuda")
    o = torch.full_like(d["v"], 7.0)
    gdn.gdn_chunk_fwd(**d, cu_seqlens=bad, output_final_state=False, workspace=ws, out=o)
    assert gdn.gdn_device_status(ws) == 1
    assert torch.all(o == 7.0)  # no kernel wrote past the failed check
    good = case.cu_seqlens.cuda()
    gdn.gdn_chunk_fwd(**d, cu_seqlens=good, output_final_state=False, workspace=ws, out=o)
    assert gdn.gdn_device_status(ws) == 0


def test_param_grad_reductions_match_gpu_dg():
    """dA_log and ddt_bias are the kernel's reductions of its own dg: they must equal the
    fp64 sums sum_t dg_t g_t and sum_t dg_raw_t of the GPU's dg / dg_raw (g from the gate
    formula), up to fp32 summation rounding relative to sum_t |terms|."""
    for case in (synth.make_case(B=2, T=700, H=2, HV=4, K=128, V=128, dtype="bf16", seed=21,
                                 h0=True, dht=True, big_a=True),
                 synth.make_case(H=2, HV=4, K=128, V=128, dtype="bf16", seed=22,
                                 lengths=[300, 1, 517, 64], dht=True)):
        gpu = run_gpu(case)
        x = case.a.double().numpy() + case.dt_bias.double().numpy()
        sp = np.where(x > 20, x, np.log1p(np.exp(np.minimum(x, 50.0))))
        g = -np.exp(case.A_log.double().numpy()) * sp
        terms = gpu["dg"] * g
        err = np.abs(gpu["dA_log"] - terms.sum(axis=(0, 1)))
        assert (err <= 1e-5 * np.abs(terms).sum(axis=(0, 1)) + 1e-6).all(), err
        terms2 = gpu["dg_raw"]
        err2 = np.abs(gpu["ddt_bias"] - terms2.sum(axis=(0, 1)))
        assert (err2 <= 1e-5 * np.abs(terms2).sum(axis=(0, 1)) + 1e-6).all(), err2


@pytest.mark.parametrize("lengths", [None, [300, 1, 517, 64, 129]])
def test_backward_reusing_forward_workspace(lengths):
    """GDN_FLAG_BWD_REUSE_FWD: the backward that reads the forward's saved intermediates from
    the shared workspace equals the recomputing backward bit for bit, and the oracle."""
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    case = synth.make_case(B=1 if lengths else 2, T=700, H=2, HV=4, K=128, V=128, dtype="bf16",
                           seed=23, lengths=lengths, h0=True, dht=True, name="reuse_fwd")
    d = lambda x: None if x is None else x.cuda()
    args = dict(q=d(case.q), k=d(case.k), v=d(case.v), g_raw=d(case.a), A_log=d(case.A_log),
                dt_bias=d(case.dt_bias), beta=d(case.beta), cu_seqlens=d(case.cu_seqlens),
                initial_state=d(case.h0))
    dims = gdn.make_dims(args["q"], args["v"], args["cu_seqlens"])
    ws = torch.empty(gdn.workspace_bytes(dims, lengths is not None, True), dtype=torch.uint8, device="cuda")
    o, ht = gdn.gdn_chunk_fwd(**args, workspace=ws)
    g1 = gdn.gdn_chunk_bwd(**args, d_o=d(case.dO), dht=d(case.dht), workspace=ws, reuse_forward=True)
    g2 = gdn.gdn_chunk_bwd(**args, d_o=d(case.dO), dht=d(case.dht))
    torch.cuda.synchronize()
    for key in g1:
        assert torch.equal(g1[key], g2[key]), key
    gpu = {k: v.double().cpu().numpy() for k, v in dict(o=o, ht=ht, **g1).items()}
    _assert_parity(case, gpu=gpu)


def test_run_to_run_bitwise_reproducible():
    case = synth.make_case(B=1, T=700, H=2, HV=4, K=128, V=128, dtype="bf16", seed=18, h0=True,
                           dht=True)
    a, b = run_gpu(case), run_gpu(case)
    for k in a:
        assert np.array_equal(a[k], b[k]), k


def test_long_sequence_four_times_the_layer_length():
    """T = 131072 (2048 chunks in one sequence, both scans 2048 steps long), one k-head with
    two value heads, random initial state and final-state gradient: the longest chain the
    suite runs, fwd and bwd against the oracle."""
    case = synth.make_case(B=1, T=131072, H=1, HV=2, K=128, V=128, dtype="bf16", seed=77,
                           h0=True, dht=True, name="long_T131072")
    _assert_parity(case)


@pytest.mark.parametrize("KV,lengths", [((128, 128), None), ((128, 128), [300, 0, 77]),
                                        ((64, 64), None), ((64, 128), [130, 5]), ((128, 64), None)])
def test_bf16_runs_on_the_tensor_core_kernels(KV, lengths):
    """bf16 always takes the tcgen05 kernels (no silent CUDA-core fallback), 64-wide heads
    included: the per-launch profile of one forward + backward names only tcgen05 and prologue
    kernels, every step of the chunk path is among them, and the results match the oracle."""
    import gated_deltanet_chunkwise_chunk_b200 as gdn
    K, V = KV
    case = synth.make_case(B=1 if lengths else 2, T=200, H=2, HV=4, K=K, V=V, dtype="bf16",
                           seed=61, lengths=lengths, h0=True, dht=True, name=f"tc_path_K{K}V{V}")
    gdn.profile(True)
    try:
        gpu = run_gpu(case)
        torch.cuda.synchronize()
        names = set(gdn.profile_read())
    finally:
        gdn.profile(False)
    _assert_parity(case, gpu=gpu)
    assert not any(n.startswith("ffma_") for n in names), names
    tc = {n for n in names if n.startswith("tc_")}
    assert len(tc) >= 6, names
    for step in ("wy", "out", "dvlocal", "dqkwg", "wy_bwd"):
        assert f"tc_{step}" in tc, (step, names)
    assert any("scan_fwd" in n for n in tc) and any("scan_bwd" in n for n in tc), names
