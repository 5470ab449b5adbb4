"""Multi-rank plumbing of bench.py on CPU: two gloo ranks on 127.0.0.1 (no GPU).

The data path shards by batch (every rank runs its own problem, no collective between the
kernels), so what needs covering with more than one rank is the host side: the timing is the
maximum over ranks, the throughput counts every rank's tokens, and the reference arm runs on
rank 0 alone while the other ranks leave cleanly.
"""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench

    r, w, local, dist = bench.init_dist("reference")  # gloo
    try:
        # rank r "took" (r + 1) ms for the step and 10 - r ms for the forward
        ms, ms_fwd = bench.max_over_ranks([float(r + 1), float(10 - r)], dist, "cpu")
        value = bench.aggregate_mtok_s(w, 1000, ms)
        q.put((r, w, ms, ms_fwd, value, dist.get_backend()))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_two_gloo_ranks():
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    for r, (rank, world, ms, ms_fwd, value, backend) in enumerate(got):
        assert (rank, world, backend) == (r, 2, "gloo")
        assert ms == 2.0 and ms_fwd == 10.0          # the slowest rank's times on every rank
        assert value == pytest.approx(2 * 1000 / 2e-3 / 1e6)  # both ranks' tokens


def test_single_rank_is_identity():
    import bench

    assert bench.max_over_ranks([3.0, 4.5], None, "cpu") == [3.0, 4.5]
    assert bench.aggregate_mtok_s(1, 32768, 8.0) == pytest.approx(32768 / 8e-3 / 1e6)


def test_reference_arm_under_torchrun_two_ranks():
    """rank 0 alone times the oracle and prints one JSON line; rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--config", "0",
           "--steps", "1", "--warmup", "3", "--ref-budget", "2"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["steps"] == 1 and line["warmup"] == 3
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "M tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
