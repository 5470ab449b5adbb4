#!/usr/bin/env python
"""Throughput of the chunkwise Gated DeltaNet forward + backward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config I]

One step = gdn_chunk_fwd + gdn_chunk_bwd (every kernel of the forward and the backward)
over one batch of the workload, inputs resident in HBM; the backward reads the chunk
intermediates that the same step's forward saved in the shared workspace
(GDN_FLAG_BWD_REUSE_FWD), as a training step keeps forward activations for its backward.  The default workload is the
Qwen3-Next-shaped layer: B=1, T=32768, H=16 q/k heads, HV=32 value heads, K=V=128, bf16
q/k/v/o/dO, fp32 gates/beta/states, random initial state and final-state gradient.
Synthetic seeded inputs (no dataset).  Every step streams ~1 GB of inputs, outputs and
intermediates, far more than the 126 MB L2, so no explicit L2 flush is needed.

Reports M tokens/s (tokens = B*T per GPU, summed over GPUs; weak scaling: every rank runs
its own batch, no collective in the data path), the end-to-end number through the public
API with host buffers, the dominant kernel's roofline, and the fp64 CPU oracle timed on a
bounded sample on the host cores.  ``--impl reference`` times that oracle alone.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_deltanet_chunkwise_chunk_b200 import synth  # noqa: E402

C = 64
METRIC = "GDN chunk fwd+bwd M tokens/s at T=32k,H=16,HV=32,D=128 bf16; % of roofline"
DATASHEET = dict(tensor_tflops=2250.0, hbm_gbs=8000.0)
FALLBACK = dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0)
# fp32 FFMA peak: 148 SMs x 128 fp32 lanes x 2 FLOP x 1.965 GHz
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


# ----------------------------------------------------------------- algorithmic work
def kernel_flops_per_token_head(K: int, V: int) -> dict:
    """FLOPs each kernel must do per token per value head (its products; 64-row tiles)."""
    per = {
        "wy": 2 * C * K + C * C / 3 + 2 * C * (K + V),
        "scan_fwd": 4 * K * V,
        "out": 2 * C * K + 2 * C * V + 2 * K * V,
        "dvlocal": 2 * C * K + 2 * C * V,
        "scan_bwd": 6 * K * V,
        "dqkwg": 6 * C * K + 2 * C * V + 6 * K * V,
        "wy_bwd": 10 * C * K + 4 * C * V + 4 * C * C,
    }
    return {f"{path}_{k}": v for k, v in per.items() for path in ("ffma", "tc")}


def kernel_bytes_per_unit(K: int, V: int, G: int, e: int) -> dict:
    """HBM bytes each tcgen05 kernel moves per (chunk, value head) unit under the current kernel
    split: every operand tile it reads and every tile it writes once (a k-head's q/k tile is
    shared by its G value heads and counted once), inter-kernel intermediates included (bf16
    tiles W^T, U~^T, D K, -N^T, U^T, S, dS, dU_loc^T, O', dU^T hi/lo, dW, T hi/lo; the k-head's
    fp32 dq/dk tiles; fp32 per-chunk vectors of 64).  Reported beside the roofline, not as the
    method's bytes."""
    tq = C * K * e / G            # q or k tile, per value head
    tv = C * V * e                # v, o, dO, dv tile
    dk = C * K * e                # D K (per value head: scaled by its own decay), O'
    wt = K * C * e                # W^T, dW
    ut = V * C * e                # U~^T, U^T, dU_loc^T, dU^T (one part)
    st = V * K * e                # S or dS entering/leaving the chunk
    nt = K * K * e                # -N^T, the state map's K x K factor
    tm = 2 * C * C * e            # T = (I + A)^-1 as a hi/lo pair
    f32 = C * K * 4 / G           # the k-head's fp32 dq or dk tile, per value head
    vec = C * 4                   # one per-chunk fp32 vector
    per = {
        "wy": tq + tv + 3 * vec + wt + ut + tm + dk + nt,
        "scan_fwd": ut + nt + dk + vec + st,
        "out": 2 * tq + st + wt + ut + vec + tv + ut,
        "dvlocal": 2 * tq + tv + 2 * vec + ut + dk,
        "scan_bwd": nt + dk + tq + dk + wt + ut + vec + st + 2 * ut,
        "dqkwg": 2 * tq + tv + 3 * ut + 2 * st + vec + wt + vec + 2 * f32,
        "wy_bwd": tq + tv + tm + wt + 2 * ut + 2 * vec + tv + 2 * vec + 2 * f32,  # dk added in L2
        "dqdk_out": 2 * f32 + 2 * tq,
    }
    return {f"tc_{k}": v for k, v in per.items()}


def step_flops_per_token_head(K: int, V: int) -> tuple[float, float]:
    """Algorithmic FLOPs of the method per token per value head (fwd, bwd)."""
    fwd = 2 * C * (3 * K + 2 * V) + 6 * K * V + C * C / 3
    bwd = 2 * C * (9 * K + 5 * V) + 16 * K * V + 4 * C * C + C * C / 3
    return fwd, bwd


def step_bytes(case, e: int) -> tuple[float, float]:
    """Minimum HBM bytes of one forward and one backward (inputs read once, outputs written
    once; intermediates not counted)."""
    B, T, H, HV, K, V = case.B, case.T, case.H, case.HV, case.K, case.V
    ntok = B * T
    Nst = case.N
    states = 4 * K * V * HV * Nst
    fwd = ntok * (2 * H * K * e + HV * V * e + 8 * HV + HV * V * e) + (states if case.h0 is not None else 0) + states
    bwd_in = ntok * (2 * H * K * e + 2 * HV * V * e + 8 * HV)
    bwd_out = ntok * (2 * H * K * e + HV * V * e + 8 * HV)
    bwd = bwd_in + bwd_out + states * (1 + (case.h0 is not None) + (case.dht is not None))
    return fwd, bwd


def peaks() -> dict:
    p = dict(FALLBACK)  # every key present even if the measured file lacks one
    src = "fallback"
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            m = json.load(f)
        p.update({k: m[k] for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained") if k in m})
        src = "measured"
    except (OSError, ValueError):
        pass
    p["source"] = src
    return p


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]),
                                 power=float(parts[3]) if parts[3] not in ("[N/A]", "N/A") else 0.0,
                                 hw=parts[5], hwt=parts[6], swt=parts[7], swp=parts[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("swp", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        load = [r for r in rows if r["power"] > 300] or rows
        return {"sm_mhz": statistics.median(r["sm"] for r in load),
                "sm_max_mhz": max(r["smax"] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows), "samples_under_load": len(load)}


# ----------------------------------------------------------------- oracle baseline
def oracle_sample(case, budget_s: float = 12.0) -> dict:
    """fp64 oracle (fwd + bwd) on a bounded sample of the workload, every head: the first Ts
    tokens of every batch row (Ts doubled from 64), or for a packed varlen batch its first m
    sequences (m doubled from 1), grown until one run costs about a third of the budget.
    Returns the sample's throughput and the measured time of that one sample run."""
    from oracle import oracle

    def run_dense(Ts):
        sub = dict(q=case.q[:, :Ts], k=case.k[:, :Ts], v=case.v[:, :Ts], a=case.a[:, :Ts],
                   A_log=case.A_log, dt_bias=case.dt_bias, beta=case.beta[:, :Ts])
        t0 = time.perf_counter()
        oracle.fwd(**sub, h0=case.h0)
        oracle.bwd(**sub, dO=case.dO[:, :Ts], h0=case.h0, dht=case.dht)
        return time.perf_counter() - t0

    def run_varlen(m):
        cu = case.cu_seqlens[: m + 1]
        Ts = int(cu[-1])
        sub = dict(q=case.q[:, :Ts], k=case.k[:, :Ts], v=case.v[:, :Ts], a=case.a[:, :Ts],
                   A_log=case.A_log, dt_bias=case.dt_bias, beta=case.beta[:, :Ts])
        h0 = None if case.h0 is None else case.h0[:m]
        dht = None if case.dht is None else case.dht[:m]
        t0 = time.perf_counter()
        oracle.fwd(**sub, cu_seqlens=cu.numpy(), h0=h0)
        oracle.bwd(**sub, dO=case.dO[:, :Ts], cu_seqlens=cu.numpy(), h0=h0, dht=dht)
        return time.perf_counter() - t0

    if case.cu_seqlens is not None:
        m, nseq = 1, case.N
        dt = run_varlen(m)
        while dt < budget_s / 3 and m * 2 <= nseq:
            m *= 2
            dt = run_varlen(m)
        tok = int(case.cu_seqlens[m])
        units = m * case.HV
        what = f"first {m} of {nseq} packed sequences ({tok} of {case.tokens} tokens)"
    else:
        Ts = 64
        dt = run_dense(Ts)
        while dt < budget_s / 3 and Ts * 2 <= case.T:
            Ts *= 2
            dt = run_dense(Ts)
        tok = case.B * Ts
        units = case.B * case.HV
        what = f"{case.B} batch rows, first {Ts} of {case.T} tokens ({tok} tokens)"
    cores = min(os.cpu_count() or 1, units)
    return {"value": tok / dt / 1e6, "unit": "M tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"fp64 token-by-token oracle fwd+bwd, all {case.HV} value heads, {what}, "
                      f"{dt:.2f} s",
            "seconds": dt, "tokens": tok}


# ----------------------------------------------------------------- ranks
def init_dist(impl: str):
    """One process per GPU, launched by torch.distributed.run (RANK / LOCAL_RANK /
    WORLD_SIZE / MASTER_* from the environment).  Every rank runs its own batch; the only
    collectives are the barriers around the timed region and the max over ranks of the
    timings (NCCL for our arm, gloo for the host-only reference arm)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() and impl == "ours" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return rank, world, local, dist


def max_over_ranks(values, dist, device) -> list[float]:
    """Element-wise maximum over ranks (identity with one rank): a multi-GPU time is the
    slowest rank's."""
    if not dist:
        return [float(x) for x in values]
    tt = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return [float(x) for x in tt.tolist()]


def aggregate_mtok_s(world: int, tokens_per_rank: int, ms: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return world * tokens_per_rank / (ms / 1e3) / 1e6


# ----------------------------------------------------------------- our arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=24)
    ap.add_argument("--T", type=int, default=None,
                    help="override the sequence length of a dense workload (smaller profiling cases)")
    ap.add_argument("--workload", default="gdn", choices=["gdn", "kda_chunk", "decode"],
                    help="kda_chunk: only the chunkwise KDA measurement (its T from --T, default 32768); "
                         "decode: only the decode-step measurement")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the lines of the other workloads in the default run")
    ap.add_argument("--ref-budget", type=float, default=90.0,
                    help="seconds of oracle work over the whole --impl reference run")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank, world, local, dist = init_dist(args.impl)

    if args.impl == "reference":
        return reference_arm(args, rank, world, dist)

    import gated_deltanet_chunkwise_chunk_b200 as gdn

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.workload == "decode":
        line = decode_measure(gdn, dev, pk_hbm=peaks()["hbm_gbs"], steps=max(1, args.steps))
        if rank == 0:
            print(json.dumps(line), flush=True)
        if dist:
            dist.destroy_process_group()
        return
    if args.workload == "kda_chunk":
        line = kda_chunk_measure(gdn, dev, pk_hbm=peaks()["hbm_gbs"], steps=max(1, args.steps),
                                 T=args.T or 32768)
        if rank == 0:
            print(json.dumps(line), flush=True)
        if dist:
            dist.destroy_process_group()
        return
    case = synth.config_case(args.config, seed=1000 + args.config + 7919 * rank, T=args.T)
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
    sampler = ClockSampler(vis[local].strip() if len(vis) > local and vis[local].strip() else local)
    m = measure_case(gdn, case, dev, args.steps, args.warmup, dist, world, sampler=sampler,
                     e2e_steps=args.e2e_steps)
    full = args.config == 2 and args.T is None
    decode = decode_measure(gdn, dev, pk_hbm=peaks()["hbm_gbs"]) if full else None
    kda = kda_gate_measure(gdn, dev, pk_hbm=peaks()["hbm_gbs"]) if full else None
    kda_decode = decode_measure(gdn, dev, pk_hbm=peaks()["hbm_gbs"], kda=True) if full else None
    kda_chunk = kda_chunk_measure(gdn, dev, pk_hbm=peaks()["hbm_gbs"]) if full else None

    line = {
        "metric": METRIC, "value": m["value"], "unit": "M tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": m["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": case.dtype, "data": "synthetic (seeded N(0,1)/sigmoid/log-uniform inputs; no dataset)",
        "config": {"workload": case.name, "B": case.B, "T": case.T, "H": case.H, "HV": case.HV,
                   "K": case.K, "V": case.V, "chunk": C, "global_batch": case.B * world,
                   "seq_len": case.T, "parallelism": f"dp{world} (independent batches)",
                   "l2": m["l2"]},
    }
    line.update({k: v for k, v in m.items() if k not in ("value", "ms_per_step", "l2")})
    line.update({"decode": decode, "kda_gate": kda, "kda_decode": kda_decode, "kda_chunk": kda_chunk,
                 "peaks_source": peaks()["source"]})
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        try:
            line["cpu_baseline"] = oracle_sample(case)
            for k in ("seconds", "tokens"):
                line["cpu_baseline"].pop(k, None)
        except Exception as ex:  # noqa: BLE001
            line["cpu_baseline"] = {"error": str(ex)}
    if full and not args.no_other_configs:
        # the other workloads of the pages' shapes: same step, same measurements
        others = {}
        for idx in (0, 1, 3, 4):
            oc = synth.config_case(idx, seed=1000 + idx + 7919 * rank)
            sub = measure_case(gdn, oc, dev, args.steps, args.warmup, dist, world, sampler=None,
                               e2e_steps=12)
            sub["config"] = {"workload": oc.name, "B": oc.B, "T": oc.T, "tokens": oc.tokens,
                             "H": oc.H, "HV": oc.HV, "K": oc.K, "V": oc.V, "dtype": oc.dtype}
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                cb = oracle_sample(oc, budget_s=6.0)
                sub["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
            others[f"config{idx}"] = sub
            del oc
        # the one shape the G_T_CONTIG page times itself (section on measured gains):
        # B=2, T=2048, H=4, HV=8 with 64-wide key and value heads
        pc = synth.make_case(B=2, T=2048, H=4, HV=8, K=64, V=64, dtype="bf16", seed=1100 + 7919 * rank,
                             name="bf16_B2_T2048_H4_HV8_D64")
        sub = measure_case(gdn, pc, dev, args.steps, args.warmup, dist, world, sampler=None, e2e_steps=12)
        sub["config"] = {"workload": pc.name, "B": pc.B, "T": pc.T, "tokens": pc.tokens, "H": pc.H,
                         "HV": pc.HV, "K": pc.K, "V": pc.V, "dtype": pc.dtype}
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            cb = oracle_sample(pc, budget_s=6.0)
            sub["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
        others["pages_k64"] = sub
        line["other_workloads"] = others
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def measure_case(gdn, case, dev, steps: int, warmup: int, dist, world: int, sampler=None,
                 e2e_steps: int = 3) -> dict:
    """One workload: W warm-up steps, then K timed training steps (forward + backward reading
    the forward's saved intermediates) and K timed forwards, CUDA events on the launching
    stream, max over ranks; then a profiled pass (events around every launch) for the
    per-kernel times and the dominant kernel's roofline, and the end-to-end number."""
    e = 2 if case.dtype == "bf16" else 4
    t = lambda x: None if x is None else x.to(dev).contiguous()
    inp = dict(q=t(case.q), k=t(case.k), v=t(case.v), g_raw=t(case.a), A_log=t(case.A_log),
               dt_bias=t(case.dt_bias), beta=t(case.beta), cu_seqlens=t(case.cu_seqlens),
               initial_state=t(case.h0))
    dO, dht = t(case.dO), t(case.dht)
    dims = gdn.make_dims(inp["q"], inp["v"], inp["cu_seqlens"])
    varlen = case.cu_seqlens is not None
    ws = torch.empty(max(gdn.workspace_bytes(dims, varlen, False), gdn.workspace_bytes(dims, varlen, True)),
                     dtype=torch.uint8, device=dev)  # shared by the forward and the backward
    o = torch.empty_like(inp["v"])
    ht = torch.empty((case.N, case.HV, case.K, case.V), dtype=torch.float32, device=dev)
    outs = dict(dq=torch.empty_like(inp["q"]), dk=torch.empty_like(inp["k"]), dv=torch.empty_like(inp["v"]),
                dg=torch.empty_like(inp["g_raw"]), dbeta=torch.empty_like(inp["beta"]),
                dh0=torch.empty_like(ht), dg_raw=torch.empty_like(inp["g_raw"]),
                dA_log=torch.empty_like(inp["A_log"]), ddt_bias=torch.empty_like(inp["A_log"]))

    def fwd():
        gdn.gdn_chunk_fwd(**inp, workspace=ws, out=o, final_state=ht)

    def step():
        # the backward reads the chunk intermediates this step's forward left in `ws`
        fwd()
        gdn.gdn_chunk_bwd(**inp, d_o=dO, dht=dht, workspace=ws, outs=outs, reuse_forward=True)

    stream = torch.cuda.current_stream()
    # a workload whose tensors fit in L2 (126 MB) is timed one step at a time with L2 flushed
    # before each (a 256 MB write outside the timed events); a larger one streams its inputs
    # from HBM anyway and is timed as one run of steps
    footprint = sum(x.numel() * x.element_size() for x in list(inp.values()) + [dO, dht]
                    if x is not None)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if footprint < (256 << 20) else None

    def timed(fn, n):
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        if flush is None:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(n):
                fn()
            b.record(stream)
            torch.cuda.synchronize()
            total = a.elapsed_time(b)
        else:
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(n)]
            for a, b in ev:
                flush.zero_()
                a.record(stream)
                fn()
                b.record(stream)
            torch.cuda.synchronize()
            total = sum(a.elapsed_time(b) for a, b in ev)
        if dist:
            dist.barrier()
        return total / n

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if sampler is not None:
        sampler.start()
        time.sleep(0.3)
    n0 = gdn.launch_count()
    ms = timed(step, steps)
    launches = (gdn.launch_count() - n0) // max(1, steps) * steps
    clocks = sampler.stop() if sampler is not None else None
    ms_fwd = timed(fwd, max(1, steps))
    ms, ms_fwd = max_over_ranks([ms, ms_fwd], dist, dev)

    # per-kernel device time (separate pass: events around every launch on its stream)
    gdn.profile(True)
    for _ in range(2):
        step()
    prof = gdn.profile_read()
    gdn.profile(False)

    e2e = e2e_measure(gdn, case, dev, ws, e2e_steps, dist)
    tokens = case.tokens
    pk = peaks()
    fflop, bflop = step_flops_per_token_head(case.K, case.V)
    th = tokens * case.HV
    fbytes, bbytes = step_bytes(case, e)
    flops = th * (fflop + bflop)
    nbytes = fbytes + bbytes
    t_roof_ds = max(flops / (DATASHEET["tensor_tflops"] * 1e12), nbytes / (DATASHEET["hbm_gbs"] * 1e9))
    t_roof_b = max(flops / (pk["bf16_tflops"] * 1e12), nbytes / (pk["hbm_gbs"] * 1e9))
    t_roof_m = max(flops / (pk["bf16_tflops_sustained"] * 1e12), nbytes / (pk["hbm_gbs"] * 1e9))
    t_froof = max(th * fflop / (pk["bf16_tflops"] * 1e12), fbytes / (pk["hbm_gbs"] * 1e9))
    del ws
    return {
        "value": round(aggregate_mtok_s(world, tokens, ms), 3), "ms_per_step": round(ms, 4),
        "fwd_mtok_s": round(aggregate_mtok_s(world, tokens, ms_fwd), 3),
        "ms_fwd": round(ms_fwd, 4),
        "step_roofline": {"flops": flops, "bytes": nbytes,
                          "bound": "tensor" if flops / 2.25e15 >= nbytes / 8e12 else "hbm",
                          "frac_datasheet": round(t_roof_ds / (ms / 1e3), 4),
                          "frac_measured_burst": round(t_roof_b / (ms / 1e3), 4),
                          "frac_measured": round(t_roof_m / (ms / 1e3), 4),
                          "fwd_frac_measured_burst": round(t_froof / (ms_fwd / 1e3), 4),
                          "roofline_mtok_s_datasheet": round(tokens / t_roof_ds / 1e6, 2),
                          "note": "max(FLOP/bf16 peak, bytes/HBM) over the whole fwd+bwd step; "
                                  "frac_measured uses the sustained bf16 peak, _burst the burst one"},
        "roofline": kernel_roofline(prof, case, pk),
        "kernels": {k: {"launches": v[0], "ms_per_step": round(v[1] / 2, 4)} for k, v in prof.items()},
        "gpu_launches": int(launches),
        "e2e": e2e,
        "clocks": clocks,
        "l2": ("flushed before each timed step (256 MB write outside the events)" if flush is not None
               else "no flush: the step's tensors exceed 256 MB, twice the 126 MB L2"),
    }


def kernel_roofline(prof: dict, case, pk: dict, steps: int = 2) -> dict | None:
    """Roofline of the kernel with the largest share of device time.  `achieved` is the
    kernel's algorithmic work per launch over its measured launch time: the FLOPs of its
    products per token and value head (the method's steps, full 64-row tiles) times the
    launch's token-heads, against the bf16 tensor peak.  The method's algorithmic bytes do not
    count the chunk intermediates that pass between kernels, and the chunk kernels' inputs
    are mostly such intermediates, so their binding bound is the tensor peak.  The bytes the
    kernel moves under the current kernel split (intermediates included) are reported
    beside it as `hbm_with_intermediates`.  `prof` covers `steps` steps; a kernel launched
    several times per step (one launch per segment of the chunks) does its step's work in
    those launches together, so a launch's work is the step's divided by its launches."""
    if not prof:
        return None
    name, (launches, total_ms) = max(prof.items(), key=lambda kv: kv[1][1])
    per_launch_s = total_ms / launches / 1e3
    per_step = launches / steps  # launches per step
    fl = kernel_flops_per_token_head(case.K, case.V).get(name)
    th = case.tokens * case.HV / per_step  # token-heads of one launch
    e = 2 if case.dtype == "bf16" else 4
    units = chunks_of(case) * case.HV / per_step
    by = kernel_bytes_per_unit(case.K, case.V, case.HV // case.H, e).get(name)
    out = {"kernel": name, "launch_ms": round(per_launch_s * 1e3, 4),
           "share": round(total_ms / sum(v[1] for v in prof.values()), 4),
           "units_per_launch": round(units, 1), "launches_per_step": per_step}
    traffic = _traffic(name, case, units)
    if fl is not None and name.startswith("ffma_"):
        achieved = fl * th / per_launch_s / 1e12
        peak = FP32_ALU_TFLOPS
        out.update({"bound": "alu", "achieved": round(achieved, 3), "peak": round(peak, 1),
                    "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                    "peak_source": "fp32 FFMA: 148 SM x 128 lanes x 2 FLOP x 1.965 GHz"})
        return out
    if fl is not None:
        achieved = fl * th / per_launch_s / 1e12
        out.update({"bound": "tensor", "achieved": round(achieved, 3), "peak": pk["bf16_tflops"],
                    "unit": "TFLOP/s", "frac": round(achieved / pk["bf16_tflops"], 4),
                    "frac_sustained_peak": round(achieved / pk.get("bf16_tflops_sustained",
                                                                    pk["bf16_tflops"]), 4),
                    "flops_per_token_head": fl, "flops_per_launch": int(fl * th),
                    "traffic": traffic,
                    "peak_source": f"bf16 dense burst, {pk['source']}"})
    if by is not None:
        gbs = by * units / per_launch_s / 1e9
        out["hbm_with_intermediates"] = {
            "bytes_per_unit": int(by), "bytes_per_launch": int(by * units), "achieved": round(gbs, 1),
            "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": round(gbs / pk["hbm_gbs"], 4),
            "note": "tiles this kernel reads and writes once under the current kernel split, "
                    "inter-kernel intermediates included (not the method's algorithmic bytes)"}
    return out


def chunks_of(case) -> int:
    """64-token chunks of the workload (sequences never share a chunk)."""
    if case.cu_seqlens is not None:
        cu = case.cu_seqlens.tolist()
        return sum((cu[i + 1] - cu[i] + C - 1) // C for i in range(len(cu) - 1))
    return case.B * ((case.T + C - 1) // C)


def _traffic(name: str, case, units_per_launch: float):
    """DRAM bytes per launch (read + write) from the committed one-kernel ncu captures, when they
    cover this kernel at this head shape: measured bytes per unit x the units of one launch."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        shape = d.get("shape", {})
        if (shape.get("K"), shape.get("V"), shape.get("G"), shape.get("dtype")) != (
                case.K, case.V, case.HV // case.H, case.dtype):
            return None
        rec = d.get("kernels", {}).get(name)
        if rec:
            return int(rec["bytes_per_unit"] * units_per_launch)
    except (OSError, ValueError, KeyError):
        pass
    return None


def e2e_measure(gdn, case, dev, ws, nsteps: int, dist) -> dict:
    """Same step through the public API, with every step's inputs copied from pinned host
    memory and every output copied back to pinned host memory inside the timed region.
    Steps are pipelined the way a training loop overlaps I/O: step i+1's host-to-device
    copies, step i's kernels and step i-1's device-to-host copies run on three streams,
    with double-buffered device tensors and events ordering each buffer's reuse."""
    pin = lambda x: None if x is None else x.contiguous().pin_memory()
    host_in = dict(q=pin(case.q), k=pin(case.k), v=pin(case.v), g_raw=pin(case.a), A_log=pin(case.A_log),
                   dt_bias=pin(case.dt_bias), beta=pin(case.beta), cu_seqlens=pin(case.cu_seqlens),
                   initial_state=pin(case.h0), d_o=pin(case.dO), dht=pin(case.dht))
    NB = 2
    dev_in = [{k: (None if v is None else torch.empty_like(v, device=dev)) for k, v in host_in.items()}
              for _ in range(NB)]

    def outs_like(di):
        ht = torch.empty((case.N, case.HV, case.K, case.V), dtype=torch.float32, device=dev)
        return dict(o=torch.empty_like(di["v"]), ht=ht, dq=torch.empty_like(di["q"]),
                    dk=torch.empty_like(di["k"]), dv=torch.empty_like(di["v"]),
                    dg=torch.empty_like(di["g_raw"]), dbeta=torch.empty_like(di["beta"]),
                    dh0=torch.empty_like(ht))

    dev_out = [outs_like(dev_in[b]) for b in range(NB)]
    host_out = [{k: torch.empty_like(v, device="cpu").pin_memory() for k, v in dev_out[0].items()}
                for _ in range(NB)]
    h2d = sum(v.numel() * v.element_size() for v in host_in.values() if v is not None)
    d2h = sum(v.numel() * v.element_size() for v in host_out[0].values())
    s_in, s_run, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    loaded = [ev() for _ in range(NB)]      # inputs of buffer b on the device
    consumed = [ev() for _ in range(NB)]    # kernels done with buffer b's inputs and outputs written
    drained = [ev() for _ in range(NB)]     # outputs of buffer b copied back
    for b in range(NB):  # nothing to wait for before the first use of each buffer
        for e_ in (consumed[b], drained[b]):
            e_.record(s_out)

    def upload(b):
        with torch.cuda.stream(s_in):
            s_in.wait_event(consumed[b])
            for k, v in host_in.items():
                if v is not None:
                    dev_in[b][k].copy_(v, non_blocking=True)
            loaded[b].record(s_in)

    def run(b):
        with torch.cuda.stream(s_run):
            s_run.wait_event(loaded[b])
            s_run.wait_event(drained[b])
            di, do = dev_in[b], dev_out[b]
            fw = {k: di[k] for k in ("q", "k", "v", "g_raw", "A_log", "dt_bias", "beta",
                                     "cu_seqlens", "initial_state")}
            gdn.gdn_chunk_fwd(**fw, workspace=ws, out=do["o"], final_state=do["ht"])
            gdn.gdn_chunk_bwd(**fw, d_o=di["d_o"], dht=di["dht"], workspace=ws,
                              outs={k: do[k] for k in ("dq", "dk", "dv", "dg", "dbeta", "dh0")},
                              want_param_grads=False, reuse_forward=True)
            consumed[b].record(s_run)

    def download(b):
        with torch.cuda.stream(s_out):
            s_out.wait_event(consumed[b])
            for k, v in dev_out[b].items():
                host_out[b][k].copy_(v, non_blocking=True)
            drained[b].record(s_out)

    def pipeline(n, t0=None):
        upload(0)
        for i in range(n):
            b = i % NB
            if i + 1 < n:
                upload((i + 1) % NB)
            run(b)
            download(b)

    pipeline(2)  # warm-up
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    pipeline(nsteps)
    s_in.wait_stream(s_out)
    z.record(s_in)
    torch.cuda.synchronize()
    ms = a.elapsed_time(z) / nsteps
    (ms,) = max_over_ranks([ms], dist, dev)
    world = dist.get_world_size() if dist else 1
    return {"value": round(aggregate_mtok_s(world, case.tokens, ms), 3), "unit": "M tokens/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(ms, 3), "steps": nsteps,
            "pipelined": "copies of step i+1 in, step i's kernels, step i-1 out on three streams; "
                         "the first step's upload and the last step's download are inside the timed "
                         "region (fill and drain)"}


DECODE = dict(B=256, H=16, HV=32, K=128, V=128)


def decode_measure(gdn, dev, pk_hbm: float, steps: int = 20, kda: bool = False) -> dict:
    """One decode step (T = 1) of 256 sequences with the layer's heads, through
    gdn_recurrent_fwd (or, with kda, gdn_kda_recurrent_fwd: a gate per key channel) with the
    state updated in place: HBM-bound on the fp32 state, read and written once per (sequence,
    value head).  A secondary measurement beside the training step."""
    c = DECODE
    case = synth.make_case(B=c["B"], T=1, H=c["H"], HV=c["HV"], K=c["K"], V=c["V"], dtype="bf16",
                           seed=4242, h0=True, name="decode")
    t = lambda x: None if x is None else x.to(dev).contiguous()
    d = dict(q=t(case.q), k=t(case.k), v=t(case.v), g_raw=t(case.a), A_log=t(case.A_log),
             dt_bias=t(case.dt_bias), beta=t(case.beta))
    if kda:
        g_raw, A_log, dt_bias = synth.kda_gate_inputs(case, 4243)
        d.update(g_raw=t(g_raw), A_log=t(A_log), dt_bias=t(dt_bias))
    st = t(case.h0)
    o = torch.empty_like(d["v"])
    ws = torch.empty(gdn.recurrent_workspace_bytes(), dtype=torch.uint8, device=dev)
    fn = gdn.gdn_kda_recurrent_fwd if kda else gdn.gdn_recurrent_fwd

    def step():
        fn(**d, initial_state=st, final_state=st, out=o, workspace=ws)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    B, H, HV, K, V = c["B"], c["H"], c["HV"], c["K"], c["V"]
    gate = B * HV * K * 4 + HV * K * 4 + HV * 4 if kda else B * HV * 4 + HV * 8
    nbytes = B * HV * K * V * 4 * 2 + B * (2 * H * K + 2 * HV * V) * 2 + B * HV * 4 + gate
    gbs = nbytes / (ms / 1e3) / 1e9
    name = "kda_decode" if kda else "decode"
    return {"workload": f"{name}_B{B}_H{H}_HV{HV}_D{K}_bf16", "tokens_per_step": B,
            "ms_per_step": round(ms, 4), "mtok_s": round(B / (ms / 1e3) / 1e6, 3),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk_hbm, "unit": "GB/s",
                         "frac": round(gbs / pk_hbm, 4), "bytes_per_step": int(nbytes),
                         "note": "fp32 state read and written once per (sequence, value head)"}}


FFMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # fp32 lanes x 2 FLOP x max SM clock: 74.4


def kda_chunk_measure(gdn, dev, pk_hbm: float, steps: int = 5, T: int = 32768) -> dict:
    """Chunkwise KDA (per-key-channel gate) at the layer's shape: B = 1, T = 32768, H = 16,
    HV = 32, K = V = 128, bf16 tokens: the forward alone and a training step (forward +
    backward reading the forward's intermediates).  fp32 on CUDA cores, so the bound is the
    FFMA rate (FLOPs per (chunk, value head): forward A and P 0.53 M FMA, W and U~ 1.05 M, scan
    2.10 M, output 1.57 M)."""
    case = synth.make_case(B=1, T=T, H=16, HV=32, K=128, V=128, dtype="bf16", seed=4244,
                           h0=True, name="kda_chunk")
    g_raw, A_log, dt_bias = synth.kda_gate_inputs(case, 4245)
    t = lambda x: None if x is None else x.to(dev).contiguous()
    d = dict(q=t(case.q), k=t(case.k), v=t(case.v), g_raw=t(g_raw), A_log=t(A_log),
             dt_bias=t(dt_bias), beta=t(case.beta))
    h0, dO = t(case.h0), t(case.dO)
    dims = gdn.make_dims(d["q"], d["v"])
    ws = torch.empty(gdn.kda_chunk_workspace_bytes(dims, False, True), dtype=torch.uint8, device=dev)
    o = torch.empty_like(d["v"])
    ht = torch.empty_like(h0)
    outs = dict(dq=torch.empty_like(d["q"]), dk=torch.empty_like(d["k"]), dv=torch.empty_like(d["v"]),
                dbeta=torch.empty_like(d["beta"]), dg=torch.empty_like(d["g_raw"]), dh0=torch.empty_like(h0),
                dg_raw=torch.empty_like(d["g_raw"]), dA_log=torch.empty_like(d["A_log"]),
                ddt_bias=torch.empty_like(d["dt_bias"]))

    def fwd():
        gdn.gdn_kda_chunk_fwd(**d, initial_state=h0, out=o, final_state=ht, workspace=ws)

    def step():
        fwd()
        gdn.gdn_kda_chunk_bwd(**d, d_o=dO, workspace=ws, outs=outs)

    stream = torch.cuda.current_stream()

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / steps

    ms = timed(step)  # the step first: a capture of the first six KDA launches sees every kernel
    ms_f = timed(fwd)
    # the same forward token by token (the recurrent kernel), for comparison
    o2, ht2 = torch.empty_like(o), torch.empty_like(ht)
    wsr = torch.empty(gdn.recurrent_workspace_bytes(), dtype=torch.uint8, device=dev)
    ms_r = timed(lambda: gdn.gdn_kda_recurrent_fwd(**d, initial_state=h0, out=o2, final_state=ht2,
                                                   workspace=wsr))
    gdn.profile(True)
    step()
    prof = gdn.profile_read()
    gdn.profile(False)
    units = (T // 64) * 32
    K = V = 128
    # FMA per (chunk, value head) of each kernel's products
    fma = {"kda_wy": 2 * 1536 * K + 2 * 544 * K + 64 * 64 * K + 64 * 64 * V,
           "kda_scan": 64 * V * K + V * K * 64, "kda_out": 64 * V * 64 + 64 * V * K,
           "kda_bwd_scan": 64 * 64 * V + 3 * 64 * V * K,
           "kda_bwd_dqk": 64 * 64 * V + 3 * 64 * V * K + 2 * (1536 + 544) * K,
           "kda_bwd_wy": 2 * 64 * 64 * (K + V) + 2 * 64 * 64 * 64 + 2 * (1536 + 544) * K}
    kern = {k: round(v[1], 4) for k, v in prof.items()}
    # bf16 with 128-wide heads runs the tcgen05 kernels (kda_tc_*): same products, tensor peak
    step_of = {k: k.replace("kda_tc_", "kda_") for k in kern if k.replace("kda_tc_", "kda_") in fma}
    top = max(step_of, key=lambda k: kern[k])
    top_tf = 2 * units * fma[step_of[top]] / (kern[top] / 1e3) / 1e12
    tensor = top.startswith("kda_tc_")
    pk = peaks()
    peak = pk["bf16_tflops"] if tensor else FFMA_TFLOPS
    src = (f"bf16 dense burst, {pk['source']}" if tensor
           else "148 SMs x 128 fp32 lanes x 2 FLOP x 1965 MHz (FFMA)")
    return {"workload": f"kda_chunk_B1_T{T}_H16_HV32_D128_bf16", "fwd_ms": round(ms_f, 4),
            "fwd_mtok_s": round(T / (ms_f / 1e3) / 1e6, 3), "step_ms": round(ms, 4),
            "step_mtok_s": round(T / (ms / 1e3) / 1e6, 3), "recurrent_fwd_ms": round(ms_r, 4),
            "kernels_ms": kern,
            "step_tflops": round(2 * units * sum(fma.values()) / (ms / 1e3) / 1e12, 2),
            "roofline": {"kernel": top, "bound": "tensor" if tensor else "alu",
                         "achieved": round(top_tf, 2), "peak": round(peak, 1), "unit": "TFLOP/s",
                         "frac": round(top_tf / peak, 4), "peak_source": src}}


def kda_gate_measure(gdn, dev, pk_hbm: float, steps: int = 20) -> dict:
    """The KDA gate at the layer's token count and heads (T = 32768, H = 16, D = 128, dt_bias
    on): forward bf16 g -> fp32 yg, and backward (bf16 g, fp32 dyg -> bf16 dg and the two
    parameter sums).  Both are element-wise and HBM-bound; each input (>= 134 MB) exceeds L2."""
    T, H, D = 32768, 16, 128
    gen = torch.Generator().manual_seed(77)
    g = torch.randn(T, H, D, generator=gen).to(torch.bfloat16).to(dev)
    A_log = torch.randn(H, generator=gen).to(dev)
    dt_bias = torch.randn(H * D, generator=gen).to(dev)
    dyg = torch.randn(T, H, D, generator=gen).to(dev)
    yg = torch.empty(T, H, D, dtype=torch.float32, device=dev)
    ws = torch.empty(gdn.kda_gate_workspace_bytes(T, H, D), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / steps

    ms_f = timed(lambda: gdn.kda_gate_fwd(g, A_log, dt_bias, output_dtype=torch.float32, out=yg))
    ms_b = timed(lambda: gdn.kda_gate_bwd(g, A_log, dyg, dt_bias, workspace=ws))
    n = T * H * D
    part = 128 * 2 * H * D * 4 * 2  # row-block partials, written then read
    bytes_f, bytes_b = n * (2 + 4), n * (2 + 4 + 2) + part
    roof = lambda nb, ms: {"bound": "hbm", "achieved": round(nb / (ms / 1e3) / 1e9, 1), "peak": pk_hbm,
                           "unit": "GB/s", "frac": round(nb / (ms / 1e3) / 1e9 / pk_hbm, 4),
                           "bytes_per_call": int(nb)}
    return {"workload": f"kda_gate_T{T}_H{H}_D{D}_bf16in", "fwd_ms": round(ms_f, 4),
            "bwd_ms": round(ms_b, 4), "fwd_roofline": roof(bytes_f, ms_f),
            "bwd_roofline": roof(bytes_b, ms_b)}


# ----------------------------------------------------------------- reference arm (oracle)
def reference_arm(args, rank, world, dist):
    if rank != 0:
        if dist:
            dist.destroy_process_group()
        return
    case = synth.config_case(args.config, seed=1000 + args.config)
    from oracle import oracle
    oracle.build()
    budget = max(0.5, args.ref_budget / max(1, args.steps + args.warmup))
    info = None
    secs, toks = [], []
    for i in range(args.warmup + args.steps):
        info = oracle_sample(case, budget_s=budget)
        if i >= args.warmup:
            secs.append(info["seconds"])
            toks.append(info["tokens"])
    # one step = one bounded sample of the workload; the time is the measured time of it
    ms = 1e3 * statistics.mean(secs)
    tokens_per_step = int(statistics.mean(toks))
    value = tokens_per_step / (ms / 1e3) / 1e6
    cpu = {k: info[k] for k in ("unit", "cores", "kind", "sample")}
    cpu["value"] = round(value, 6)
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "M tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 3), "tokens_per_step": tokens_per_step,
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": case.name, "B": case.B, "T": case.T, "H": case.H, "HV": case.HV,
                       "K": case.K, "V": case.V, "chunk": C},
            "cpu_baseline": cpu,
            "e2e": {"value": round(value, 6), "unit": "M tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "note": "the reference arm is the fp64 token-by-token oracle on the host cores; each "
                    "step is a bounded sample of the workload (tokens_per_step tokens, all heads) "
                    "and ms_per_step its measured time"}
    print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
