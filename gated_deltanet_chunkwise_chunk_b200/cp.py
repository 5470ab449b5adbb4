"""Context parallelism over T: a dense batch of sequences split along time into one contiguous
segment per rank, with one exchange of per-segment state summaries.

Every step of the recurrence maps the state linearly (S_t = e^{g_t} S_{t-1} (I - beta_t k_t k_t^T)
+ beta_t v_t k_t^T), so a whole segment maps the state entering it affinely.  In the [K][V] layout
of the library's states,
    h_end = Mt h_start + Bh,
with Mt (K x K) the final state the segment's forward returns from h_start = I with v = 0
(K = V) and Bh the one it returns from h_start = 0.  Forward on rank r: compute (Mt_r, Bh_r),
all-gather them, fold h_start = Mt_{r-1}(... (Mt_0 h0 + Bh_0) ...) + Bh_{r-1}, then run the
segment's forward from h_start.  Backward: with D_r the gradient entering the segment when
nothing leaves it (dh0 of the backward with dht = 0), the gradient leaving segment r is
    dht_r = Mt_{r+1}^T (... (Mt_{N-1}^T dht + D_{N-1}) ...) + D_{r+1};
all-gather the D_r, fold, run the segment's backward with dht_r, and all-reduce the gradients
of the shared gate parameters (A_log, dt_bias).

This module is plumbing: the per-rank computations run in the library's kernels (Ops), the
exchange goes through torch.distributed (DistExchange).  Both are injectable, so the algebra
can be driven one rank at a time in one process and the collectives tested on CPU ranks.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


class Ops:
    """The per-rank computations, in the library's kernels."""

    def __init__(self):
        from . import binding
        self.b = binding

    def fwd(self, q, k, v, g_raw, A_log, dt_bias, beta, h0, workspace=None):
        return self.b.gdn_chunk_fwd(q, k, v, g_raw, A_log, dt_bias, beta, initial_state=h0,
                                    workspace=workspace)

    def bwd(self, q, k, v, g_raw, A_log, dt_bias, beta, h0, d_o, dht, workspace):
        return self.b.gdn_chunk_bwd(q, k, v, g_raw, A_log, dt_bias, beta, d_o, initial_state=h0,
                                    dht=dht, workspace=workspace, reuse_forward=True)

    def affine(self, A, X, B=None, transpose=False):
        return self.b.state_affine(A, X, B, transpose=transpose)

    def workspace(self, q, v):
        dims = self.b.make_dims(q, v)
        n = max(self.b.workspace_bytes(dims, False, False), self.b.workspace_bytes(dims, False, True))
        return torch.empty(n, dtype=torch.uint8, device=q.device)


class DistExchange:
    """All-gather and all-reduce over a torch.distributed group (NCCL on GPUs, gloo on CPU)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def all_gather(self, t):
        out = [torch.empty_like(t) for _ in range(self.world)]
        self.dist.all_gather(out, t.contiguous(), group=self.group)
        return out

    def all_reduce_sum(self, t):
        self.dist.all_reduce(t, op=self.dist.ReduceOp.SUM, group=self.group)
        return t


@dataclass
class Context:
    Mts: list          # every rank's Mt, [B, HV, K, K]
    h_start: torch.Tensor
    workspace: object


def segment_summary(ops, q, k, v, g_raw, A_log, dt_bias, beta):
    """(Mt, Bh) of this segment: the final states from h_start = I with v = 0, and from 0."""
    B, HV, K, V = q.shape[0], v.shape[2], q.shape[3], v.shape[3]
    if K != V:
        raise ValueError("context parallelism needs K == V (the segment map is read from an identity state)")
    eye = torch.eye(K, dtype=torch.float32, device=q.device).expand(B, HV, K, K).contiguous()
    _, Mt = ops.fwd(q, k, torch.zeros_like(v), g_raw, A_log, dt_bias, beta, eye)
    _, Bh = ops.fwd(q, k, v, g_raw, A_log, dt_bias, beta, None)
    return Mt, Bh


def start_state(ops, Mts, Bhs, rank, h0):
    """State entering segment `rank`: the segments before it applied to h0 in order."""
    h = h0 if h0 is not None else torch.zeros_like(Bhs[0])
    for j in range(rank):
        h = ops.affine(Mts[j], h, Bhs[j])
    return h


def end_gradient(ops, Mts, Ds, rank, dht):
    """Gradient leaving segment `rank`: the segments after it, last first, applied to dht."""
    world = len(Mts)
    g = dht if dht is not None else torch.zeros_like(Ds[0])
    for j in range(world - 1, rank, -1):
        g = ops.affine(Mts[j], g, Ds[j], transpose=True)
    return g


def cp_forward(q, k, v, g_raw, A_log, dt_bias, beta, initial_state, exchange, ops=None):
    """This rank's segment: returns (o, h_end, ctx).  h_end on the last rank is the final state
    of the whole sequences; initial_state (the state before the first segment) is read on
    every rank and may be None."""
    ops = ops or Ops()
    Mt, Bh = segment_summary(ops, q, k, v, g_raw, A_log, dt_bias, beta)
    Mts, Bhs = exchange.all_gather(Mt), exchange.all_gather(Bh)
    h = start_state(ops, Mts, Bhs, exchange.rank, initial_state)
    ws = ops.workspace(q, v)
    o, ht = ops.fwd(q, k, v, g_raw, A_log, dt_bias, beta, h, workspace=ws)
    return o, ht, Context(Mts, h, ws)


def cp_backward(q, k, v, g_raw, A_log, dt_bias, beta, d_o, dht, ctx, exchange, ops=None):
    """Gradients of this rank's segment for sum(d_o * o) + sum(dht * final state); dht (the
    gradient of the whole sequences' final state, may be None) is read on every rank.  dh0 on
    rank 0 is the gradient of initial_state; dA_log and ddt_bias are summed over the ranks."""
    ops = ops or Ops()
    D = ops.bwd(q, k, v, g_raw, A_log, dt_bias, beta, ctx.h_start, d_o, None, ctx.workspace)["dh0"]
    Ds = exchange.all_gather(D)
    g_end = end_gradient(ops, ctx.Mts, Ds, exchange.rank, dht)
    grads = ops.bwd(q, k, v, g_raw, A_log, dt_bias, beta, ctx.h_start, d_o, g_end, ctx.workspace)
    for name in ("dA_log", "ddt_bias"):
        if grads.get(name) is not None:
            exchange.all_reduce_sum(grads[name])
    return grads
