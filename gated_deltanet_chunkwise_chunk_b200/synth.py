"""Seeded synthetic inputs for the chunkwise Gated DeltaNet workloads.

This module holds no arithmetic of the method itself (no gate, no recurrence, no chunk
algebra): it only draws the inputs, in the shapes and value distributions of the
workloads, so that the CUDA library and the fp64 oracle read identical bytes.

Distributions (names follow the flash-linear-attention gated delta rule API):
  q, k   ~ N(0,1), then L2-normalised over the head dimension, then cast to the dtype
  v, dO  ~ N(0,1), cast to the dtype
  beta   = sigmoid(N(0,1))                  [B,T,HV] fp32
  a      ~ N(0,1)   (raw gate input)         [B,T,HV] fp32
  A_log  = log(U(1,16))                     [HV]     fp32
  dt_bias~ N(0, 0.5) (0.5 is the std)         [HV]     fp32
  h0, dht~ N(0, 0.1) when requested          [Nst,HV,K,V] fp32
Optional extras: ``big_a`` replaces a seeded 1/256 of ``a`` by U(20.5,40) and another
1/256 by U(-40,-20.5) (exercises the softplus pass-through branch x > 20 and the
underflow side); ``long_memory`` draws A_log = log U(0.01,0.1) and dt_bias = -4 so the
per-token decay is tiny and the state carries information across many chunks.

All randomness comes from numpy's PCG64 generator seeded with the case seed.
bf16 rounding is round-to-nearest-even, done once here.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

CHUNK = 64

# The five workloads (seed = 1000 + index).
CONFIGS = {
    0: dict(name="fp32_B1_T512_H4_HV4_D64", dtype="fp32", B=1, T=512, H=4, HV=4, K=64, V=64,
            h0=False, dht=False),
    1: dict(name="bf16_B2_T2048_H4_HV8_D128", dtype="bf16", B=2, T=2048, H=4, HV=8, K=128, V=128,
            h0=False, dht=False),
    2: dict(name="bf16_B1_T32768_H16_HV32_D128_h0", dtype="bf16", B=1, T=32768, H=16, HV=32,
            K=128, V=128, h0=True, dht=True),
    3: dict(name="bf16_varlen32_H16_HV32_D128", dtype="bf16", B=1, T=None, H=16, HV=32, K=128,
            V=128, h0=False, dht=True, nseq=32, len_lo=257, len_hi=4095),
    4: dict(name="bf16_B8_T8192_H16_HV16_D128_h0_bigA", dtype="bf16", B=8, T=8192, H=16, HV=16,
            K=128, V=128, h0=True, dht=True, big_a=True),
}


@dataclass
class Case:
    """One seeded problem.  Tensors are CPU torch tensors in the library's layouts."""
    B: int
    T: int
    H: int
    HV: int
    K: int
    V: int
    dtype: str                      # "bf16" or "fp32" (q,k,v,o,dO,dq,dk,dv)
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    a: torch.Tensor                 # raw gate input g_raw [B,T,HV] fp32
    A_log: torch.Tensor
    dt_bias: torch.Tensor
    beta: torch.Tensor
    dO: torch.Tensor
    cu_seqlens: torch.Tensor | None = None   # int64 [N+1]
    h0: torch.Tensor | None = None
    dht: torch.Tensor | None = None
    seed: int = 0
    name: str = ""
    extras: dict = field(default_factory=dict)

    @property
    def N(self) -> int:
        return (len(self.cu_seqlens) - 1) if self.cu_seqlens is not None else self.B

    @property
    def tokens(self) -> int:
        return self.B * self.T

    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


def varlen_lengths(rng: np.random.Generator, n: int, lo: int, hi: int) -> list[int]:
    """n lengths uniform in [lo, hi], redrawn while a length is a multiple of the chunk."""
    out = []
    while len(out) < n:
        x = int(rng.integers(lo, hi + 1))
        if x % CHUNK:
            out.append(x)
    return out


def _normal(rng, shape, std=1.0):
    return (rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std))


def _l2norm_lastdim(x: np.ndarray) -> np.ndarray:
    n = np.sqrt((x.astype(np.float64) ** 2).sum(-1, keepdims=True))
    return (x / np.maximum(n, 1e-12)).astype(np.float32)


def make_case(B=1, T=64, H=1, HV=1, K=64, V=64, dtype="fp32", seed=0, lengths=None,
              h0=False, dht=False, big_a=False, long_memory=False, name="") -> Case:
    """Draw one seeded case.  ``lengths`` packs len(lengths) sequences into B=1 (varlen)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    cu = None
    if lengths is not None:
        B = 1
        T = int(sum(lengths))
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64))
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q = _l2norm_lastdim(_normal(rng, (B, T, H, K)))
    k = _l2norm_lastdim(_normal(rng, (B, T, H, K)))
    v = _normal(rng, (B, T, HV, V))
    beta = (1.0 / (1.0 + np.exp(-_normal(rng, (B, T, HV)).astype(np.float64)))).astype(np.float32)
    a = _normal(rng, (B, T, HV))
    if long_memory:
        A_log = np.log(rng.uniform(0.01, 0.1, size=HV)).astype(np.float32)
        dt_bias = np.full(HV, -4.0, dtype=np.float32)
    else:
        A_log = np.log(rng.uniform(1.0, 16.0, size=HV)).astype(np.float32)
        dt_bias = _normal(rng, (HV,), 0.5)
    if big_a:
        flat = a.reshape(-1)
        n = flat.size
        m = max(1, n // 256)
        idx = rng.permutation(n)[: 2 * m]
        flat[idx[:m]] = rng.uniform(20.5, 40.0, size=m).astype(np.float32)
        flat[idx[m:]] = rng.uniform(-40.0, -20.5, size=m).astype(np.float32)
    dO = _normal(rng, (B, T, HV, V))
    Nst = (len(lengths) if lengths is not None else B)
    h0_t = torch.from_numpy(_normal(rng, (Nst, HV, K, V), 0.1)) if h0 else None
    dht_t = torch.from_numpy(_normal(rng, (Nst, HV, K, V), 0.1)) if dht else None
    return Case(B=B, T=T, H=H, HV=HV, K=K, V=V, dtype=dtype,
                q=torch.from_numpy(q).to(tdt), k=torch.from_numpy(k).to(tdt),
                v=torch.from_numpy(v).to(tdt), a=torch.from_numpy(a),
                A_log=torch.from_numpy(A_log), dt_bias=torch.from_numpy(dt_bias),
                beta=torch.from_numpy(beta), dO=torch.from_numpy(dO).to(tdt),
                cu_seqlens=cu, h0=h0_t, dht=dht_t, seed=seed, name=name)


def kda_gate_inputs(case: Case, seed: int, with_bias: bool = True, long_memory: bool = False):
    """Per-key-channel gate inputs for the KDA form of a case: g_raw [B,T,HV,K] ~ N(0,1) and
    dt_bias [HV*K] ~ N(0, 0.5) (or None), with the case's A_log; ``long_memory`` gives
    A_log = log U(0.01, 0.1) and dt_bias = -4 as for the scalar gate.  Returns
    (g_raw, A_log, dt_bias) as fp32 CPU tensors."""
    rng = np.random.Generator(np.random.PCG64(seed))
    g = _normal(rng, (case.B, case.T, case.HV, case.K))
    if long_memory:
        A_log = np.log(rng.uniform(0.01, 0.1, size=case.HV)).astype(np.float32)
        dtb = np.full(case.HV * case.K, -4.0, dtype=np.float32)
    else:
        A_log = case.A_log.numpy()
        dtb = _normal(rng, (case.HV * case.K,), 0.5)
    return (torch.from_numpy(g), torch.from_numpy(np.ascontiguousarray(A_log)),
            torch.from_numpy(dtb) if with_bias else None)


def config_case(idx: int, seed: int | None = None, T: int | None = None) -> Case:
    """The seeded case of workload ``idx`` (seed defaults to 1000 + idx).  ``T`` overrides
    the sequence length of a dense workload (a smaller case of the same shape)."""
    c = dict(CONFIGS[idx])
    if T is not None:
        if c.get("nseq"):
            raise ValueError("T applies to dense workloads only")
        c["T"] = T
        c["name"] = c["name"].replace(f"_T{CONFIGS[idx]['T']}_", f"_T{T}_")
    seed = 1000 + idx if seed is None else seed
    lengths = None
    if c.get("nseq"):
        rng = np.random.Generator(np.random.PCG64(seed + 7919))
        lengths = varlen_lengths(rng, c["nseq"], c["len_lo"], c["len_hi"])
    return make_case(B=c["B"], T=c["T"], H=c["H"], HV=c["HV"], K=c["K"], V=c["V"],
                     dtype=c["dtype"], seed=seed, lengths=lengths, h0=c["h0"], dht=c["dht"],
                     big_a=c.get("big_a", False), name=c["name"])


def subset_heads(case: Case, kheads: list[int]) -> Case:
    """The same problem restricted to some k-heads and their value heads (heads are
    independent problems, so this is how one checks sampled outputs at full size)."""
    G = case.HV // case.H
    vh = [h * G + j for h in kheads for j in range(G)]
    sel = lambda t, ax, idx: None if t is None else t.index_select(ax, torch.tensor(idx))
    return Case(B=case.B, T=case.T, H=len(kheads), HV=len(vh), K=case.K, V=case.V,
                dtype=case.dtype, q=sel(case.q, 2, kheads), k=sel(case.k, 2, kheads),
                v=sel(case.v, 2, vh), a=sel(case.a, 2, vh), A_log=sel(case.A_log, 0, vh),
                dt_bias=sel(case.dt_bias, 0, vh), beta=sel(case.beta, 2, vh),
                dO=sel(case.dO, 2, vh), cu_seqlens=case.cu_seqlens, h0=sel(case.h0, 1, vh),
                dht=sel(case.dht, 1, vh), seed=case.seed, name=case.name + f"[k{kheads}]")
