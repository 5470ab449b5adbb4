"""ctypes wrapper around the fp64 token-by-token Gated DeltaNet oracle (gdn_oracle.cpp).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the bench's
CPU-baseline leg call this module; the product path never does.  It imports nothing
from the CUDA library package and the library imports nothing from here.

Every array is converted to contiguous float64 before the call; bf16 inputs are
widened exactly.  Layouts follow the library's documented ones:
q,k [B,T,H,K]; v,o,dO [B,T,HV,V]; a (raw gate input), beta [B,T,HV]; A_log, dt_bias [HV];
states [Nst,HV,K,V] with h[k][v] = S[v][k].
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

FLAG_NO_ERASE = 1  # test-only: plain gated linear attention (no delta-rule erase)


def build(force: bool = False) -> str:
    """Compile the oracle with the host C++ compiler (g++ -O2, fp64, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-pthread",
                               "-fno-fast-math", _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64, dbl, ptr, i32 = ctypes.c_int64, ctypes.c_double, ctypes.c_void_p, ctypes.c_int
            lib.oracle_gdn_fwd.argtypes = [i64] * 7 + [dbl] + [ptr] * 12 + [i32, i32]
            lib.oracle_gdn_fwd.restype = i32
            lib.oracle_gdn_bwd.argtypes = [i64] * 7 + [dbl] + [ptr] * 20 + [i32, i32]
            lib.oracle_gdn_bwd.restype = i32
            lib.oracle_gate.argtypes = [ptr, i64, dbl, dbl, ptr]
            lib.oracle_gate.restype = None
            _lib = lib
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: every float dtype widened exactly to float64
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(x):
    return None if x is None else x.ctypes.data_as(ctypes.c_void_p)


def gate(a, A_log: float, dt_bias: float) -> np.ndarray:
    """g = -exp(A_log) * softplus(a + dt_bias), softplus passing x through for x > 20."""
    a = _f64(a).ravel()
    out = np.empty_like(a)
    _load().oracle_gate(_p(a), a.size, float(A_log), float(dt_bias), _p(out))
    return out


def _dims(q, v, cu):
    B, T, H, K = q.shape
    HV, V = v.shape[2], v.shape[3]
    N = (len(cu) - 1) if cu is not None else B
    return B, T, H, HV, K, V, N


def fwd(q, k, v, a, A_log, dt_bias, beta, scale=None, cu_seqlens=None, h0=None,
        flags: int = 0, nthreads: int = 0):
    """Forward: returns (o [B,T,HV,V], h_final [Nst,HV,K,V], g [B,T,HV]) in float64."""
    q, k, v, a, A_log, dt_bias, beta, h0 = map(_f64, (q, k, v, a, A_log, dt_bias, beta, h0))
    cu = None if cu_seqlens is None else np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    B, T, H, HV, K, V, N = _dims(q, v, cu)
    if scale is None:
        scale = K ** -0.5
    o = np.zeros((B, T, HV, V))
    ht = np.zeros((N, HV, K, V))
    g = np.zeros((B, T, HV))
    rc = _load().oracle_gdn_fwd(B, T, H, HV, K, V, N, float(scale), _p(q), _p(k), _p(v), _p(a),
                                _p(A_log), _p(dt_bias), _p(beta), _p(cu), _p(h0), _p(o), _p(ht),
                                _p(g), int(flags), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_gdn_fwd rejected its arguments")
    return o, ht, g


def bwd(q, k, v, a, A_log, dt_bias, beta, dO, scale=None, cu_seqlens=None, h0=None, dht=None,
        flags: int = 0, nthreads: int = 0):
    """Backward of L = sum(dO*o) + sum(dht*h_final).

    Returns a dict with dq, dk [B,T,H,K]; dv [B,T,HV,V]; dg, dbeta, da [B,T,HV];
    dh0 [Nst,HV,K,V]; dA_log, ddt_bias [HV]   (all float64).
    """
    q, k, v, a, A_log, dt_bias, beta, dO, h0, dht = map(
        _f64, (q, k, v, a, A_log, dt_bias, beta, dO, h0, dht))
    cu = None if cu_seqlens is None else np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    B, T, H, HV, K, V, N = _dims(q, v, cu)
    if scale is None:
        scale = K ** -0.5
    out = dict(dq=np.zeros((B, T, H, K)), dk=np.zeros((B, T, H, K)), dv=np.zeros((B, T, HV, V)),
               dg=np.zeros((B, T, HV)), dbeta=np.zeros((B, T, HV)), da=np.zeros((B, T, HV)),
               dh0=np.zeros((N, HV, K, V)), dA_log=np.zeros(HV), ddt_bias=np.zeros(HV))
    rc = _load().oracle_gdn_bwd(B, T, H, HV, K, V, N, float(scale), _p(q), _p(k), _p(v), _p(a),
                                _p(A_log), _p(dt_bias), _p(beta), _p(cu), _p(h0), _p(dO), _p(dht),
                                _p(out["dq"]), _p(out["dk"]), _p(out["dv"]), _p(out["dg"]),
                                _p(out["dbeta"]), _p(out["da"]), _p(out["dh0"]),
                                _p(out["dA_log"]), _p(out["ddt_bias"]), int(flags), int(nthreads))
    if rc != 0:
        raise ValueError("oracle_gdn_bwd rejected its arguments")
    return out
