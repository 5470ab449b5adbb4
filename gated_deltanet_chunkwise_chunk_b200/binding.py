"""Thin ctypes binding of libgdn_b200.so (include/gdn.h).

Argument marshalling only: it checks torch tensors (device, dtype, contiguity, shape),
allocates outputs and the workspace with torch, and passes raw pointers plus the current
CUDA stream to the C entry points of the same names.  Every step of the computation runs
in the library's CUDA kernels.  There is no fallback: the shared library is loaded on the
first call into it (so that processes which only use the seeded input generators never map
it), and that call raises if the library is missing.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn_b200.so")

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_WORKSPACE, GDN_ERR_CUDA, GDN_ERR_TIMEOUT = range(6)
GDN_DTYPE_FP32, GDN_DTYPE_BF16, GDN_DTYPE_FP16 = 0, 1, 2
GDN_FLAG_BWD_REUSE_FWD = 1
GDN_FLAG_TEST_WAIT_TIMEOUT = 1 << 30  # tests of the failure path only

# Every symbol include/gdn.h declares (checked by the tests).
EXPORTED = ("gdn_workspace_bytes", "gdn_chunk_fwd", "gdn_chunk_bwd", "gdn_max_chunks",
            "gdn_build_chunk_indices", "gdn_chunk_table_device", "gdn_device_status",
            "gdn_status_string", "gdn_version", "gdn_launch_count", "gdn_profile",
            "gdn_profile_read", "gdn_chunk_fwd_noalloc", "gdn_noalloc_scratch_bytes", "gdn_noalloc_device_status",
            "gdn_recurrent_fwd", "gdn_recurrent_workspace_bytes", "gdn_kda_gate_fwd",
            "gdn_kda_gate_bwd", "gdn_kda_gate_workspace_bytes", "gdn_kda_recurrent_fwd",
            "gdn_kda_chunk_fwd", "gdn_kda_chunk_bwd", "gdn_kda_chunk_workspace_bytes",
            "gdn_state_affine")


class gdn_dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("T", ctypes.c_int64), ("H", ctypes.c_int64),
                ("HV", ctypes.c_int64), ("K", ctypes.c_int64), ("V", ctypes.c_int64),
                ("N", ctypes.c_int64), ("dtype", ctypes.c_int32), ("scale", ctypes.c_float),
                ("flags", ctypes.c_int32)]


class GDNError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python gated_deltanet_chunkwise_chunk_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    D = ctypes.POINTER(gdn_dims)
    lib.gdn_workspace_bytes.argtypes = [D, I32, I32]
    lib.gdn_workspace_bytes.restype = SZ
    lib.gdn_chunk_fwd.argtypes = [D] + [P] * 12 + [SZ, P]
    lib.gdn_chunk_fwd.restype = I32
    lib.gdn_chunk_bwd.argtypes = [D] + [P] * 21 + [SZ, P]
    lib.gdn_chunk_bwd.restype = I32
    lib.gdn_recurrent_fwd.argtypes = [D] + [P] * 12 + [SZ, P]
    lib.gdn_recurrent_fwd.restype = I32
    lib.gdn_kda_chunk_fwd.argtypes = [D] + [P] * 12 + [SZ, P]
    lib.gdn_kda_chunk_fwd.restype = I32
    lib.gdn_state_affine.argtypes = [I64, I64, I64, P, I32, P, P, P, P]
    lib.gdn_state_affine.restype = I32
    lib.gdn_kda_chunk_bwd.argtypes = [D] + [P] * 20 + [SZ, P]
    lib.gdn_kda_chunk_bwd.restype = I32
    lib.gdn_kda_chunk_workspace_bytes.argtypes = [D, I32, I32]
    lib.gdn_kda_chunk_workspace_bytes.restype = SZ
    lib.gdn_kda_recurrent_fwd.argtypes = [D] + [P] * 12 + [SZ, P]
    lib.gdn_kda_recurrent_fwd.restype = I32
    lib.gdn_recurrent_workspace_bytes.argtypes = []
    lib.gdn_recurrent_workspace_bytes.restype = SZ
    lib.gdn_kda_gate_fwd.argtypes = [I64, I64, I64, I32, P, P, P, I32, P, P]
    lib.gdn_kda_gate_fwd.restype = I32
    lib.gdn_kda_gate_bwd.argtypes = [I64, I64, I64, I32, P, P, P, I32, P, P, P, P, P, SZ, P]
    lib.gdn_kda_gate_bwd.restype = I32
    lib.gdn_kda_gate_workspace_bytes.argtypes = [I64, I64, I64]
    lib.gdn_kda_gate_workspace_bytes.restype = SZ
    lib.gdn_max_chunks.argtypes = [D, I32]
    lib.gdn_max_chunks.restype = I64
    lib.gdn_build_chunk_indices.argtypes = [D, P, P, I64]
    lib.gdn_build_chunk_indices.restype = I64
    lib.gdn_chunk_table_device.argtypes = [D, P, P, I64, P, P]
    lib.gdn_chunk_table_device.restype = I32
    lib.gdn_device_status.argtypes = [P, P]
    lib.gdn_device_status.restype = I32
    lib.gdn_status_string.argtypes = [I32]
    lib.gdn_status_string.restype = ctypes.c_char_p
    lib.gdn_version.argtypes = []
    lib.gdn_version.restype = ctypes.c_char_p
    lib.gdn_chunk_fwd_noalloc.argtypes = [D] + [P] * 12
    lib.gdn_chunk_fwd_noalloc.restype = I32
    lib.gdn_noalloc_scratch_bytes.argtypes = []
    lib.gdn_noalloc_scratch_bytes.restype = SZ
    lib.gdn_noalloc_device_status.argtypes = [P]
    lib.gdn_noalloc_device_status.restype = I32
    lib.gdn_launch_count.argtypes = []
    lib.gdn_launch_count.restype = I64
    lib.gdn_profile.argtypes = [I32]
    lib.gdn_profile.restype = I32
    lib.gdn_profile_read.argtypes = [ctypes.c_char_p, SZ]
    lib.gdn_profile_read.restype = I64
    return lib


class _Lazy:
    """The loaded library, opened on first attribute access (raises ImportError if missing)."""

    _lib = None

    def __getattr__(self, name):
        if _Lazy._lib is None:
            _Lazy._lib = _load()
        return getattr(_Lazy._lib, name)


lib = _Lazy()


def status_string(status: int) -> str:
    return lib.gdn_status_string(int(status)).decode()


def version() -> str:
    return lib.gdn_version().decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def make_dims(q, v, cu_seqlens=None, scale=0.0) -> gdn_dims:
    B, T, H, K = q.shape
    HV, V = v.shape[2], v.shape[3]
    N = (cu_seqlens.numel() - 1) if cu_seqlens is not None else B
    dt = GDN_DTYPE_BF16 if q.dtype == torch.bfloat16 else GDN_DTYPE_FP32
    return gdn_dims(B, T, H, HV, K, V, N, dt, float(scale or 0.0))


def workspace_bytes(dims: gdn_dims, varlen: bool, backward: bool) -> int:
    return int(lib.gdn_workspace_bytes(ctypes.byref(dims), int(varlen), int(backward)))


def max_chunks(dims: gdn_dims, varlen: bool) -> int:
    return int(lib.gdn_max_chunks(ctypes.byref(dims), int(varlen)))


def _workspace(dims, varlen, backward, workspace, device):
    n = workspace_bytes(dims, varlen, backward)
    if n == 0:
        raise GDNError("gdn_workspace_bytes", GDN_ERR_INVALID_ARG)
    if workspace is not None and workspace.numel() >= n:
        return workspace
    return torch.empty(n, dtype=torch.uint8, device=device)


def _check(name, t, dtype, shape, device):
    if t is None:
        return
    if t.device != device or t.dtype != dtype or not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected contiguous {dtype} {tuple(shape)} on {device}, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device} (contiguous={t.is_contiguous()})")


def _check_inputs(q, k, v, g_raw, A_log, dt_bias, beta, cu_seqlens, initial_state):
    dev = q.device
    B, T, H, K = q.shape
    HV, V = v.shape[2], v.shape[3]
    Nst = (cu_seqlens.numel() - 1) if cu_seqlens is not None else B
    _check("q", q, q.dtype, (B, T, H, K), dev)
    _check("k", k, q.dtype, (B, T, H, K), dev)
    _check("v", v, q.dtype, (B, T, HV, V), dev)
    _check("g_raw", g_raw, torch.float32, (B, T, HV), dev)
    _check("beta", beta, torch.float32, (B, T, HV), dev)
    _check("A_log", A_log, torch.float32, (HV,), dev)
    _check("dt_bias", dt_bias, torch.float32, (HV,), dev)
    _check("cu_seqlens", cu_seqlens, torch.int64, (Nst + 1,), dev)
    _check("initial_state", initial_state, torch.float32, (Nst, HV, K, V), dev)
    return Nst


def gdn_chunk_fwd(q, k, v, g_raw, A_log, dt_bias, beta, cu_seqlens=None, initial_state=None,
                  scale=0.0, output_final_state=True, workspace=None, out=None, final_state=None,
                  flags=0):
    """Forward: returns (o, final_state or None).  See include/gdn.h for layouts; `flags` is
    passed through in gdn_dims.flags."""
    Nst = _check_inputs(q, k, v, g_raw, A_log, dt_bias, beta, cu_seqlens, initial_state)
    dims = make_dims(q, v, cu_seqlens, scale)
    dims.flags = int(flags)
    ws = _workspace(dims, cu_seqlens is not None, False, workspace, q.device)
    o = out if out is not None else torch.empty(v.shape, dtype=q.dtype, device=q.device)
    ht = None
    if output_final_state:
        ht = final_state if final_state is not None else torch.empty(
            (Nst, v.shape[2], q.shape[3], v.shape[3]), dtype=torch.float32, device=q.device)
    rc = lib.gdn_chunk_fwd(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(g_raw), _ptr(A_log),
                           _ptr(dt_bias), _ptr(beta), _ptr(cu_seqlens), _ptr(initial_state), _ptr(o),
                           _ptr(ht), _ptr(ws), ws.numel(), _stream())
    if rc != GDN_OK:
        raise GDNError("gdn_chunk_fwd", rc)
    return o, ht


def gdn_chunk_fwd_noalloc(q, k, v, g_raw, A_log, dt_bias, beta, cu_seqlens=None,
                          initial_state=None, scale=0.0, out=None, final_state=None):
    """Forward through the library's allocation-free entry point: the scratch is the
    library's own fixed device array (gdn_noalloc_scratch_bytes()), so the C call allocates
    nothing.  The caller provides (or here: torch allocates) o and final_state only."""
    Nst = _check_inputs(q, k, v, g_raw, A_log, dt_bias, beta, cu_seqlens, initial_state)
    dims = make_dims(q, v, cu_seqlens, scale)
    o = out if out is not None else torch.empty(v.shape, dtype=q.dtype, device=q.device)
    ht = final_state if final_state is not None else torch.empty(
        (Nst, v.shape[2], q.shape[3], v.shape[3]), dtype=torch.float32, device=q.device)
    rc = lib.gdn_chunk_fwd_noalloc(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(g_raw),
                                   _ptr(A_log), _ptr(dt_bias), _ptr(beta), _ptr(cu_seqlens),
                                   _ptr(initial_state), _ptr(o), _ptr(ht), _stream())
    if rc != GDN_OK:
        raise GDNError("gdn_chunk_fwd_noalloc", rc)
    return o, ht


def gdn_recurrent_fwd(q, k, v, g_raw, A_log, dt_bias, beta, cu_seqlens=None, initial_state=None,
                      scale=0.0, out=None, final_state=None, workspace=None):
    """Token-by-token forward (decode steps, short prefills): returns (o, final_state).  Same
    arguments and layouts as gdn_chunk_fwd; final_state may be initial_state itself (the
    state is updated in place).  `workspace` (optional) holds the device status word."""
    Nst = _check_inputs(q, k, v, g_raw, A_log, dt_bias, beta, cu_seqlens, initial_state)
    dims = make_dims(q, v, cu_seqlens, scale)
    need = int(lib.gdn_recurrent_workspace_bytes())
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    elif workspace.numel() < need:
        raise ValueError(f"workspace holds {workspace.numel()} bytes, the call needs {need}")
    o = out if out is not None else torch.empty(v.shape, dtype=q.dtype, device=q.device)
    ht = final_state if final_state is not None else torch.empty(
        (Nst, v.shape[2], q.shape[3], v.shape[3]), dtype=torch.float32, device=q.device)
    rc = lib.gdn_recurrent_fwd(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(g_raw),
                               _ptr(A_log), _ptr(dt_bias), _ptr(beta), _ptr(cu_seqlens),
                               _ptr(initial_state), _ptr(o), _ptr(ht), _ptr(workspace),
                               workspace.numel(), _stream())
    if rc != GDN_OK:
        raise GDNError("gdn_recurrent_fwd", rc)
    return o, ht


def gdn_kda_recurrent_fwd(q, k, v, g_raw, A_log, dt_bias, beta, cu_seqlens=None,
                          initial_state=None, scale=0.0, out=None, final_state=None, workspace=None):
    """KDA (per-key-channel gate) token-by-token forward: returns (o, final_state).  As
    gdn_recurrent_fwd with g_raw [B,T,HV,K] and dt_bias [HV*K] (or None)."""
    B, T, H, K = q.shape
    HV = v.shape[2]
    Nst = _check_inputs(q, k, v, None, A_log, None, beta, cu_seqlens, initial_state)
    _check("g_raw", g_raw, torch.float32, (B, T, HV, K), q.device)
    _check("dt_bias", dt_bias, torch.float32, (HV * K,), q.device)
    dims = make_dims(q, v, cu_seqlens, scale)
    need = int(lib.gdn_recurrent_workspace_bytes())
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    elif workspace.numel() < need:
        raise ValueError(f"workspace holds {workspace.numel()} bytes, the call needs {need}")
    o = out if out is not None else torch.empty(v.shape, dtype=q.dtype, device=q.device)
    ht = final_state if final_state is not None else torch.empty(
        (Nst, HV, K, v.shape[3]), dtype=torch.float32, device=q.device)
    rc = lib.gdn_kda_recurrent_fwd(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(g_raw),
                                   _ptr(A_log), _ptr(dt_bias), _ptr(beta), _ptr(cu_seqlens),
                                   _ptr(initial_state), _ptr(o), _ptr(ht), _ptr(workspace),
                                   workspace.numel(), _stream())
    if rc != GDN_OK:
        raise GDNError("gdn_kda_recurrent_fwd", rc)
    return o, ht


def kda_chunk_workspace_bytes(dims: gdn_dims, varlen: bool, backward: bool = False) -> int:
    return int(lib.gdn_kda_chunk_workspace_bytes(ctypes.byref(dims), int(varlen), int(backward)))


def gdn_kda_chunk_fwd(q, k, v, g_raw, A_log, dt_bias, beta, cu_seqlens=None, initial_state=None,
                      scale=0.0, output_final_state=True, out=None, final_state=None, workspace=None):
    """Chunkwise KDA forward (per-key-channel gate, long sequences): returns (o, final_state or
    None).  Arguments as gdn_kda_recurrent_fwd.  For a gdn_kda_chunk_bwd afterwards, pass a
    workspace of kda_chunk_workspace_bytes(dims, varlen, backward=True) bytes: the forward then
    keeps in it what the backward reads."""
    B, T, H, K = q.shape
    HV = v.shape[2]
    Nst = _check_inputs(q, k, v, None, A_log, None, beta, cu_seqlens, initial_state)
    _check("g_raw", g_raw, torch.float32, (B, T, HV, K), q.device)
    _check("dt_bias", dt_bias, torch.float32, (HV * K,), q.device)
    dims = make_dims(q, v, cu_seqlens, scale)
    need = kda_chunk_workspace_bytes(dims, cu_seqlens is not None)
    if need == 0:
        raise GDNError("gdn_kda_chunk_workspace_bytes", GDN_ERR_INVALID_ARG)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    o = out if out is not None else torch.empty(v.shape, dtype=q.dtype, device=q.device)
    ht = None
    if output_final_state:
        ht = final_state if final_state is not None else torch.empty(
            (Nst, HV, K, v.shape[3]), dtype=torch.float32, device=q.device)
    rc = lib.gdn_kda_chunk_fwd(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(g_raw),
                               _ptr(A_log), _ptr(dt_bias), _ptr(beta), _ptr(cu_seqlens),
                               _ptr(initial_state), _ptr(o), _ptr(ht), _ptr(workspace),
                               workspace.numel(), _stream())
    if rc != GDN_OK:
        raise GDNError("gdn_kda_chunk_fwd", rc)
    return o, ht


def gdn_kda_chunk_bwd(q, k, v, g_raw, A_log, dt_bias, beta, d_o, workspace, cu_seqlens=None,
                      dht=None, scale=0.0, want_dh0=True, want_param_grads=True, outs=None):
    """Backward of gdn_kda_chunk_fwd.  `workspace` must be the one a gdn_kda_chunk_fwd call with
    the same inputs used, sized with kda_chunk_workspace_bytes(dims, varlen, backward=True).
    Returns a dict with dq, dk, dv, dbeta, dg (dL/dyg, [B,T,HV,K]) and, when asked, dh0,
    dg_raw, dA_log, ddt_bias (None without dt_bias)."""
    B, T, H, K = q.shape
    HV, V = v.shape[2], v.shape[3]
    Nst = _check_inputs(q, k, v, None, A_log, None, beta, cu_seqlens, None)
    _check("g_raw", g_raw, torch.float32, (B, T, HV, K), q.device)
    _check("dt_bias", dt_bias, torch.float32, (HV * K,), q.device)
    _check("d_o", d_o, q.dtype, (B, T, HV, V), q.device)
    _check("dht", dht, torch.float32, (Nst, HV, K, V), q.device)
    dims = make_dims(q, v, cu_seqlens, scale)
    need = kda_chunk_workspace_bytes(dims, cu_seqlens is not None, True)
    if workspace.numel() < need:
        raise ValueError(f"workspace holds {workspace.numel()} bytes, the backward needs {need}")
    dev = q.device
    if outs is None:
        outs = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
                    dbeta=torch.empty((B, T, HV), dtype=torch.float32, device=dev),
                    dg=torch.empty((B, T, HV, K), dtype=torch.float32, device=dev))
        if want_dh0:
            outs["dh0"] = torch.empty((Nst, HV, K, V), dtype=torch.float32, device=dev)
        if want_param_grads:
            outs["dg_raw"] = torch.empty((B, T, HV, K), dtype=torch.float32, device=dev)
            outs["dA_log"] = torch.empty(HV, dtype=torch.float32, device=dev)
            outs["ddt_bias"] = (torch.empty(HV * K, dtype=torch.float32, device=dev)
                                if dt_bias is not None else None)
    g = lambda name: _ptr(outs.get(name))
    rc = lib.gdn_kda_chunk_bwd(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(g_raw), _ptr(A_log),
                               _ptr(dt_bias), _ptr(beta), _ptr(cu_seqlens), _ptr(d_o), _ptr(dht),
                               g("dq"), g("dk"), g("dv"), g("dg"), g("dbeta"), g("dh0"), g("dg_raw"),
                               g("dA_log"), g("ddt_bias"), _ptr(workspace), workspace.numel(), _stream())
    if rc != GDN_OK:
        raise GDNError("gdn_kda_chunk_bwd", rc)
    return outs


def state_affine(A, X, B=None, transpose=False, out=None):
    """out[n] = op(A[n]) X[n] + B[n] over the leading dims: A [..., K, K], X and B [..., K, V]
    fp32 (op = transpose when asked).  `out` may be X."""
    K, V = X.shape[-2], X.shape[-1]
    count = X.numel() // (K * V) if X.numel() else 0
    _check("A", A, torch.float32, tuple(X.shape[:-2]) + (K, K), X.device)
    _check("B", B, torch.float32, tuple(X.shape), X.device)
    if not X.is_contiguous() or X.dtype != torch.float32:
        raise ValueError("X: expected contiguous float32")
    out = out if out is not None else torch.empty_like(X)
    _check("out", out, torch.float32, tuple(X.shape), X.device)
    rc = lib.gdn_state_affine(count, K, V, _ptr(A), int(bool(transpose)), _ptr(X), _ptr(B), _ptr(out),
                              _stream())
    if rc != GDN_OK:
        raise GDNError("gdn_state_affine", rc)
    return out


_TORCH_DT = {torch.float32: GDN_DTYPE_FP32, torch.bfloat16: GDN_DTYPE_BF16,
             torch.float16: GDN_DTYPE_FP16}


def _kda_shape(g, A_log, dt_bias):
    if g.dim() < 2:
        raise ValueError("g needs at least [H, D] trailing dims")
    H, D = g.shape[-2], g.shape[-1]
    T = g.numel() // (H * D) if H * D else 0
    _check("g", g, g.dtype, tuple(g.shape), g.device)
    _check("A_log", A_log, torch.float32, (H,), g.device)
    if dt_bias is not None:
        _check("dt_bias", dt_bias, torch.float32, (H * D,), g.device)
    if g.dtype not in _TORCH_DT:
        raise ValueError(f"g dtype {g.dtype} is not fp32, bf16 or fp16")
    return T, H, D


def kda_gate_fwd(g, A_log, dt_bias=None, output_dtype=torch.float32, out=None):
    """KDA gate: yg = -exp(A_log[h]) * softplus(g + dt_bias[h*D+d]) for g [..., H, D]."""
    T, H, D = _kda_shape(g, A_log, dt_bias)
    yg = out if out is not None else torch.empty(g.shape, dtype=output_dtype, device=g.device)
    _check("out", yg, output_dtype, tuple(g.shape), g.device)
    rc = lib.gdn_kda_gate_fwd(T, H, D, _TORCH_DT[g.dtype], _ptr(g), _ptr(A_log), _ptr(dt_bias),
                              _TORCH_DT[output_dtype], _ptr(yg), _stream())
    if rc != GDN_OK:
        raise GDNError("gdn_kda_gate_fwd", rc)
    return yg


def kda_gate_bwd(g, A_log, dyg, dt_bias=None, workspace=None):
    """Backward of kda_gate_fwd: returns (dg, dA_log, ddt_bias or None)."""
    T, H, D = _kda_shape(g, A_log, dt_bias)
    _check("dyg", dyg, dyg.dtype, tuple(g.shape), g.device)
    need = int(lib.gdn_kda_gate_workspace_bytes(T, H, D))
    ws = workspace if workspace is not None else torch.empty(need, dtype=torch.uint8, device=g.device)
    dg = torch.empty_like(g)
    dA = torch.empty(H, dtype=torch.float32, device=g.device)
    ddt = torch.empty(H * D, dtype=torch.float32, device=g.device) if dt_bias is not None else None
    rc = lib.gdn_kda_gate_bwd(T, H, D, _TORCH_DT[g.dtype], _ptr(g), _ptr(A_log), _ptr(dt_bias),
                              _TORCH_DT[dyg.dtype], _ptr(dyg), _ptr(dg), _ptr(dA), _ptr(ddt),
                              _ptr(ws), ws.numel(), _stream())
    if rc != GDN_OK:
        raise GDNError("gdn_kda_gate_bwd", rc)
    return dg, dA, ddt


def kda_gate_workspace_bytes(T: int, H: int, D: int) -> int:
    return int(lib.gdn_kda_gate_workspace_bytes(T, H, D))


def recurrent_workspace_bytes() -> int:
    return int(lib.gdn_recurrent_workspace_bytes())


def noalloc_scratch_bytes() -> int:
    return int(lib.gdn_noalloc_scratch_bytes())


def noalloc_device_status() -> int:
    """Status word of the last gdn_chunk_fwd_noalloc call on this device (synchronises)."""
    return int(lib.gdn_noalloc_device_status(_stream()))


def gdn_chunk_bwd(q, k, v, g_raw, A_log, dt_bias, beta, d_o, cu_seqlens=None, initial_state=None,
                  dht=None, scale=0.0, want_dh0=True, want_param_grads=True, workspace=None,
                  outs=None, reuse_forward=False):
    """Backward of sum(d_o*o) + sum(dht*final_state).  Returns a dict with dq, dk, dv, dg,
    dbeta and (when asked) dh0, dg_raw, dA_log, ddt_bias.  reuse_forward=True passes
    GDN_FLAG_BWD_REUSE_FWD: `workspace` must be the one the matching gdn_chunk_fwd call used
    (sized for the backward) with inputs unchanged since."""
    Nst = _check_inputs(q, k, v, g_raw, A_log, dt_bias, beta, cu_seqlens, initial_state)
    B, T, H, K = q.shape
    HV, V = v.shape[2], v.shape[3]
    _check("d_o", d_o, q.dtype, (B, T, HV, V), q.device)
    _check("dht", dht, torch.float32, (Nst, HV, K, V), q.device)
    dims = make_dims(q, v, cu_seqlens, scale)
    if reuse_forward:
        if workspace is None:
            raise ValueError("reuse_forward needs the forward's workspace")
        dims.flags = GDN_FLAG_BWD_REUSE_FWD
    ws = _workspace(dims, cu_seqlens is not None, True, workspace, q.device)
    if reuse_forward and ws is not workspace:
        raise ValueError("the forward's workspace is smaller than the backward needs")
    dev = q.device
    if outs is None:
        outs = dict(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v),
                    dg=torch.empty((B, T, HV), dtype=torch.float32, device=dev),
                    dbeta=torch.empty((B, T, HV), dtype=torch.float32, device=dev))
        if want_dh0:
            outs["dh0"] = torch.empty((Nst, HV, K, V), dtype=torch.float32, device=dev)
        if want_param_grads:
            outs["dg_raw"] = torch.empty((B, T, HV), dtype=torch.float32, device=dev)
            outs["dA_log"] = torch.empty((HV,), dtype=torch.float32, device=dev)
            outs["ddt_bias"] = torch.empty((HV,), dtype=torch.float32, device=dev)
    g = outs.get
    rc = lib.gdn_chunk_bwd(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(g_raw), _ptr(A_log),
                           _ptr(dt_bias), _ptr(beta), _ptr(cu_seqlens), _ptr(initial_state),
                           _ptr(d_o), _ptr(dht), _ptr(g("dq")), _ptr(g("dk")), _ptr(g("dv")),
                           _ptr(g("dg")), _ptr(g("dbeta")), _ptr(g("dh0")), _ptr(g("dg_raw")),
                           _ptr(g("dA_log")), _ptr(g("ddt_bias")), _ptr(ws), ws.numel(), _stream())
    if rc != GDN_OK:
        raise GDNError("gdn_chunk_bwd", rc)
    return outs


def gdn_build_chunk_indices(dims: gdn_dims, cu_host=None):
    """Host chunk table as a [count, 4] int32 tensor (see include/gdn.h)."""
    import numpy as np
    cu = None if cu_host is None else np.ascontiguousarray(np.asarray(cu_host, dtype=np.int64))
    cp = None if cu is None else cu.ctypes.data_as(ctypes.c_void_p)
    n = lib.gdn_build_chunk_indices(ctypes.byref(dims), cp, None, 0)
    if n < 0:
        raise GDNError("gdn_build_chunk_indices", -n)
    out = np.zeros((max(n, 1), 4), dtype=np.int32)
    lib.gdn_build_chunk_indices(ctypes.byref(dims), cp, out.ctypes.data_as(ctypes.c_void_p), n)
    return out[:n]


def gdn_chunk_table_device(dims: gdn_dims, cu_seqlens=None, cap=None, device="cuda"):
    """Device-built chunk table ([cap, 4] int32 on the device) and its count (int)."""
    if cap is None:
        cap = max_chunks(dims, cu_seqlens is not None)
    table = torch.empty((cap, 4), dtype=torch.int32, device=device)
    count = torch.empty((4,), dtype=torch.int32, device=device)
    rc = lib.gdn_chunk_table_device(ctypes.byref(dims), _ptr(cu_seqlens), _ptr(table), int(cap),
                                    _ptr(count), _stream())
    if rc != GDN_OK:
        raise GDNError("gdn_chunk_table_device", rc)
    return table, int(count[0].item())


def gdn_device_status(workspace) -> int:
    return int(lib.gdn_device_status(_ptr(workspace), _stream()))


def launch_count() -> int:
    """Kernel launches issued by the library since it was loaded."""
    return int(lib.gdn_launch_count())


def profile(enable: bool) -> None:
    """Bracket every launch with CUDA events on its stream (measurement passes only)."""
    lib.gdn_profile(int(bool(enable)))


def profile_read() -> dict:
    """Per-kernel {name: (launches, total_ms)} since the last read (synchronises)."""
    import json
    buf = ctypes.create_string_buffer(1 << 16)
    n = lib.gdn_profile_read(buf, len(buf))
    if n < 0:
        raise GDNError("gdn_profile_read", -n)
    if n >= len(buf):
        raise RuntimeError("profile record does not fit the buffer")
    return {k: tuple(v) for k, v in json.loads(buf.value.decode() or "{}").items()}
