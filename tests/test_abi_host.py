"""The C-ABI library on the CPU: it loads, exports every symbol include/gdn.h declares,
rejects bad arguments before any launch, and builds the chunk table bit-exactly."""
import ctypes
import os
import re

import numpy as np
import pytest

import gated_deltanet_chunkwise_chunk_b200 as gdn
from gated_deltanet_chunkwise_chunk_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "gdn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 9
    lib = ctypes.CDLL(binding.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(binding.EXPORTED) == names


def test_status_strings_and_version():
    assert gdn.status_string(0) == "GDN_OK"
    assert gdn.status_string(5) == "GDN_ERR_TIMEOUT"
    assert gdn.status_string(99) == "GDN_ERR_UNKNOWN"
    assert "sm_100a" in gdn.version()


def _dims(**kw):
    base = dict(B=1, T=256, H=2, HV=4, K=128, V=128, N=1, dtype=1, scale=0.0)
    base.update(kw)
    return gdn.gdn_dims(**base)


def test_workspace_bytes_rejects_bad_dims():
    assert gdn.workspace_bytes(_dims(), False, False) > 0
    assert gdn.workspace_bytes(_dims(), False, True) > gdn.workspace_bytes(_dims(), False, False)
    assert gdn.workspace_bytes(_dims(K=96), False, False) == 0      # unsupported head dim
    assert gdn.workspace_bytes(_dims(HV=3), False, False) == 0      # HV not a multiple of H
    assert gdn.workspace_bytes(_dims(B=2, N=2), True, False) == 0   # varlen needs B = 1
    assert gdn.workspace_bytes(_dims(dtype=7), False, False) == 0


def test_size_limits():
    """Tokens < 2^31 and chunks x HV x 128 < 2^31 (32-bit tensor-map rows); at the limits the
    dimensions are rejected before any allocation or launch."""
    assert gdn.workspace_bytes(_dims(T=1 << 20, H=16, HV=32), False, True) > 0
    assert gdn.workspace_bytes(_dims(T=1 << 24, H=16, HV=32), False, True) > 0  # 2^18 chunks x 32 x 128 = 2^30
    assert gdn.workspace_bytes(_dims(T=1 << 25, H=16, HV=32), False, True) == 0  # = 2^31
    assert gdn.workspace_bytes(_dims(B=1 << 12, T=1 << 19, H=1, HV=1), False, False) == 0  # 2^31 tokens


def test_entry_points_reject_bad_arguments_before_launch():
    d = _dims()
    lib = binding.lib
    P = ctypes.c_void_p
    al = P(4096)  # an aligned non-null address; never dereferenced because validation fails first
    mis = P(4097)
    null = None
    # null required input
    rc = lib.gdn_chunk_fwd(ctypes.byref(d), null, al, al, al, al, al, al, null, null, al, null,
                           al, 1 << 40, null)
    assert rc == binding.GDN_ERR_INVALID_ARG
    # misaligned pointer
    rc = lib.gdn_chunk_fwd(ctypes.byref(d), mis, al, al, al, al, al, al, null, null, al, null,
                           al, 1 << 40, null)
    assert rc == binding.GDN_ERR_INVALID_ARG
    # too small a workspace
    rc = lib.gdn_chunk_fwd(ctypes.byref(d), al, al, al, al, al, al, al, null, null, al, null,
                           al, 16, null)
    assert rc == binding.GDN_ERR_WORKSPACE
    # unsupported K
    d2 = _dims(K=32)
    rc = lib.gdn_chunk_fwd(ctypes.byref(d2), al, al, al, al, al, al, al, null, null, al, null,
                           al, 1 << 40, null)
    assert rc == binding.GDN_ERR_UNSUPPORTED
    # backward: null required output
    rc = lib.gdn_chunk_bwd(ctypes.byref(d), al, al, al, al, al, al, al, null, null, al, null,
                           al, al, al, null, al, null, null, null, null, al, 1 << 40, null)
    assert rc == binding.GDN_ERR_INVALID_ARG
    # recurrent forward: null input, small workspace, unsupported V
    rc = lib.gdn_recurrent_fwd(ctypes.byref(d), null, al, al, al, al, al, al, null, null, al, null,
                               al, 1 << 20, null)
    assert rc == binding.GDN_ERR_INVALID_ARG
    rc = lib.gdn_recurrent_fwd(ctypes.byref(d), al, al, al, al, al, al, al, null, null, al, null,
                               al, 64, null)
    assert rc == binding.GDN_ERR_WORKSPACE
    rc = lib.gdn_recurrent_fwd(ctypes.byref(_dims(V=96)), al, al, al, al, al, al, al, null, null,
                               al, null, al, 1 << 20, null)
    assert rc == binding.GDN_ERR_UNSUPPORTED
    assert lib.gdn_recurrent_workspace_bytes() == 256


def test_kda_and_state_entry_points_reject_bad_arguments_before_launch():
    d = _dims()
    lib = binding.lib
    P = ctypes.c_void_p
    al, mis, null = P(4096), P(4097), None
    # KDA gate: bad sizes, unknown dtype, null input, misaligned pointer, small workspace
    assert lib.gdn_kda_gate_fwd(8, 0, 64, 1, al, al, null, 0, al, null) == binding.GDN_ERR_INVALID_ARG
    assert lib.gdn_kda_gate_fwd(8, 4, 64, 9, al, al, null, 0, al, null) == binding.GDN_ERR_UNSUPPORTED
    assert lib.gdn_kda_gate_fwd(8, 4, 64, 1, null, al, null, 0, al, null) == binding.GDN_ERR_INVALID_ARG
    assert lib.gdn_kda_gate_fwd(8, 4, 64, 1, mis, al, null, 0, al, null) == binding.GDN_ERR_INVALID_ARG
    assert lib.gdn_kda_gate_bwd(8, 4, 64, 1, al, al, null, 0, al, al, al, null, al, 16, null) == \
        binding.GDN_ERR_WORKSPACE
    assert lib.gdn_kda_gate_workspace_bytes(8, 4, 64) > 0
    assert lib.gdn_kda_gate_workspace_bytes(8, 1 << 13, 1 << 12) == 0  # H*D > 2^24
    # KDA recurrence: dt_bias may be NULL, A_log may not
    rc = lib.gdn_kda_recurrent_fwd(ctypes.byref(d), al, al, al, al, null, null, al, null, null, al,
                                   null, al, 1 << 20, null)
    assert rc == binding.GDN_ERR_INVALID_ARG
    # chunkwise KDA: workspace sizes by pass, too small a workspace, backward needs pass-1 size
    w0 = lib.gdn_kda_chunk_workspace_bytes(ctypes.byref(d), 0, 0)
    w1 = lib.gdn_kda_chunk_workspace_bytes(ctypes.byref(d), 0, 1)
    assert 0 < w0 < w1
    assert lib.gdn_kda_chunk_workspace_bytes(ctypes.byref(d), 0, 2) == 0
    assert lib.gdn_kda_chunk_workspace_bytes(ctypes.byref(_dims(K=96)), 0, 0) == 0
    rc = lib.gdn_kda_chunk_fwd(ctypes.byref(d), al, al, al, al, al, null, al, null, null, al, null,
                               al, w0 - 256, null)
    assert rc == binding.GDN_ERR_WORKSPACE
    rc = lib.gdn_kda_chunk_bwd(ctypes.byref(d), al, al, al, al, al, null, al, null, al, null, al, al,
                               al, al, al, null, null, null, null, al, w0, null)
    assert rc == binding.GDN_ERR_WORKSPACE
    rc = lib.gdn_kda_chunk_bwd(ctypes.byref(d), al, al, al, al, al, null, al, null, al, null, al, al,
                               al, al, al, null, null, null, al, al, w1, null)  # ddt_bias without dt_bias
    assert rc == binding.GDN_ERR_INVALID_ARG
    # state affine maps: K, V limits, null operands
    assert lib.gdn_state_affine(4, 129, 128, al, 0, al, null, al, null) == binding.GDN_ERR_INVALID_ARG
    assert lib.gdn_state_affine(4, 128, 48, al, 0, al, null, al, null) == binding.GDN_ERR_INVALID_ARG
    assert lib.gdn_state_affine(4, 128, 128, null, 0, al, null, al, null) == binding.GDN_ERR_INVALID_ARG
    assert lib.gdn_state_affine(4, 128, 128, al, 0, mis, null, al, null) == binding.GDN_ERR_INVALID_ARG


def _enumerate(cu, B, T):
    """Plain enumeration of 64-token chunks: (sequence, chunk, tokens, first flat token)."""
    out = []
    if cu is None:
        for b in range(B):
            for c in range((T + 63) // 64):
                out.append((b, c, min(64, T - 64 * c), b * T + 64 * c))
    else:
        for n in range(len(cu) - 1):
            L = cu[n + 1] - cu[n]
            for c in range((L + 63) // 64):
                out.append((n, c, min(64, L - 64 * c), cu[n] + 64 * c))
    return np.array(out, dtype=np.int32).reshape(-1, 4)


@pytest.mark.parametrize("lens", [[5, 1, 70, 64, 17], [64], [1], [0, 3, 0, 128, 129],
                                  [257, 4095, 1000, 63, 65, 127, 128]])
def test_chunk_indices_varlen_bit_exact(lens):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    d = _dims(T=int(cu[-1]), N=len(lens))
    got = gdn.gdn_build_chunk_indices(d, cu)
    ref = _enumerate(list(cu), 1, int(cu[-1]))
    assert got.dtype == np.int32 and np.array_equal(got, ref)
    assert len(got) <= gdn.max_chunks(d, True)


@pytest.mark.parametrize("B,T", [(1, 1), (2, 63), (2, 64), (3, 65), (8, 8192), (1, 32768)])
def test_chunk_indices_dense_bit_exact(B, T):
    d = _dims(B=B, T=T)
    got = gdn.gdn_build_chunk_indices(d, None)
    assert np.array_equal(got, _enumerate(None, B, T))
    assert len(got) == gdn.max_chunks(d, False)


def test_chunk_indices_reject_invalid_cu():
    d = _dims(T=10, N=2)
    with pytest.raises(gdn.GDNError):
        gdn.gdn_build_chunk_indices(d, [0, 6, 5])   # decreasing
    with pytest.raises(gdn.GDNError):
        gdn.gdn_build_chunk_indices(d, [0, 4, 9])   # does not end at T
    with pytest.raises(gdn.GDNError):
        gdn.gdn_build_chunk_indices(d, [1, 4, 10])  # does not start at 0


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "gated_deltanet_chunkwise_chunk_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                txt = open(os.path.join(dirpath, f)).read()
                for bad in ("from oracle", "import oracle", "liboracle", "gdn_oracle"):
                    assert bad not in txt, (f, bad)
