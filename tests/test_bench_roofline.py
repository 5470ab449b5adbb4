"""bench.py's roofline arithmetic on CPU: the dominant kernel by device time, its per-launch
algorithmic bytes (per-unit bytes x units), achieved = bytes / launch time, frac = achieved /
peak, and the HBM-versus-tensor choice of the binding bound."""
from __future__ import annotations

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from gated_deltanet_chunkwise_chunk_b200 import synth  # noqa: E402


def _case():
    return synth.make_case(B=1, T=8192, H=16, HV=32, K=128, V=128, dtype="bf16", seed=1, name="roof")


def test_dominant_kernel_and_hbm_fraction():
    case = _case()
    pk = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "source": "test"}
    prof = {"tc_scan_bwd": (2, 0.6), "tc_wy": (2, 0.3), "chunk_table": (2, 0.01)}
    r = bench.kernel_roofline(prof, case, pk)
    units = (8192 // 64) * 32
    per_unit = bench.kernel_bytes_per_unit(128, 128, 2, 2)["tc_scan_bwd"]
    assert r["kernel"] == "tc_scan_bwd" and r["units_per_launch"] == units
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    achieved = per_unit * units / 0.3e-3 / 1e9  # 0.6 ms over 2 launches
    assert r["achieved"] == pytest.approx(achieved, rel=1e-3)
    assert r["frac"] == pytest.approx(achieved / 6000.0, rel=1e-3)
    assert r["share"] == pytest.approx(0.6 / 0.91, rel=1e-3)
    assert r["algorithmic_bytes"] == int(per_unit * units)


def test_tensor_bound_when_the_flops_take_longer():
    case = _case()
    pk = {"hbm_gbs": 1e9, "bf16_tflops": 1.0, "source": "test"}  # absurd peaks force the tensor side
    r = bench.kernel_roofline({"tc_dqkwg": (1, 1.0)}, case, pk)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    fl = bench.kernel_flops_per_token_head(128, 128)["tc_dqkwg"]
    assert r["achieved"] == pytest.approx(fl * 8192 * 32 / 1e-3 / 1e12, rel=1e-3)


def test_no_profile_no_roofline():
    assert bench.kernel_roofline({}, _case(), {"hbm_gbs": 1.0, "bf16_tflops": 1.0, "source": "t"}) is None
