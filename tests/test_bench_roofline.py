"""bench.py's roofline arithmetic on CPU: the dominant kernel by device time, its per-launch
algorithmic FLOPs (the method's products per token and value head x the launch's
token-heads), achieved = FLOPs / launch time against the bf16 peak, and the separately
reported bytes the kernel moves with the inter-kernel intermediates included."""
from __future__ import annotations

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from gated_deltanet_chunkwise_chunk_b200 import synth  # noqa: E402

PK = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "source": "test"}


def _case():
    return synth.make_case(B=1, T=8192, H=16, HV=32, K=128, V=128, dtype="bf16", seed=1, name="roof")


def test_dominant_kernel_tensor_fraction_from_algorithmic_flops():
    case = _case()
    prof = {"tc_scan_bwd": (2, 0.6), "tc_wy": (2, 0.3), "chunk_table": (2, 0.01)}
    r = bench.kernel_roofline(prof, case, PK)
    units = (8192 // 64) * 32
    assert r["kernel"] == "tc_scan_bwd" and r["units_per_launch"] == units
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    fl = 6 * 128 * 128  # the reverse scan's products per token and value head
    assert bench.kernel_flops_per_token_head(128, 128)["tc_scan_bwd"] == fl
    achieved = fl * 8192 * 32 / 0.3e-3 / 1e12  # 0.6 ms over 2 launches
    assert r["achieved"] == pytest.approx(achieved, rel=1e-3)
    assert r["frac"] == pytest.approx(achieved / 1600.0, rel=1e-3)
    assert r["frac_sustained_peak"] == pytest.approx(achieved / 1400.0, rel=1e-3)
    assert r["share"] == pytest.approx(0.6 / 0.91, rel=1e-3)


def test_bytes_with_intermediates_reported_separately():
    case = _case()
    r = bench.kernel_roofline({"tc_wy": (1, 0.5)}, case, PK, steps=1)
    units = (8192 // 64) * 32
    per_unit = bench.kernel_bytes_per_unit(128, 128, 2, 2)["tc_wy"]
    h = r["hbm_with_intermediates"]
    assert h["bytes_per_launch"] == int(per_unit * units)
    assert h["achieved"] == pytest.approx(per_unit * units / 0.5e-3 / 1e9, rel=1e-3)
    assert h["frac"] == pytest.approx(h["achieved"] / 6000.0, rel=1e-3)


def test_segmented_launches_share_the_step():
    """A kernel launched once per segment (8 per step, 2 steps profiled) does a step's work
    in 8 launches: per launch an eighth of the units, achieved over the step's kernel time."""
    case = _case()
    r = bench.kernel_roofline({"tc_scan_bwd": (16, 2.4), "tc_wy": (16, 0.8)}, case, PK, steps=2)
    units = (8192 // 64) * 32
    assert r["kernel"] == "tc_scan_bwd" and r["launches_per_step"] == 8
    assert r["units_per_launch"] == units / 8
    fl = 6 * 128 * 128
    assert r["achieved"] == pytest.approx(fl * 8192 * 32 / 1.2e-3 / 1e12, rel=1e-3)
    assert r["launch_ms"] == pytest.approx(2.4 / 16, rel=1e-3)


def test_no_profile_no_roofline():
    assert bench.kernel_roofline({}, _case(), PK) is None
