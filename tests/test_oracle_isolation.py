"""Processes that only use the oracle and the seeded input generators never map the product
library: importing the package's input module leaves libgdn_b200.so unloaded."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_PROBE = r"""
import sys
sys.path.insert(0, {root!r})
from gated_deltanet_chunkwise_chunk_b200 import synth
from oracle import oracle
case = synth.make_case(B=1, T=5, H=1, HV=2, K=8, V=8, dtype="fp32", seed=1)
oracle.fwd(case.q, case.k, case.v, case.a, case.A_log, case.dt_bias, case.beta)
maps = open("/proc/self/maps").read()
print("MAPPED" if "libgdn_b200" in maps else "CLEAN")
"""


def test_oracle_and_inputs_do_not_load_the_product_library():
    r = subprocess.run([sys.executable, "-c", _PROBE.format(root=ROOT)], capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip().endswith("CLEAN"), r.stdout
