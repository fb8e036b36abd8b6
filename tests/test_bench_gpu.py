"""The bench line on a GPU: one short run of each arm-independent field of the JSON contract.

bench.py's own arm is run in a subprocess on a small m130 layer (2 timed steps after 3 warm-up
steps, host-buffer e2e on, the oracle baseline off) and its line is checked for the keys and
relations the contract fixes: the HBM roofline against the measured peak, live ALU fractions,
clock samples inside the timed region, the library's launch count, and an e2e measurement that
moved the inputs and outputs through host memory.
"""

import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_line_contract(cuda_device):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--workload", "m130", "--seqlen", "512",
           "--steps", "2", "--warmup", "3", "--no-cpu-baseline"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    line = json.loads(res.stdout.strip().splitlines()[-1])
    assert line["unit"] == "GB/s" and line["higher_is_better"] is True
    assert line["n_gpus"] == 1 and line["steps"] == 2 and line["warmup"] >= 3
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert line["config"]["name"] == "m130" and line["config"]["seqlen"] == 512
    r = line["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert 0 < r["kernel_ms"] <= line["ms_per_step"] * 1.05
    for key in ("fp32", "mufu"):
        assert 0 < r["alu"][key]["frac"] < 1.5
    assert line["gpu_launches"] >= line["steps"]
    clocks = line["clocks"]
    assert clocks is None or (clocks["samples"] >= 1 and clocks["sm_max_mhz"] > 0)
    e2e = line["e2e"]
    assert e2e["value"] > 0 and e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
    assert e2e["value"] < line["value"]  # the host link is far slower than HBM
