"""Writes tests/golden/tiny_oracle.json: the oracle's output on the seeded tiny workload.

It calls only the oracle (and the seeded input generator, which holds no step of the scan), so
the stored values are the oracle's own; the fixture guards the oracle and the generator against
unintended changes.  Regenerate only when a change to either is justified by a passage of the
pages, and name that passage in the commit message.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from selective_state_space_13_b200 import workloads as wl  # noqa: E402


def main():
    inp = wl.make_inputs("tiny")
    f = wl.inputs_f64(inp)
    out, last = oracle.selective_scan(f["u"], f["delta"], f["A"], f["B"], f["C"], Dskip=f["Dskip"],
                                      z=f["z"], delta_bias=f["delta_bias"], softplus=True)
    doc = {
        "what": "fp64 oracle output on the tiny workload (batch 1, L 64, D 16, N 4, fp32, seed "
                "20260): out [1,64,16] and last_state [1,1,16,4]",
        "written_by": "tests/golden/make_golden.py (oracle only)",
        "sum_u": float(np.sum(f["u"])),
        "out": out.tolist(),
        "last_state": last.tolist(),
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json")
    with open(path, "w") as fh:
        json.dump(doc, fh, separators=(",", ":"))
    print("wrote", path)


if __name__ == "__main__":
    main()
