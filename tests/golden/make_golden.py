"""Writes tests/golden/oracle_small.json: small seeded inputs (from the input
generator module) and the float64 oracle's outputs on them: y, the final
state, and the gradient for a seeded dy.

Run from the repository root:  python tests/golden/make_golden.py
Only the oracle computes the stored expected values; nothing here calls the
CUDA library. The pages print no numeric example of the scan, so this file is
a regression fixture of the pinned oracle, not a value from the pages.
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from selective_state_space_42_b200.workloads import (ScanWorkload,  # noqa: E402
                                                     make_scan_inputs)

CASES = [
    ScanWorkload("golden_bf16_gate", 2, 24, 8, 4, "bf16", gate=True, seed=101),
    ScanWorkload("golden_f32_nogate", 1, 19, 5, 16, "f32", gate=False, seed=102,
                 skip_ones=True),
]


def _lst(t):
    return None if t is None else t.float().flatten().tolist()


def main():
    orc = oracle.default()
    out = {"note": "inputs from the seeded generator; expected values from the "
                   "float64 oracle (tests/golden/make_golden.py)", "cases": []}
    for w in CASES:
        inp = make_scan_inputs(w)
        y, hs = orc.fwd(*(None if inp[k] is None else inp[k].double().numpy()
                          for k in ("x", "delta", "A", "B", "C", "D", "z",
                                    "delta_bias")), softplus=True, threads=1)
        # the gradient for a seeded dy (an input of the fixture, stored with it)
        dy = np.random.default_rng(w.seed).standard_normal(y.shape)
        g = orc.bwd(*(None if inp[k] is None else inp[k].double().numpy()
                      for k in ("x", "delta", "A", "B", "C", "D", "z", "delta_bias")),
                    softplus=True, dy=dy, threads=1)
        out["cases"].append({
            "name": w.name, "batch": w.batch, "seqlen": w.seqlen, "dim": w.dim,
            "dstate": w.dstate, "dtype": w.dtype, "gate": w.gate,
            "inputs": {k: _lst(inp[k]) for k in inp},
            "y": y.flatten().tolist(), "final_state": hs.flatten().tolist(),
            "dy": dy.flatten().tolist(),
            "grads": {k: (None if v is None else v.flatten().tolist())
                      for k, v in g.items() if k != "dh0"},
        })
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                        "oracle_small.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=0)
    print("wrote", path)


if __name__ == "__main__":
    main()
