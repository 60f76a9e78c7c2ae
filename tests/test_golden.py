"""The oracle still reproduces its stored golden fixture (CPU only)."""
import json
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))


def load_golden():
    with open(os.path.join(HERE, "golden", "oracle_small.json")) as f:
        return json.load(f)["cases"]


def golden_arrays(case):
    b, L, D, N = case["batch"], case["seqlen"], case["dim"], case["dstate"]
    shapes = {"x": (b, L, D), "delta": (b, L, D), "z": (b, L, D), "B": (b, L, N),
              "C": (b, L, N), "A": (D, N), "D": (D,), "delta_bias": (D,)}
    inp = {k: (None if v is None else np.asarray(v, dtype=np.float64).reshape(shapes[k]))
           for k, v in case["inputs"].items()}
    return inp, np.asarray(case["y"]).reshape(b, L, D), \
        np.asarray(case["final_state"]).reshape(b, D, N)


def test_oracle_matches_golden(orc):
    for case in load_golden():
        inp, y_ref, h_ref = golden_arrays(case)
        y, h = orc.fwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"],
                       inp["D"], inp["z"], inp["delta_bias"], threads=1)
        assert np.array_equal(y, y_ref), case["name"]
        assert np.array_equal(h, h_ref), case["name"]


def test_oracle_gradient_matches_golden(orc):
    """The gradient for the stored dy: the reverse sweep of the oracle has not
    drifted (its channel sums may round in another order across thread
    counts, hence a relative bound of 1e-13 rather than bit equality)."""
    for case in load_golden():
        inp, y_ref, _ = golden_arrays(case)
        dy = np.asarray(case["dy"]).reshape(y_ref.shape)
        g = orc.bwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["z"],
                    inp["delta_bias"], dy=dy, threads=1)
        for k, ref in case["grads"].items():
            if ref is None:
                assert g[k] is None, (case["name"], k)
                continue
            ref = np.asarray(ref).reshape(g[k].shape)
            scale = max(float(np.max(np.abs(ref))), 1e-300)
            assert float(np.max(np.abs(g[k] - ref))) <= 1e-13 * scale, (case["name"], k)
