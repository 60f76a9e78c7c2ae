"""The float64 oracle against closed forms, invariants, library routines and
brute force (CPU only)."""
import pytest

import oracle_pins


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_threads_do_not_change_results(orc):
    """OpenMP spreads independent chains only: 1 thread and many threads give
    bit-identical results."""
    import numpy as np
    c = oracle_pins._rand_case(21, batch=3, L=50, D=17, N=16)
    args = (c["x"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
            c["delta_bias"])
    y1, h1 = orc.fwd(*args, threads=1)
    y8, h8 = orc.fwd(*args, threads=8)
    assert np.array_equal(y1, y8) and np.array_equal(h1, h8)


def test_bwd_threads_agree(orc):
    """The backward oracle with 1 and 8 threads: per-element outputs are
    identical; the channel sums dB, dC differ only in rounding order."""
    import numpy as np
    c = oracle_pins._rand_case(22, batch=2, L=40, D=19, N=16)
    r = np.random.default_rng(23)
    dy = r.standard_normal(c["x"].shape)
    args = (c["x"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
            c["delta_bias"])
    g1 = orc.bwd(*args, dy=dy, threads=1)
    g8 = orc.bwd(*args, dy=dy, threads=8)
    for k in ("dx", "ddelta", "dz", "dA", "dD", "ddelta_bias"):
        assert np.array_equal(g1[k], g8[k]), k
    for k in ("dB", "dC"):
        assert np.allclose(g1[k], g8[k], rtol=1e-13, atol=1e-13), k
