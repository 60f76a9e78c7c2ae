"""The float64 oracle against closed forms, invariants, library routines and
brute force (CPU only)."""
import pytest
from hypothesis import given, settings, strategies as st

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



@settings(max_examples=60, deadline=None)
@given(batch=st.integers(1, 2), L=st.integers(1, 9), D=st.integers(1, 4), N=st.integers(1, 7),
       seed=st.integers(0, 10_000), gate=st.booleans(), softplus=st.booleans(),
       zoh=st.booleans(), chunk=st.integers(1, 12))
def test_recurrence_equals_unrolled_sum_any_shape(orc, batch, L, D, N, seed, gate, softplus,
                                                  zoh, chunk):
    """On every tiny shape the C recurrence equals the unrolled closed sum
    (one exponential of a sum of Δ per term, no running product), and the
    chunk-aggregate / carry / rescan form equals the plain scan for any chunk
    length, shorter or longer than the sequence."""
    import numpy as np
    c = oracle_pins._rand_case(seed, batch=batch, L=L, D=D, N=N, gate=gate)
    if not softplus:
        c["delta"] = np.abs(c["delta"]) + 0.05
        c["delta_bias"] = np.zeros_like(c["delta_bias"])
    args = (c["x"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"], c["delta_bias"])
    y, hs = orc.fwd(*args, softplus=softplus, bbar=int(zoh), threads=1)
    ye, he = oracle_pins.explicit_sum_fwd(c, softplus=softplus, zoh=zoh)
    assert oracle_pins._rel(y, ye) < 1e-12
    assert oracle_pins._rel(hs, he) < 1e-12
    yc, hc = orc.fwd_chunked(*args, softplus=softplus, bbar=int(zoh), chunk=chunk, threads=1)
    assert oracle_pins._rel(yc, y) < 1e-12
    assert oracle_pins._rel(hc, hs) < 1e-12


@settings(max_examples=40, deadline=None)
@given(batch=st.integers(1, 2), L=st.integers(1, 8), D=st.integers(1, 3), N=st.integers(1, 20),
       seed=st.integers(0, 10_000), gate=st.booleans(), softplus=st.booleans(),
       zoh=st.booleans(), with_h0=st.booleans())
def test_gradient_directional_derivative_any_shape(orc, batch, L, D, N, seed, gate, softplus,
                                                   zoh, with_h0):
    """For the loss Σ dy·y + Σ dfinal·h_last, the reverse sweep's gradients
    dotted with a random direction v through every input at once equal the
    central difference of the forward oracle along v, on every tiny shape."""
    import numpy as np
    c, dy, dfinal = oracle_pins._bwd_case(seed, gate=gate, with_h0=with_h0, batch=batch, L=L,
                                          D=D, N=N)
    if not softplus:
        c["delta"] = np.abs(c["delta"]) + 0.05
        c["delta_bias"] = np.full_like(c["delta_bias"], 0.01)
    names = [k for k in oracle_pins._BWD_GRADS if c[k] is not None]
    r = np.random.default_rng(seed + 77)
    v = {k: r.standard_normal(c[k].shape) for k in names}

    def inputs(cc):
        return (cc["x"], cc["delta"], cc["A"], cc["B"], cc["C"], cc["D"], cc["z"],
                cc["delta_bias"])

    def loss(eps):
        cc = dict(c)
        for k in names:
            cc[k] = c[k] + eps * v[k]
        y, hs = orc.fwd(*inputs(cc), softplus=softplus, bbar=int(zoh), h0=cc["h0"], threads=1)
        return float(np.sum(dy * y) + np.sum(dfinal * hs))

    g = orc.bwd(*inputs(c), softplus=softplus, bbar=int(zoh), h0=c["h0"], dy=dy,
                dfinal=dfinal, threads=1)
    terms = [g[oracle_pins._BWD_GRADS[k]] * v[k] for k in names]
    want = sum(float(np.sum(t)) for t in terms)
    scale = sum(float(np.sum(np.abs(t))) for t in terms)
    eps = 1e-6
    fd = (loss(eps) - loss(-eps)) / (2 * eps)
    assert abs(fd - want) <= 1e-6 * max(scale, 1e-12), (fd, want, scale)


@settings(max_examples=60, deadline=None)
@given(batch=st.integers(1, 2), L=st.integers(1, 12), D=st.integers(1, 4), K=st.integers(1, 4),
       seed=st.integers(0, 10_000), bias=st.booleans(), silu=st.booleans())
def test_conv1d_equals_library_convolution_any_shape(orc, batch, L, D, K, seed, bias, silu):
    """The causal conv against numpy's full convolution with the reversed
    filter on every small shape, sequences shorter than the filter included."""
    import numpy as np
    import scipy.special
    r = np.random.default_rng(seed)
    x = r.standard_normal((batch, L, D))
    w = r.standard_normal((D, K))
    cb = r.standard_normal(D) if bias else None
    got = orc.causal_conv1d(x, w, cb, silu=silu)
    ref = np.empty_like(x)
    for b in range(batch):
        for d in range(D):
            pre = np.convolve(x[b, :, d], w[d, ::-1])[:L] + (cb[d] if bias else 0.0)
            ref[b, :, d] = pre * scipy.special.expit(pre) if silu else pre
    assert oracle_pins._rel(got, ref) < 1e-13


@settings(max_examples=50, deadline=None)
@given(batch=st.integers(1, 2), L=st.integers(1, 8), D=st.integers(1, 4), N=st.integers(1, 7),
       seed=st.integers(0, 10_000), gate=st.booleans(), softplus=st.booleans())
def test_decode_steps_equal_the_scan_any_shape(orc, batch, L, D, N, seed, gate, softplus):
    """Recurrent inference token by token from an initial state gives the
    whole-sequence scan from that state: the same y at every token and the
    same final state, on every small shape."""
    import numpy as np
    c = oracle_pins._rand_case(seed, batch=batch, L=L, D=D, N=N, gate=gate)
    if not softplus:
        c["delta"] = np.abs(c["delta"]) + 0.05
        c["delta_bias"] = np.zeros_like(c["delta_bias"])
    h0 = np.random.default_rng(seed + 9).standard_normal((batch, D, N))
    y, hs = orc.fwd(c["x"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                    c["delta_bias"], softplus=softplus, h0=h0, threads=1)
    st_ = h0
    for t in range(L):
        yt, st_ = orc.state_update(st_, c["x"][:, t], c["delta"][:, t], c["A"], c["B"][:, t],
                                   c["C"][:, t], c["D"], None if c["z"] is None else c["z"][:, t],
                                   c["delta_bias"], softplus=softplus)
        assert oracle_pins._rel(yt, y[:, t]) < 1e-13
    assert oracle_pins._rel(st_, hs) < 1e-13
