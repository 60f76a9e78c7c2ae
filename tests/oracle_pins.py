"""Pins of the float64 oracle against facts other than the oracle itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when the oracle disagrees with a closed form, an invariant, a library routine
or an independent brute-force formula. ``test_oracle_pins.py`` runs them on
the real oracle; ``test_oracle_mutants.py`` runs them on oracles with planted
mistakes and checks that every mistake trips at least one pin.

Pages (title, section) the facts come from:
  "Mamba & State Space Models — Guide Complet" (Guide Complet): §1
  "Discrétisation" (ZOH formulas, discrete recurrence), §2 "S4" (convolution
  kernel K = (CB, CAB, CA²B, …), y = K * u), §4 "Implémentation du SSM
  sélectif (S6)" and "Parallel Associative Scan".
  "Mamba и State Space Models: альтернатива Transformer" (johe.ru): "SSM as
  RNN", "SSM as Convolution", "Hardware-Aware Scan".
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np
import scipy.linalg
import scipy.special

RNG = np.random.default_rng


def _rel(a, b):
    """Max |a − b| over max |b|; infinite when either side holds a NaN or an
    infinity, so that a non-finite result never passes a bound."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    if not a.size:
        return 0.0
    if not (np.isfinite(a).all() and np.isfinite(b).all()):
        return math.inf
    scale = max(float(np.max(np.abs(b))), 1e-300)
    return float(np.max(np.abs(a - b))) / scale


def _rand_case(seed, batch=2, L=7, D=3, N=4, gate=True):
    r = RNG(seed)
    c = dict(
        x=r.standard_normal((batch, L, D)),
        delta=0.5 * r.standard_normal((batch, L, D)),
        A=-np.exp(r.uniform(-1.0, 1.5, (D, N))),
        B=r.standard_normal((batch, L, N)),
        C=r.standard_normal((batch, L, N)),
        D=1.0 + 0.1 * r.standard_normal(D),
        z=r.standard_normal((batch, L, D)) if gate else None,
        delta_bias=np.log(np.expm1(r.uniform(1e-3, 1e-1, D))),
    )
    return c


def _softplus(v):
    return np.logaddexp(0.0, v)


def explicit_sum_fwd(c, softplus=True, zoh=False):
    """Brute force, no recurrence: the unrolled form of the discrete system
    (Guide Complet §1 with §4's per-token Δ, B, C),
        h_t[n] = Σ_{s≤t} exp(A[n]·Σ_{s<k≤t} Δ_k) · Bbar_s[n] · x_s,
    with the decay taken as ONE exponential of a sum of Δ (never a running
    product), then y_t = Σ_n C_t[n] h_t[n] + D x_t, times silu(z_t)."""
    x, A, B, C = c["x"], c["A"], c["B"], c["C"]
    batch, L, D = x.shape
    N = A.shape[1]
    v = c["delta"] + c["delta_bias"][None, None, :]
    dt = _softplus(v) if softplus else v
    y = np.zeros_like(x)
    hL = np.zeros((batch, D, N))
    for b in range(batch):
        for d in range(D):
            cum = np.concatenate([[0.0], np.cumsum(dt[b, :, d])])  # cum[t+1]=Σ_{k≤t}
            for t in range(L):
                h = np.zeros(N)
                for s in range(t + 1):
                    decay = np.exp(A[d] * (cum[t + 1] - cum[s + 1]))
                    if zoh:
                        coef = np.expm1(dt[b, s, d] * A[d]) / A[d]
                    else:
                        coef = dt[b, s, d]
                    h += decay * coef * B[b, s] * x[b, s, d]
                out = float(C[b, t] @ h) + c["D"][d] * x[b, t, d]
                if c["z"] is not None:
                    out *= float(scipy.special.expit(c["z"][b, t, d])) * c["z"][b, t, d]
                y[b, t, d] = out
                if t == L - 1:
                    hL[b, d] = h
    return y, hL


# --------------------------------------------------------------------------- #
def pin_explicit_sum(orc):
    """Recurrence == unrolled closed sum (both input-term modes, gate on/off,
    softplus on/off)."""
    for seed, gate, sp, zoh in [(1, True, True, False), (2, False, True, False),
                                (3, True, False, False), (4, True, True, True)]:
        c = _rand_case(seed, gate=gate)
        if not sp:
            c["delta"] = np.abs(c["delta"]) + 0.05
            c["delta_bias"] = np.zeros_like(c["delta_bias"])
        y, hs = orc.fwd(c["x"], c["delta"], c["A"], c["B"], c["C"], c["D"],
                        c["z"], c["delta_bias"], softplus=sp, bbar=int(zoh),
                        threads=1)
        ye, he = explicit_sum_fwd(c, softplus=sp, zoh=zoh)
        assert _rel(y, ye) < 1e-12, ("explicit sum y", seed, _rel(y, ye))
        assert _rel(hs, he) < 1e-12, ("explicit sum state", seed)


def pin_single_token(orc):
    """L = 1 closed form: h = Δ B x, y = (Σ_n C_n B_n) Δ x + D x, gated."""
    c = _rand_case(5, batch=3, L=1, D=4, N=6)
    y, hs = orc.fwd(c["x"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                    c["delta_bias"], threads=1)
    dt = _softplus(c["delta"][:, 0, :] + c["delta_bias"])  # [b, d]
    x0 = c["x"][:, 0, :]
    cb = np.einsum("bn,bn->b", c["C"][:, 0], c["B"][:, 0])
    z0 = c["z"][:, 0, :]
    ye = (cb[:, None] * dt * x0 + c["D"] * x0) * z0 * scipy.special.expit(z0)
    he = dt[:, :, None] * c["B"][:, 0][:, None, :] * x0[:, :, None]
    assert _rel(y[:, 0, :], ye) < 1e-14, "single token y"
    assert _rel(hs, he) < 1e-14, "single token state"


def pin_lti_convolution(orc):
    """With Δ, B, C constant in t the scan is the LTI convolution of
    "SSM as Convolution" / Guide Complet §2: y = K * x + D x with
    K_k = Σ_n C[n]·exp(kΔA[n])·ΔB[n]; the convolution is numpy's."""
    r = RNG(6)
    L, D, N = 300, 3, 5
    A = -np.exp(r.uniform(-2, 1, (D, N)))
    Bv = r.standard_normal(N)
    Cv = r.standard_normal(N)
    dtv = r.uniform(0.01, 0.3, D)
    x = r.standard_normal((1, L, D))
    delta = np.broadcast_to(dtv, (1, L, D)).copy()
    B = np.broadcast_to(Bv, (1, L, N)).copy()
    C = np.broadcast_to(Cv, (1, L, N)).copy()
    Dv = r.standard_normal(D)
    y, _ = orc.fwd(x, delta, A, B, C, Dv, None, None, softplus=False,
                   threads=1)
    k = np.arange(L)[:, None]
    for d in range(D):
        K = (Cv[None, :] * np.exp(k * dtv[d] * A[d][None, :]) * dtv[d]
             * Bv[None, :]).sum(axis=1)
        ye = np.convolve(x[0, :, d], K)[:L] + Dv[d] * x[0, :, d]
        assert _rel(y[0, :, d], ye) < 1e-12, ("lti conv", d, _rel(y[0, :, d], ye))


def pin_zoh_matrix(orc):
    """Diagonal ZOH equals the matrix formulas of Guide Complet §1,
    A_bar = expm(ΔA), B_bar = (A_bar − I)·A⁻¹·B, evaluated with scipy."""
    r = RNG(7)
    N = 6
    A = -np.exp(r.uniform(-1, 2, N))
    B = r.standard_normal(N)
    for dt in (1e-3, 0.05, 0.7, 3.0):
        Ab, Bb = orc.zoh_discretize(dt, A, B)
        Am = np.diag(A)
        Abm = scipy.linalg.expm(dt * Am)
        Bbm = (Abm - np.eye(N)) @ np.linalg.inv(Am) @ B
        assert _rel(Ab, np.diag(Abm)) < 1e-13, ("zoh A_bar", dt)
        assert _rel(Bb, Bbm) < 1e-12, ("zoh B_bar", dt)
    # the A → 0 limit is Δ·B
    Ab, Bb = orc.zoh_discretize(0.25, np.zeros(3), np.array([1.0, -2.0, 4.0]))
    assert np.array_equal(Ab, np.ones(3)) and _rel(Bb, [0.25, -0.5, 1.0]) < 1e-15


def pin_euler_vs_zoh(orc):
    """The two input terms differ by Δ²·A·B/2 + O(Δ³) (Taylor of
    (e^{ΔA} − 1)/A): checked through one token, where
    y_zoh − y_delta = Σ_n C_n B_n x (Δ²A_n/2 + …)."""
    c = _rand_case(8, batch=1, L=1, D=2, N=4, gate=False)
    c["delta_bias"] = np.zeros(2)
    for dt in (1e-3, 5e-4):
        delta = np.full((1, 1, 2), dt)
        y1, _ = orc.fwd(c["x"], delta, c["A"], c["B"], c["C"], c["D"], None,
                        None, softplus=False, bbar=0, threads=1)
        y2, _ = orc.fwd(c["x"], delta, c["A"], c["B"], c["C"], c["D"], None,
                        None, softplus=False, bbar=1, threads=1)
        lead = np.array([np.sum(c["C"][0, 0] * c["B"][0, 0] * c["A"][d]) * dt * dt
                         / 2 * c["x"][0, 0, d] for d in range(2)])
        assert np.max(np.abs((y2 - y1)[0, 0] - lead)) < 5 * dt * np.max(np.abs(lead)), \
            "euler vs zoh second order"


def pin_linearity(orc):
    """For fixed Δ, B, C, z the map x -> y is linear ("SSM as RNN": h and y
    are linear in the input)."""
    c = _rand_case(9, batch=2, L=20, D=3, N=4)
    r = RNG(10)
    x1, x2 = c["x"], r.standard_normal(c["x"].shape)
    al, be = 1.7, -0.6
    args = (c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"], c["delta_bias"])
    y1, h1 = orc.fwd(x1, *args, threads=1)
    y2, h2 = orc.fwd(x2, *args, threads=1)
    y3, h3 = orc.fwd(al * x1 + be * x2, *args, threads=1)
    assert _rel(y3, al * y1 + be * y2) < 1e-12, "linearity y"
    assert _rel(h3, al * h1 + be * h2) < 1e-12, "linearity state"


def pin_delta_to_zero(orc):
    """Δ → 0: A_bar → 1 and Δ·B → 0, so the decode state is unchanged and the
    output reduces to the gated skip D·x·silu(z)."""
    c = _rand_case(11, batch=2, L=5, D=3, N=4)
    tiny = np.full(c["x"].shape, 1e-12)
    y, hs = orc.fwd(c["x"], tiny, c["A"], c["B"], c["C"], c["D"], c["z"], None,
                    softplus=False, threads=1)
    ye = c["D"] * c["x"] * c["z"] * scipy.special.expit(c["z"])
    assert np.max(np.abs(y - ye)) < 1e-10, "delta->0 output"
    assert np.max(np.abs(hs)) < 1e-10, "delta->0 state from zero"
    r = RNG(12)
    st = r.standard_normal((2, 3, 4))
    yd, st2 = orc.state_update(st, c["x"][:, 0], tiny[:, 0], c["A"], c["B"][:, 0],
                               c["C"][:, 0], c["D"], c["z"][:, 0], None,
                               softplus=False)
    assert _rel(st2, st) < 1e-10, "delta->0 decode state"


def pin_chunked(orc):
    """Chunk aggregates + carry + rescan ("Hardware-Aware Scan" blocks with
    the Guide Complet operator) == the plain sequential scan."""
    c = _rand_case(13, batch=2, L=40, D=3, N=4)
    ref = orc.fwd(c["x"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                  c["delta_bias"], threads=1)
    for chunk in (1, 7, 16, 39, 40, 256):
        got = orc.fwd_chunked(c["x"], c["delta"], c["A"], c["B"], c["C"], c["D"],
                              c["z"], c["delta_bias"], chunk=chunk, threads=1)
        assert _rel(got[0], ref[0]) < 1e-12, ("chunked y", chunk)
        assert _rel(got[1], ref[1]) < 1e-12, ("chunked state", chunk)


def pin_associativity(orc):
    """The operator is associative, and compose(later, earlier) applied to h
    equals applying earlier then later (the affine maps h -> a h + b)."""
    r = RNG(14)
    for _ in range(20):
        e = r.uniform(0.1, 1.0, 3)
        f = r.standard_normal(3)
        left = orc.compose(*orc.compose(e[2], f[2], e[1], f[1]), e[0], f[0])
        right = orc.compose(e[2], f[2], *orc.compose(e[1], f[1], e[0], f[0]))
        assert abs(left[0] - right[0]) < 1e-15 and abs(left[1] - right[1]) < 1e-14
        h = r.standard_normal()
        a, b = orc.compose(e[1], f[1], e[0], f[0])
        assert abs((a * h + b) - (e[1] * (e[0] * h + f[0]) + f[1])) < 1e-14


def pin_geometric(orc):
    """Constant Δ, B and x = 1: h_t = ΔB (1 − A_bar^{t+1}) / (1 − A_bar), a
    geometric series; checked over a long sequence (state continuity)."""
    L, D, N = 4000, 2, 3
    A = np.array([[-0.5, -1.0, -4.0], [-0.01, -2.0, -16.0]])
    dtv = np.array([1e-3, 0.2])
    Bv = np.array([0.7, -1.3, 2.0])
    Cv = np.array([1.1, 0.4, -0.9])
    x = np.ones((1, L, D))
    delta = np.broadcast_to(dtv, (1, L, D)).copy()
    B = np.broadcast_to(Bv, (1, L, N)).copy()
    C = np.broadcast_to(Cv, (1, L, N)).copy()
    y, hs = orc.fwd(x, delta, A, B, C, None, None, None, softplus=False,
                    threads=1)
    for d in range(D):
        ab = np.exp(dtv[d] * A[d])
        t = np.arange(L)[:, None]
        h = dtv[d] * Bv * (1 - ab ** (t + 1)) / (1 - ab)
        assert _rel(y[0, :, d], h @ Cv) < 1e-10, ("geometric y", d)
        assert _rel(hs[0, d], h[-1]) < 1e-10, ("geometric state", d)


def pin_decay(orc):
    """x = 0 after t0: h_L = exp(A·Σ_{t>t0} Δ_t) ⊙ h_{t0} (pure decay)."""
    c = _rand_case(15, batch=1, L=50, D=3, N=4, gate=False)
    t0 = 20
    x = c["x"].copy()
    x[:, t0:, :] = 0.0
    _, h_t0 = orc.fwd(x[:, :t0], c["delta"][:, :t0], c["A"], c["B"][:, :t0],
                      c["C"][:, :t0], c["D"], None, c["delta_bias"], threads=1)
    _, h_L = orc.fwd(x, c["delta"], c["A"], c["B"], c["C"], c["D"], None,
                     c["delta_bias"], threads=1)
    dt = _softplus(c["delta"][0] + c["delta_bias"])  # [L, D]
    s = dt[t0:].sum(axis=0)  # [D]
    he = np.exp(c["A"] * s[:, None]) * h_t0[0]
    assert _rel(h_L[0], he) < 1e-12, "decay"


def pin_cross_entry(orc):
    """L single-token steps from a zero state reproduce the sequence scan,
    and a scan resumed from a prefix's final state reproduces the rest."""
    c = _rand_case(16, batch=2, L=12, D=3, N=4)
    y, hs = orc.fwd(c["x"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                    c["delta_bias"], threads=1)
    st = np.zeros((2, 3, 4))
    for t in range(12):
        yt, st = orc.state_update(st, c["x"][:, t], c["delta"][:, t], c["A"],
                                  c["B"][:, t], c["C"][:, t], c["D"], c["z"][:, t],
                                  c["delta_bias"])
        assert _rel(yt, y[:, t]) < 1e-13, ("decode vs fwd", t)
    assert _rel(st, hs) < 1e-13, "decode final state"
    L1 = 5
    sl = lambda a, s: None if a is None else a[:, s]  # noqa: E731
    _, h1 = orc.fwd(sl(c["x"], slice(0, L1)), sl(c["delta"], slice(0, L1)), c["A"],
                    sl(c["B"], slice(0, L1)), sl(c["C"], slice(0, L1)), c["D"],
                    sl(c["z"], slice(0, L1)), c["delta_bias"], threads=1)
    y2, h2 = orc.fwd(sl(c["x"], slice(L1, None)), sl(c["delta"], slice(L1, None)),
                     c["A"], sl(c["B"], slice(L1, None)), sl(c["C"], slice(L1, None)),
                     c["D"], sl(c["z"], slice(L1, None)), c["delta_bias"], h0=h1,
                     threads=1)
    assert _rel(y2, y[:, L1:]) < 1e-13 and _rel(h2, hs) < 1e-13, "resume"


def pin_decode_layout(orc):
    """State layout [batch, D, N] with n fastest, checked exactly: with A = 0
    (A_bar = 1) and x = 0 the state comes back bit-identical; a one-hot x at
    (b0, d0) with B one-hot at n0 changes exactly state[b0, d0, n0], by Δ·B·x."""
    r = RNG(17)
    batch, D, N = 3, 5, 4
    st = r.standard_normal((batch, D, N))
    A = np.zeros((D, N))
    delta = r.uniform(0.1, 1.0, (batch, D))
    Bm = r.standard_normal((batch, N))
    Cm = r.standard_normal((batch, N))
    _, st2 = orc.state_update(st, np.zeros((batch, D)), delta, A, Bm, Cm,
                              softplus=False)
    assert np.array_equal(st2, st), "A=0, x=0 must leave the state bit-identical"
    b0, d0, n0 = 2, 3, 1
    x = np.zeros((batch, D))
    x[b0, d0] = 1.5
    Bo = np.zeros((batch, N))
    Bo[b0, n0] = -0.75
    _, st3 = orc.state_update(st, x, delta, A, Bo, Cm, softplus=False)
    diff = st3 != st
    assert diff.sum() == 1 and diff[b0, d0, n0], "one-hot must touch one element"
    assert st3[b0, d0, n0] == st[b0, d0, n0] + delta[b0, d0] * -0.75 * 1.5


def pin_softplus_and_gate(orc):
    """Δ = softplus(delta + bias) for both signs, including large |v|, and
    the gate silu(z) = z·expit(z), read back through a 1-state scan whose
    output is exactly Δ (A = 0, B = C = x = 1, D = 0) or D·x·silu(z) (B = 0)."""
    v = np.array([-40.0, -12.0, -3.0, -1e-3, 0.0, 1e-3, 2.5, 19.0, 45.0])
    Lv = v.size
    bias = np.array([0.125])
    x = np.ones((1, Lv, 1))
    y, _ = orc.fwd(x, (v - 0.125)[None, :, None], np.zeros((1, 1)),
                   np.ones((1, Lv, 1)), np.ones((1, Lv, 1)), None, None, bias,
                   threads=1)
    cum = np.cumsum([math.log1p(math.exp(t)) if t < 30 else t + math.log1p(math.exp(-t))
                     for t in v])
    assert _rel(y[0, :, 0], cum) < 1e-14, "softplus"
    z = np.array([-30.0, -2.0, -1e-4, 0.0, 0.7, 8.0, 30.0])
    Lz = z.size
    y, _ = orc.fwd(np.full((1, Lz, 1), 2.0), np.zeros((1, Lz, 1)), np.zeros((1, 1)),
                   np.zeros((1, Lz, 1)), np.ones((1, Lz, 1)), np.array([0.5]),
                   z[None, :, None], None, threads=1)
    assert _rel(y[0, :, 0], 1.0 * z * scipy.special.expit(z)) < 1e-15, "silu gate"


def pin_hand_worked(orc):
    """A hand-worked example in exact arithmetic (Fractions): one channel,
    N = 2, A = (0, −ln 2) and Δ = 1 give A_bar = (1, 1/2); the recurrence of
    Guide Complet §1 with the delta-scaled input of "SSM as RNN"."""
    x = [Fraction(1), Fraction(2), Fraction(-1)]
    Bs = [(1, 1), (0, 2), (1, 0)]
    Cs = [(1, 0), (1, 1), (0, 2)]
    Dsk = Fraction(1, 2)
    ab = (Fraction(1), Fraction(1, 2))
    h = [Fraction(0), Fraction(0)]
    ye = []
    for t in range(3):
        h = [ab[n] * h[n] + Bs[t][n] * x[t] for n in range(2)]
        ye.append(sum(Cs[t][n] * h[n] for n in range(2)) + Dsk * x[t])
    # ye == [3/2, 13/2, 4], final h == [0, 9/4]
    y, hs = orc.fwd(np.array(x, dtype=float)[None, :, None], np.ones((1, 3, 1)),
                    np.array([[0.0, -math.log(2.0)]]),
                    np.array(Bs, dtype=float)[None], np.array(Cs, dtype=float)[None],
                    np.array([0.5]), None, None, softplus=False, threads=1)
    assert _rel(y[0, :, 0], [float(v) for v in ye]) < 1e-15, "hand-worked y"
    assert _rel(hs[0, 0], [float(v) for v in h]) < 1e-15, "hand-worked state"


# ---------------------------------------------------------------------------
# Backward pass (gradient of the scan). The loss is Σ dy·y + Σ dfinal·h_{L−1};
# the pins below check the oracle's reverse sweep against numerical
# differentiation of the (separately pinned) forward, against exact
# homogeneity identities of the recurrence, and against closed forms.

_BWD_GRADS = {"x": "dx", "delta": "ddelta", "A": "dA", "B": "dB", "C": "dC",
              "D": "dD", "z": "dz", "delta_bias": "ddelta_bias", "h0": "dh0"}


def _bwd_case(seed, gate=True, with_h0=True, batch=2, L=5, D=3, N=4):
    c = _rand_case(seed, batch=batch, L=L, D=D, N=N, gate=gate)
    r = RNG(seed + 1000)
    c["h0"] = r.standard_normal((batch, D, N)) if with_h0 else None
    dy = r.standard_normal((batch, L, D))
    dfinal = r.standard_normal((batch, D, N))
    return c, dy, dfinal


def _fwd_of(orc, c, softplus):
    return orc.fwd(c["x"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                   c["delta_bias"], softplus=softplus, h0=c["h0"], threads=1)


def _bwd_of(orc, c, dy, dfinal, softplus):
    return orc.bwd(c["x"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"],
                   c["delta_bias"], softplus=softplus, h0=c["h0"], dy=dy,
                   dfinal=dfinal, threads=1)


def pin_bwd_finite_differences(orc):
    """Every gradient against central differences of the forward oracle,
    element by element, with and without softplus, gate and initial state."""
    for seed, softplus, gate, with_h0 in ((40, True, True, True),
                                          (41, False, False, False)):
        c, dy, dfinal = _bwd_case(seed, gate=gate, with_h0=with_h0)
        if not softplus:  # Δ = delta + bias itself: keep it positive
            c["delta"] = np.abs(c["delta"]) + 0.05
            c["delta_bias"] = np.full_like(c["delta_bias"], 0.01)
        g = _bwd_of(orc, c, dy, dfinal, softplus)

        def loss(cc):
            y, hs = _fwd_of(orc, cc, softplus)
            return float(np.sum(dy * y) + np.sum(dfinal * hs))

        for name, gname in _BWD_GRADS.items():
            if c[name] is None:
                assert g[gname] is None, f"{gname} returned without {name}"
                continue
            arr = c[name]
            fd = np.zeros_like(arr)
            for idx in np.ndindex(arr.shape):
                e = 1e-6 * max(1.0, abs(arr[idx]))
                cp = dict(c)
                cp[name] = arr.copy()
                cp[name][idx] += e
                cm = dict(c)
                cm[name] = arr.copy()
                cm[name][idx] -= e
                fd[idx] = (loss(cp) - loss(cm)) / (2 * e)
            assert _rel(g[gname], fd) < 1e-6, f"{gname} vs finite differences"


def pin_bwd_wide_state_finite_differences(orc):
    """The gradient at d_state 20 (more states than one 16-state group of the
    CUDA gradient) against central differences of the forward oracle, element
    by element, with gate and initial state."""
    c, dy, dfinal = _bwd_case(47, gate=True, with_h0=True, batch=1, L=4, D=2, N=20)
    g = _bwd_of(orc, c, dy, dfinal, True)

    def loss(cc):
        y, hs = _fwd_of(orc, cc, True)
        return float(np.sum(dy * y) + np.sum(dfinal * hs))

    for name, gname in _BWD_GRADS.items():
        arr = c[name]
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            e = 1e-6 * max(1.0, abs(arr[idx]))
            cp = dict(c)
            cp[name] = arr.copy()
            cp[name][idx] += e
            cm = dict(c)
            cm[name] = arr.copy()
            cm[name][idx] -= e
            fd[idx] = (loss(cp) - loss(cm)) / (2 * e)
        assert _rel(g[gname], fd) < 1e-6, f"N=20 {gname} vs finite differences"


def pin_bwd_zoh_finite_differences(orc):
    """The gradient with the ZOH input term c·B·x, c = (exp(Δ·A) − 1)/A
    ([Guide] §1), against central differences of the forward oracle in the
    same mode, element by element; one A entry is 0 (the c → Δ limit)."""
    c, dy, dfinal = _bwd_case(45, gate=True, with_h0=True)
    c["A"] = c["A"].copy()
    c["A"][0, 1] = 0.0
    g = orc.bwd(c["x"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"], c["delta_bias"],
                h0=c["h0"], dy=dy, dfinal=dfinal, threads=1, bbar=1)

    def loss(cc):
        y, hs = orc.fwd(cc["x"], cc["delta"], cc["A"], cc["B"], cc["C"], cc["D"], cc["z"],
                        cc["delta_bias"], h0=cc["h0"], threads=1, bbar=1)
        return float(np.sum(dy * y) + np.sum(dfinal * hs))

    for name, gname in _BWD_GRADS.items():
        arr = c[name]
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            e = 1e-6 * max(1.0, abs(arr[idx]))
            cp = dict(c)
            cp[name] = arr.copy()
            cp[name][idx] += e
            cm = dict(c)
            cm[name] = arr.copy()
            cm[name][idx] -= e
            fd[idx] = (loss(cp) - loss(cm)) / (2 * e)
        assert _rel(g[gname], fd) < 1e-6, f"ZOH {gname} vs finite differences"
    # the input-term gradients differ from the Euler ones (the pin has teeth)
    ge = orc.bwd(c["x"], c["delta"], c["A"], c["B"], c["C"], c["D"], c["z"], c["delta_bias"],
                 h0=c["h0"], dy=dy, dfinal=dfinal, threads=1)
    assert _rel(g["dA"], ge["dA"]) > 1e-3 and _rel(g["dx"], ge["dx"]) > 1e-4


def pin_bwd_homogeneity(orc):
    """Exact identities (no truncation error). Without the gate, y and h_{L−1}
    are linear in (x, h0) jointly, and y − D·x and h_{L−1} are linear in
    (B, h0) jointly and y − D·x in C; Euler's theorem for such maps gives
        Σ dy·y + Σ dfinal·h_{L−1} = Σ dx·x + Σ dh0·h0,
        Σ dy·(y − D·x) + Σ dfinal·h_{L−1} = Σ dB·B + Σ dh0·h0,
        Σ dy·(y − D·x) = Σ dC·C (with dfinal = 0),   Σ dD·D = Σ dy·D·x."""
    c, dy, dfinal = _bwd_case(50, gate=False, with_h0=True, L=9, D=4, N=5)
    y, hs = _fwd_of(orc, c, True)
    g = _bwd_of(orc, c, dy, dfinal, True)
    dx_ = c["D"][None, None, :] * c["x"]
    lhs1 = np.sum(dy * y) + np.sum(dfinal * hs)
    rhs1 = np.sum(g["dx"] * c["x"]) + np.sum(g["dh0"] * c["h0"])
    assert abs(lhs1 - rhs1) < 1e-12 * max(1.0, abs(lhs1)), "x/h0 homogeneity"
    lhs2 = np.sum(dy * (y - dx_)) + np.sum(dfinal * hs)
    rhs2 = np.sum(g["dB"] * c["B"]) + np.sum(g["dh0"] * c["h0"])
    assert abs(lhs2 - rhs2) < 1e-12 * max(1.0, abs(lhs2)), "B/h0 homogeneity"
    g0 = _bwd_of(orc, c, dy, np.zeros_like(dfinal), True)
    lhs3 = np.sum(dy * (y - dx_))
    assert abs(lhs3 - np.sum(g0["dC"] * c["C"])) < 1e-12 * max(1.0, abs(lhs3)), \
        "C homogeneity"
    lhs4 = np.sum(dy * dx_)
    assert abs(lhs4 - np.sum(g0["dD"] * c["D"])) < 1e-12 * max(1.0, abs(lhs4)), \
        "D homogeneity"


def pin_bwd_single_token(orc):
    """L = 1 from a zero state, no gate, softplus off: y = Σ_n C B Δ x + D x,
    h = Δ x B, so with u = Δ·x
        dx = dy (Σ C B Δ + D) + Δ Σ dfinal·B,   dΔ = x (dy Σ C B + Σ dfinal·B),
        dB = (dy C + dfinal) Δ x (summed over channels),  dC = dy Δ x B
        (summed over channels),  dA = 0,  dD = dy x."""
    r = RNG(60)
    D, N = 3, 4
    x = r.standard_normal((1, 1, D))
    dl = r.uniform(0.1, 0.9, (1, 1, D))
    A = -r.uniform(0.5, 2.0, (D, N))
    B = r.standard_normal((1, 1, N))
    C = r.standard_normal((1, 1, N))
    Dv = r.standard_normal(D)
    dy = r.standard_normal((1, 1, D))
    dfin = r.standard_normal((1, D, N))
    g = orc.bwd(x, dl, A, B, C, Dv, None, None, softplus=False, dy=dy,
                dfinal=dfin, threads=1)
    cb = float(np.sum(C * B))
    xv, dt, gy = x[0, 0], dl[0, 0], dy[0, 0]
    fb = dfin[0] @ B[0, 0]                       # Σ_n dfinal[d, n]·B[n]
    assert _rel(g["dx"][0, 0], gy * (cb * dt + Dv) + dt * fb) < 1e-14, "dx"
    assert _rel(g["ddelta"][0, 0], xv * (gy * cb + fb)) < 1e-14, "ddelta"
    dB = np.sum((gy[:, None] * C[0, 0][None, :] + dfin[0]) * (dt * xv)[:, None], axis=0)
    assert _rel(g["dB"][0, 0], dB) < 1e-14, "dB"
    assert _rel(g["dC"][0, 0], np.sum((gy * dt * xv)[:, None] * B[0, 0][None, :], axis=0)) < 1e-14, "dC"
    assert np.all(g["dA"] == 0.0), "dA from a zero state"
    assert _rel(g["dD"], gy * xv) < 1e-14, "dD"


# ---------------------------------------------------------------------------
# Causal depthwise convolution in front of the scan.

def pin_conv1d_library(orc):
    """Each channel against numpy's full convolution with the reversed filter
    (a cross-correlation with K − 1 leading zeros keeps the first L outputs),
    plus the bias, then SiLU; widths 1 to 4."""
    r = RNG(70)
    for K in (1, 2, 3, 4):
        x = r.standard_normal((2, 9, 3))
        w = r.standard_normal((3, K))
        cb = r.standard_normal(3)
        got = orc.causal_conv1d(x, w, cb, silu=True)
        ref = np.empty_like(x)
        for b in range(2):
            for d in range(3):
                pre = np.convolve(x[b, :, d], w[d, ::-1])[:9] + cb[d]
                ref[b, :, d] = pre * scipy.special.expit(pre)
        assert _rel(got, ref) < 1e-13, f"conv width {K}"


def pin_conv1d_impulse(orc):
    """A unit impulse at token t0, no bias, no SiLU: the output from t0 on is
    the filter read backwards (w[K−1] at t0, w[K−2] at t0 + 1, ...), zero
    elsewhere, exactly; and the impulse's channel only."""
    K, L, t0 = 4, 10, 3
    w = np.array([[0.5, -1.0, 2.0, 3.0], [1.0, 1.0, 1.0, 1.0]])
    x = np.zeros((1, L, 2))
    x[0, t0, 0] = 1.0
    got = orc.causal_conv1d(x, w, None, silu=False)
    want = np.zeros((1, L, 2))
    for j in range(K):
        want[0, t0 + j, 0] = w[0, K - 1 - j]
    assert np.array_equal(got, want), "impulse response"


def pin_conv1d_bwd_finite_differences(orc):
    """The conv gradient against central differences of the (pinned) conv,
    for every input, weight and bias element, widths 1 and 4, with and
    without SiLU."""
    r = RNG(80)
    for K, silu in ((4, True), (1, False), (3, True)):
        x = r.standard_normal((2, 6, 3))
        w = r.standard_normal((3, K))
        cb = r.standard_normal(3)
        dxc = r.standard_normal((2, 6, 3))
        dx, dw, dcb = orc.causal_conv1d_bwd(x, w, cb, dxc, silu=silu)

        def loss(xx, ww, bb):
            return float(np.sum(dxc * orc.causal_conv1d(xx, ww, bb, silu=silu)))

        for arr, got, which in ((x, dx, 0), (w, dw, 1), (cb, dcb, 2)):
            fd = np.zeros_like(arr)
            for idx in np.ndindex(arr.shape):
                e = 1e-6 * max(1.0, abs(arr[idx]))
                ap, am = arr.copy(), arr.copy()
                ap[idx] += e
                am[idx] -= e
                args_p = [x, w, cb]
                args_m = [x, w, cb]
                args_p[which], args_m[which] = ap, am
                fd[idx] = (loss(*args_p) - loss(*args_m)) / (2 * e)
            assert _rel(got, fd) < 1e-6, f"conv gradient {which} K={K}"


ALL_PINS = [
    pin_explicit_sum, pin_single_token, pin_lti_convolution, pin_zoh_matrix,
    pin_euler_vs_zoh, pin_linearity, pin_delta_to_zero, pin_chunked,
    pin_associativity, pin_geometric, pin_decay, pin_cross_entry,
    pin_decode_layout, pin_softplus_and_gate, pin_hand_worked,
    pin_bwd_finite_differences, pin_bwd_wide_state_finite_differences,
    pin_bwd_zoh_finite_differences, pin_bwd_homogeneity,
    pin_bwd_single_token,
    pin_conv1d_library, pin_conv1d_impulse, pin_conv1d_bwd_finite_differences,
]
