"""The matrix (semiseparable) form of the scalar-A-per-head scan, written out
in float64 numpy, against the recurrence oracle, closed forms and the mask's
structure (CPU only). Source: "Mamba & State Space Models — Guide Complet"
§5 "Mamba-2" / "SSD — State Space Dual"."""
import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

from oracle import ssd_matrix


def _case(seed, batch=2, T=37, H=3, P=4, N=5, gate=True, h0=True):
    r = np.random.default_rng(seed)
    c = dict(
        x=r.standard_normal((batch, T, H * P)),
        dt=0.5 * r.standard_normal((batch, T, H)),
        A=-(r.random(H) * 3.5 + 0.5),
        B=r.standard_normal((batch, T, N)),
        C=r.standard_normal((batch, T, N)),
        D=1.0 + 0.1 * r.standard_normal(H),
        z=r.standard_normal((batch, T, H * P)) if gate else None,
        dt_bias=np.log(np.expm1(1e-3 + (1e-1 - 1e-3) * r.random(H))),
        h0=0.3 * r.standard_normal((batch, H * P, N)) if h0 else None,
    )
    return c


def _scan(orc, c, P, softplus=True):
    """The recurrence oracle with the heads' parameters repeated over their
    channels."""
    N = c["B"].shape[2]
    rep = lambda v: None if v is None else np.repeat(v, P, axis=-1)  # noqa: E731
    A_full = np.repeat(c["A"][:, None], P, axis=0).repeat(N, axis=1)
    return orc.fwd(c["x"], rep(c["dt"]), A_full, c["B"], c["C"], rep(c["D"]), c["z"],
                   rep(c["dt_bias"]), softplus=softplus, h0=c["h0"])


def _close(a, b, tol=1e-11):
    scale = max(float(np.max(np.abs(b))), 1e-300)
    assert float(np.max(np.abs(a - b))) <= tol * scale, float(np.max(np.abs(a - b))) / scale


@pytest.mark.parametrize("gate,h0,softplus", [(True, True, True), (False, False, True),
                                              (True, False, False)])
def test_matrix_form_equals_recurrence(orc, gate, h0, softplus):
    c = _case(9100 + 2 * gate + h0, gate=gate, h0=h0)
    if not softplus:  # positive Δ without the softplus
        c["dt"] = np.abs(c["dt"]) * 0.2 + 0.01
        c["dt_bias"] = np.zeros_like(c["dt_bias"])
    y, hf = ssd_matrix.ssd_matrix_form(c["x"], c["dt"], c["A"], c["B"], c["C"], c["D"], c["z"],
                                       c["dt_bias"], softplus=softplus, h0=c["h0"])
    yo, ho = _scan(orc, c, 4, softplus=softplus)
    _close(y, yo)
    _close(hf, ho)


def test_single_token_closed_form():
    """T = 1: y = ((C·B)·Δ + D)·x + exp(Δ·A)·C·h0, gated; final = exp(Δ·A)·h0 + Δ·B ⊗ x."""
    c = _case(9200, batch=1, T=1, H=2, P=3, N=4)
    y, hf = ssd_matrix.ssd_matrix_form(c["x"], c["dt"], c["A"], c["B"], c["C"], c["D"], c["z"],
                                       c["dt_bias"], h0=c["h0"])
    for h in range(2):
        delta = np.logaddexp(0.0, c["dt"][0, 0, h] + c["dt_bias"][h])
        a = np.exp(delta * c["A"][h])
        cb = float(c["C"][0, 0] @ c["B"][0, 0])
        for p in range(3):
            d = h * 3 + p
            xv, zv = c["x"][0, 0, d], c["z"][0, 0, d]
            h0v = c["h0"][0, d]
            want = (cb * delta * xv + c["D"][h] * xv + a * float(c["C"][0, 0] @ h0v))
            want *= zv / (1.0 + np.exp(-zv))
            assert abs(y[0, 0, d] - want) <= 1e-13 * max(1.0, abs(want))
            np.testing.assert_allclose(hf[0, d], a * h0v + delta * c["B"][0, 0] * xv,
                                       rtol=1e-13, atol=1e-15)


def test_mask_is_semiseparable():
    """Every block of the mask strictly below the diagonal has rank 1:
    L[i, j] = exp(Acum_i)·exp(−Acum_j) (the structure [Guide] §5 names)."""
    r = np.random.default_rng(9300)
    L = ssd_matrix.decay_mask(0.5 * r.standard_normal(40), -1.3, dt_bias=-2.0)
    for i0 in range(1, 40, 7):
        for j0 in range(0, i0, 5):
            block = L[i0:, :j0 + 1]
            s = np.linalg.svd(block, compute_uv=False)
            assert s[1] <= 1e-12 * s[0] if s.size > 1 else True


def _slipped_matrix_form(c, slip):
    """The matrix form with one plausible slip planted (test-local copy):
    'shifted_mask' takes the decay from Acum_{j-1}; 'S_transposed' forms
    B·Cᵀ instead of C·Bᵀ; 'delta_on_rows' scales the rows of L ◦ S by Δ
    instead of its columns; 'state_without_delta' drops Δ_j from the final
    state's sum."""
    x, dt, A, B, C = c["x"], c["dt"], c["A"], c["B"], c["C"]
    batch, T, dim = x.shape
    H = dt.shape[2]
    P = dim // H
    y = np.zeros_like(x)
    final = np.zeros((batch, dim, B.shape[2]))
    for b in range(batch):
        S = (B[b] @ C[b].T) if slip == "S_transposed" else (C[b] @ B[b].T)
        for h in range(H):
            delta = np.logaddexp(0.0, dt[b, :, h] + c["dt_bias"][h])
            acum = np.cumsum(delta * A[h])
            prev = np.concatenate([[0.0], acum[:-1]]) if slip == "shifted_mask" else acum
            L = np.tril(np.exp(acum[:, None] - prev[None, :]))
            M = L * S
            M = M * (delta[:, None] if slip == "delta_on_rows" else delta[None, :])
            xh = x[b, :, h * P:(h + 1) * P]
            h0h = c["h0"][b, h * P:(h + 1) * P, :].T
            yh = M @ xh + c["D"][h] * xh + np.exp(acum)[:, None] * (C[b] @ h0h)
            zh = c["z"][b, :, h * P:(h + 1) * P]
            y[b, :, h * P:(h + 1) * P] = yh * zh / (1.0 + np.exp(-zh))
            w = np.exp(acum[-1] - acum) * (1.0 if slip == "state_without_delta" else delta)
            final[b, h * P:(h + 1) * P, :] = ((w[:, None] * B[b]).T @ xh
                                              + np.exp(acum[-1]) * h0h).T
    return y, final


@pytest.mark.parametrize("slip", ["shifted_mask", "S_transposed", "delta_on_rows",
                                  "state_without_delta"])
def test_a_planted_slip_is_caught(orc, slip):
    """Each plausible slip in the matrix form misses the recurrence oracle by
    far more than the pin's tolerance, in y or in the final state."""
    c = _case(9400)
    yo, ho = _scan(orc, c, 4)
    y, hf = _slipped_matrix_form(c, slip)
    err = max(float(np.max(np.abs(y - yo))) / float(np.max(np.abs(yo))),
              float(np.max(np.abs(hf - ho))) / float(np.max(np.abs(ho))))
    assert err > 1e-3, (slip, err)


def test_the_slip_free_copy_matches(orc):
    """The test-local copy without a slip equals the recurrence: the slips
    above are the only difference."""
    c = _case(9400)
    yo, ho = _scan(orc, c, 4)
    y, hf = _slipped_matrix_form(c, None)
    _close(y, yo)
    _close(hf, ho)


@settings(max_examples=40, deadline=None)
@given(batch=st.integers(1, 2), T=st.integers(1, 24), H=st.integers(1, 3), P=st.integers(1, 4),
       N=st.integers(1, 6), seed=st.integers(0, 10_000), gate=st.booleans(), h0=st.booleans(),
       softplus=st.booleans())
def test_matrix_form_equals_recurrence_any_shape(orc, batch, T, H, P, N, seed, gate, h0, softplus):
    """The dense semiseparable form and the recurrence agree to float64
    rounding on every small shape, with or without gate, initial state and
    softplus."""
    c = _case(seed, batch=batch, T=T, H=H, P=P, N=N, gate=gate, h0=h0)
    if not softplus:
        c["dt"] = np.abs(c["dt"]) * 0.2 + 0.01
        c["dt_bias"] = np.zeros_like(c["dt_bias"])
    y, hf = ssd_matrix.ssd_matrix_form(c["x"], c["dt"], c["A"], c["B"], c["C"], c["D"], c["z"],
                                       c["dt_bias"], softplus=softplus, h0=c["h0"])
    yo, ho = _scan(orc, c, P, softplus=softplus)
    _close(y, yo)
    _close(hf, ho)


# --------------------------------------------------------------------------- #
# The oracle's scalar-A-per-head entry points against the matrix form, which
# shares no code with the C recurrence they are built on.

_SSD_GRADS = {"x": "dx", "dt": "ddt", "A": "dA", "B": "dB", "C": "dC", "D": "dD",
              "z": "dz", "dt_bias": "ddt_bias", "h0": "dh0"}


def _matrix(c, softplus=True):
    return ssd_matrix.ssd_matrix_form(c["x"], c["dt"], c["A"], c["B"], c["C"], c["D"], c["z"],
                                      c["dt_bias"], softplus=softplus, h0=c["h0"])


def _positive_dt(c):
    c["dt"] = np.abs(c["dt"]) * 0.2 + 0.01
    c["dt_bias"] = np.full_like(c["dt_bias"], 0.01)
    return c


@pytest.mark.parametrize("gate,h0,softplus", [(True, True, True), (False, False, False)])
def test_ssd_fwd_method_equals_matrix_form(orc, gate, h0, softplus):
    c = _case(9500 + gate, gate=gate, h0=h0)
    if not softplus:
        _positive_dt(c)
    y, hf = orc.ssd_fwd(c["x"], c["dt"], c["A"], c["B"], c["C"], c["D"], c["z"], c["dt_bias"],
                        softplus=softplus, h0=c["h0"], threads=1)
    ym, hm = _matrix(c, softplus)
    _close(y, ym)
    _close(hf, hm)


@pytest.mark.parametrize("gate,h0,softplus", [(True, True, True), (False, False, False)])
def test_ssd_gradient_finite_differences(orc, gate, h0, softplus):
    """Every element of every gradient of the head form against central
    differences of the matrix form's loss Σ dy·y + Σ dfinal·h_last."""
    c = _case(9600 + gate, batch=1, T=6, H=2, P=2, N=3, gate=gate, h0=h0)
    if not softplus:
        _positive_dt(c)
    r = np.random.default_rng(9601)
    dy = r.standard_normal(c["x"].shape)
    dfinal = r.standard_normal((1, 4, 3))
    g = orc.ssd_bwd(c["x"], c["dt"], c["A"], c["B"], c["C"], c["D"], c["z"], c["dt_bias"],
                    softplus=softplus, h0=c["h0"], dy=dy, dfinal=dfinal, threads=1)

    def loss(cc):
        y, hf = _matrix(cc, softplus)
        return float(np.sum(dy * y) + np.sum(dfinal * hf))

    for name, gname in _SSD_GRADS.items():
        if c[name] is None:
            assert g[gname] is None, gname
            continue
        arr = c[name]
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            e = 1e-6 * max(1.0, abs(arr[idx]))
            cp, cm = dict(c), dict(c)
            cp[name] = arr.copy()
            cp[name][idx] += e
            cm[name] = arr.copy()
            cm[name][idx] -= e
            fd[idx] = (loss(cp) - loss(cm)) / (2 * e)
        scale = max(float(np.max(np.abs(fd))), 1e-12)
        assert float(np.max(np.abs(g[gname] - fd))) <= 1e-6 * scale, gname


@settings(max_examples=40, deadline=None)
@given(batch=st.integers(1, 2), T=st.integers(1, 12), H=st.integers(1, 3), P=st.integers(1, 3),
       N=st.integers(1, 5), seed=st.integers(0, 10_000), gate=st.booleans(), h0=st.booleans(),
       softplus=st.booleans())
def test_ssd_gradient_directional_derivative_any_shape(orc, batch, T, H, P, N, seed, gate, h0,
                                                       softplus):
    """The head form's gradients dotted with a random direction through
    every input equal the central difference of the matrix form along it."""
    c = _case(seed, batch=batch, T=T, H=H, P=P, N=N, gate=gate, h0=h0)
    if not softplus:
        _positive_dt(c)
    r = np.random.default_rng(seed + 3)
    dy = r.standard_normal(c["x"].shape)
    dfinal = r.standard_normal((batch, H * P, N))
    names = [k for k in _SSD_GRADS if c[k] is not None]
    v = {k: r.standard_normal(np.shape(c[k])) for k in names}
    g = orc.ssd_bwd(c["x"], c["dt"], c["A"], c["B"], c["C"], c["D"], c["z"], c["dt_bias"],
                    softplus=softplus, h0=c["h0"], dy=dy, dfinal=dfinal, threads=1)

    def loss(eps):
        cc = dict(c)
        for k in names:
            cc[k] = c[k] + eps * v[k]
        y, hf = _matrix(cc, softplus)
        return float(np.sum(dy * y) + np.sum(dfinal * hf))

    terms = [g[_SSD_GRADS[k]] * v[k] for k in names]
    want = sum(float(np.sum(t)) for t in terms)
    scale = sum(float(np.sum(np.abs(t))) for t in terms)
    fd = (loss(1e-6) - loss(-1e-6)) / 2e-6
    assert abs(fd - want) <= 1e-6 * max(scale, 1e-12), (fd, want, scale)
