"""ctypes loader for the float64 selective-scan oracle in ``selscan_oracle.c``.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers. The CUDA library never imports this
module and this module never imports the CUDA library.

All array arguments are numpy arrays of any real dtype; they are widened to
float64 (exact for fp32 and bf16 values) before the call. Layouts follow the
pages' statement of the selective SSM ("Mamba & State Space Models — Guide
Complet", §4 "Implémentation du SSM sélectif (S6)"): x, delta, z, y
[batch, L, D]; B, C [batch, L, N]; A [D, N]; D, delta_bias [D]; states
[batch, D, N].
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "selscan_oracle.c")
LIBRARY = os.path.join(_HERE, "_build", "libselscan_oracle.so")

BBAR_DELTA = 0  # B_bar = Δ·B (the hot path's input term)
BBAR_ZOH = 1  # B_bar = (exp(Δ·A) − 1)/A·B (diagonal zero-order hold)

_dp = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64


def build(source: str = SOURCE, out: str = LIBRARY) -> str:
    """Compile the oracle with gcc (IEEE float64, no fast-math)."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
           "-o", tmp, source, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    return a.ctypes.data_as(_dp)


def _f64(a, shape=None) -> Optional[np.ndarray]:
    if a is None:
        return None
    arr = np.ascontiguousarray(np.asarray(a, dtype=np.float64))
    if shape is not None and arr.shape != tuple(shape):
        raise ValueError(f"expected shape {tuple(shape)}, got {arr.shape}")
    return arr


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


class Oracle:
    """Handle on one compiled oracle library (the default one, or a variant
    compiled from edited source by the planted-mistake tests)."""

    def __init__(self, lib_path: Optional[str] = None):
        if lib_path is None:
            lib_path = LIBRARY
            if (not os.path.exists(lib_path)
                    or os.path.getmtime(lib_path) < os.path.getmtime(SOURCE)):
                build()
        self.path = lib_path
        lib = ctypes.CDLL(lib_path)
        lib.oracle_selscan_fwd.restype = None
        lib.oracle_selscan_fwd.argtypes = [
            _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int,
            _dp, _dp, _dp, _i64, _i64, _i64, _i64, ctypes.c_int]
        lib.oracle_selscan_fwd_chunked.restype = None
        lib.oracle_selscan_fwd_chunked.argtypes = [
            _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int,
            _dp, _dp, _dp, _i64, _i64, _i64, _i64, _i64, ctypes.c_int]
        lib.oracle_state_update.restype = None
        lib.oracle_state_update.argtypes = [
            _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, ctypes.c_int, _dp,
            _i64, _i64, _i64]
        lib.oracle_compose.restype = None
        lib.oracle_compose.argtypes = [ctypes.c_double] * 4 + [_dp, _dp]
        lib.oracle_selscan_bwd.restype = None
        lib.oracle_selscan_bwd.argtypes = (
            [_dp] * 8 + [ctypes.c_int, ctypes.c_int] + [_dp] * 3 + [_dp] * 9
            + [_i64, _i64, _i64, _i64, ctypes.c_int])
        lib.oracle_causal_conv1d.restype = None
        lib.oracle_causal_conv1d.argtypes = [_dp, _dp, _dp, _dp, _i64, _i64, _i64, _i64,
                                             ctypes.c_int]
        lib.oracle_causal_conv1d_bwd.restype = None
        lib.oracle_causal_conv1d_bwd.argtypes = [_dp] * 7 + [_i64, _i64, _i64, _i64,
                                                             ctypes.c_int]
        lib.oracle_zoh_discretize.restype = None
        lib.oracle_zoh_discretize.argtypes = [ctypes.c_double, _dp, _dp, _dp,
                                              _dp, _i64]
        self.lib = lib

    # -- whole-sequence scan -------------------------------------------------
    def _fwd_args(self, x, delta, A, B, C, D, z, delta_bias, h0):
        x = _f64(x)
        if x.ndim != 3:
            raise ValueError("x must be [batch, L, D]")
        batch, L, dim = x.shape
        A = _f64(A)
        if A.ndim != 2 or A.shape[0] != dim:
            raise ValueError("A must be [D, N]")
        N = A.shape[1]
        args = dict(
            x=x,
            delta=_f64(delta, x.shape),
            A=A,
            B=_f64(B, (batch, L, N)),
            C=_f64(C, (batch, L, N)),
            D=_f64(D, (dim,)),
            z=_f64(z, x.shape),
            delta_bias=_f64(delta_bias, (dim,)),
            h0=_f64(h0, (batch, dim, N)),
        )
        return args, (batch, L, dim, N)

    def fwd(self, x, delta, A, B, C, D=None, z=None, delta_bias=None,
            softplus=True, bbar=BBAR_DELTA, h0=None, threads=None):
        """Return (y, final_state) as float64 arrays."""
        a, (batch, L, dim, N) = self._fwd_args(x, delta, A, B, C, D, z,
                                               delta_bias, h0)
        y = np.empty((batch, L, dim), dtype=np.float64)
        hs = np.empty((batch, dim, N), dtype=np.float64)
        self.lib.oracle_selscan_fwd(
            _ptr(a["x"]), _ptr(a["delta"]), _ptr(a["A"]), _ptr(a["B"]),
            _ptr(a["C"]), _ptr(a["D"]), _ptr(a["z"]), _ptr(a["delta_bias"]),
            int(bool(softplus)), int(bbar), _ptr(a["h0"]), _ptr(y), _ptr(hs),
            batch, L, dim, N, int(threads or default_threads()))
        return y, hs

    def fwd_chunked(self, x, delta, A, B, C, D=None, z=None, delta_bias=None,
                    softplus=True, bbar=BBAR_DELTA, h0=None, chunk=256,
                    threads=None):
        """Chunk-aggregate / carry / rescan form; returns (y, final_state)."""
        a, (batch, L, dim, N) = self._fwd_args(x, delta, A, B, C, D, z,
                                               delta_bias, h0)
        y = np.empty((batch, L, dim), dtype=np.float64)
        hs = np.empty((batch, dim, N), dtype=np.float64)
        self.lib.oracle_selscan_fwd_chunked(
            _ptr(a["x"]), _ptr(a["delta"]), _ptr(a["A"]), _ptr(a["B"]),
            _ptr(a["C"]), _ptr(a["D"]), _ptr(a["z"]), _ptr(a["delta_bias"]),
            int(bool(softplus)), int(bbar), _ptr(a["h0"]), _ptr(y), _ptr(hs),
            batch, L, dim, N, int(chunk), int(threads or default_threads()))
        return y, hs

    def bwd(self, x, delta, A, B, C, D=None, z=None, delta_bias=None,
            softplus=True, h0=None, dy=None, dfinal=None, threads=None, bbar=BBAR_DELTA):
        """Gradient of the loss Σ dy·y + Σ dfinal·final_state with respect to
        every input of ``fwd`` (input term Δ·B·x, or the ZOH term with
        ``bbar=BBAR_ZOH``). Returns a dict with dx,
        ddelta, dA, dB, dC, dD, dz (None without z), ddelta_bias and dh0
        (None without h0), all float64."""
        a, (batch, L, dim, N) = self._fwd_args(x, delta, A, B, C, D, z,
                                               delta_bias, h0)
        dy = _f64(dy, (batch, L, dim))
        dfinal = _f64(dfinal, (batch, dim, N))
        out = dict(
            dx=np.empty((batch, L, dim)), ddelta=np.empty((batch, L, dim)),
            dA=np.empty((dim, N)), dB=np.empty((batch, L, N)),
            dC=np.empty((batch, L, N)), dD=np.empty((dim,)),
            dz=np.empty((batch, L, dim)) if a["z"] is not None else None,
            ddelta_bias=np.empty((dim,)),
            dh0=np.empty((batch, dim, N)) if a["h0"] is not None else None)
        self.lib.oracle_selscan_bwd(
            _ptr(a["x"]), _ptr(a["delta"]), _ptr(a["A"]), _ptr(a["B"]),
            _ptr(a["C"]), _ptr(a["D"]), _ptr(a["z"]), _ptr(a["delta_bias"]),
            int(bool(softplus)), int(bbar), _ptr(a["h0"]), _ptr(dy), _ptr(dfinal),
            _ptr(out["dx"]), _ptr(out["ddelta"]), _ptr(out["dA"]), _ptr(out["dB"]),
            _ptr(out["dC"]), _ptr(out["dD"]), _ptr(out["dz"]),
            _ptr(out["ddelta_bias"]), _ptr(out["dh0"]),
            batch, L, dim, N, int(threads or default_threads()))
        return out

    # -- one scalar A per head ("Mamba & State Space Models — Guide Complet" §5
    #    "Mamba-2": the state matrix is a scalar times the identity per head) --
    @staticmethod
    def _heads(x, dt, A, B):
        x = _f64(x)
        dt = _f64(dt)
        if x.ndim != 3 or dt.ndim != 3 or dt.shape[:2] != x.shape[:2]:
            raise ValueError("x must be [batch, L, H·P] and dt [batch, L, H]")
        H = dt.shape[2]
        if H < 1 or x.shape[2] % H:
            raise ValueError("the channel count must be a multiple of the head count")
        N = np.asarray(B).shape[2]
        return x, dt, H, x.shape[2] // H, N

    def ssd_fwd(self, x, dt, A, B, C, D=None, z=None, dt_bias=None, softplus=True,
                h0=None, threads=None):
        """The scan with one scalar A per head: channel d = h·P + p of head h
        takes Δ from dt[..., h] + dt_bias[h], decay exp(Δ·A[h]) on every
        state, and skip D[h]; B and C are shared by all heads. x, z
        [batch, L, H·P]; dt [batch, L, H]; A, D, dt_bias [H]; B, C
        [batch, L, N]; h0 [batch, H·P, N]. It is the selective scan with each
        head's parameters repeated over its P channels (and A over the N
        states). Returns (y, final_state)."""
        x, dt, H, P, N = self._heads(x, dt, A, B)
        rep = (lambda v: None if v is None else np.repeat(_f64(v), P, axis=-1))  # noqa: E731
        A_ch = np.repeat(_f64(A, (H,))[:, None], P, axis=0) * np.ones((1, N))
        return self.fwd(x, rep(dt), A_ch, B, C, rep(D), z, rep(dt_bias), softplus=softplus,
                        h0=h0, threads=threads)

    def ssd_bwd(self, x, dt, A, B, C, D=None, z=None, dt_bias=None, softplus=True,
                h0=None, dy=None, dfinal=None, threads=None):
        """Gradient of Σ dy·y + Σ dfinal·final_state for ``ssd_fwd``. A head's
        Δ, A, D and Δ-bias reach the loss through each of its channels (and
        A through each state), so their gradients are the per-channel
        gradients of the selective scan summed over those channels and
        states; x, z, B, C and h0 enter unchanged. Returns dx, ddt, dA, dB,
        dC, dD, dz (None without z), ddt_bias and dh0 (None without h0)."""
        x, dt, H, P, N = self._heads(x, dt, A, B)
        rep = (lambda v: None if v is None else np.repeat(_f64(v), P, axis=-1))  # noqa: E731
        A_ch = np.repeat(_f64(A, (H,))[:, None], P, axis=0) * np.ones((1, N))
        g = self.bwd(x, rep(dt), A_ch, B, C, rep(D), z, rep(dt_bias), softplus=softplus,
                     h0=h0, dy=dy, dfinal=dfinal, threads=threads)

        def per_head(v):  # [..., H·P] -> [..., H], summed over each head's channels
            return v.reshape(*v.shape[:-1], H, P).sum(axis=-1)

        return dict(dx=g["dx"], ddt=per_head(g["ddelta"]),
                    dA=g["dA"].reshape(H, P, N).sum(axis=(1, 2)), dB=g["dB"], dC=g["dC"],
                    dD=per_head(g["dD"]), dz=g["dz"], ddt_bias=per_head(g["ddelta_bias"]),
                    dh0=g["dh0"])

    def causal_conv1d(self, x_in, w, cb=None, silu=True):
        """Causal depthwise convolution (+ SiLU) in front of the scan:
        x_in [batch, L, D], w [D, K], cb [D] or None -> [batch, L, D]."""
        x_in = _f64(x_in)
        batch, L, dim = x_in.shape
        w = _f64(w)
        if w.ndim != 2 or w.shape[0] != dim:
            raise ValueError("w must be [D, K]")
        cb = _f64(cb, (dim,))
        out = np.empty_like(x_in)
        self.lib.oracle_causal_conv1d(_ptr(x_in), _ptr(w), _ptr(cb), _ptr(out), batch, L,
                                      dim, w.shape[1], int(bool(silu)))
        return out

    def causal_conv1d_bwd(self, x_in, w, cb, dxc, silu=True):
        """Gradient of ``causal_conv1d`` for the loss Σ dxc·x: returns
        (dx_in, dw, dcb) as float64 arrays (dcb None without a bias)."""
        x_in = _f64(x_in)
        batch, L, dim = x_in.shape
        w = _f64(w)
        K = w.shape[1]
        cb = _f64(cb, (dim,))
        dxc = _f64(dxc, x_in.shape)
        dx = np.empty_like(x_in)
        dw = np.empty_like(w)
        dcb = np.empty(dim) if cb is not None else None
        self.lib.oracle_causal_conv1d_bwd(_ptr(x_in), _ptr(w), _ptr(cb), _ptr(dxc), _ptr(dx),
                                          _ptr(dw), _ptr(dcb), batch, L, dim, K,
                                          int(bool(silu)))
        return dx, dw, dcb

    # -- single-token decode -------------------------------------------------
    def state_update(self, state, x, delta, A, B, C, D=None, z=None,
                     delta_bias=None, softplus=True):
        """One recurrent step. Returns (y [batch, D], new_state); the input
        state array is not modified."""
        st = np.array(state, dtype=np.float64, copy=True, order="C")
        if st.ndim != 3:
            raise ValueError("state must be [batch, D, N]")
        batch, dim, N = st.shape
        x = _f64(x, (batch, dim))
        y = np.empty((batch, dim), dtype=np.float64)
        self.lib.oracle_state_update(
            _ptr(st), _ptr(x), _ptr(_f64(delta, (batch, dim))),
            _ptr(_f64(A, (dim, N))), _ptr(_f64(B, (batch, N))),
            _ptr(_f64(C, (batch, N))), _ptr(_f64(D, (dim,))),
            _ptr(_f64(z, (batch, dim))), _ptr(_f64(delta_bias, (dim,))),
            int(bool(softplus)), _ptr(y), batch, dim, N)
        return y, st

    # -- pieces exposed for the pins -----------------------------------------
    def compose(self, a_later, b_later, a_earlier, b_earlier):
        ao = ctypes.c_double()
        bo = ctypes.c_double()
        self.lib.oracle_compose(float(a_later), float(b_later),
                                float(a_earlier), float(b_earlier),
                                ctypes.byref(ao), ctypes.byref(bo))
        return ao.value, bo.value

    def zoh_discretize(self, dt, A, B):
        A = _f64(A)
        B = _f64(B, A.shape)
        Ab = np.empty_like(A)
        Bb = np.empty_like(A)
        self.lib.oracle_zoh_discretize(float(dt), _ptr(A), _ptr(B), _ptr(Ab),
                                       _ptr(Bb), A.shape[0])
        return Ab, Bb


_DEFAULT: Optional[Oracle] = None


def default() -> Oracle:
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle()
    return _DEFAULT
