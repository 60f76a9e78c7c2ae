"""Shared pieces of the GPU parity tests: run the CUDA path through the
binding, run the float64 oracle on the same values, compare."""
import math
import os
from contextlib import contextmanager

import numpy as np
import torch

import oracle
import selective_state_space_42_b200 as ss

# Tolerances (written in the tests' terms): |gpu − oracle| ≤ rtol·(|oracle| +
# rms(oracle)) elementwise; rtol 1e-4 for float32 I/O, 2e-2 for bfloat16 I/O
# with float32 state.
RTOL = {"f32": 1e-4, "bf16": 2e-2}


def dtype_name(t):
    return "f32" if t.dtype == torch.float32 else "bf16"


def to_np(t):
    return None if t is None else t.detach().to("cpu", torch.float64).numpy()


def compare(got, ref, rtol, what=""):
    """Assert the elementwise bound; return (max |err| / (|o| + rms), max rel
    over |o| > rms, max|err| / max|o|) for reporting."""
    g = np.asarray(got, dtype=np.float64)
    o = np.asarray(ref, dtype=np.float64)
    assert g.shape == o.shape, (what, g.shape, o.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU output"
    if o.size == 0:
        return 0.0, 0.0, 0.0
    rms = math.sqrt(float(np.mean(o * o)))
    err = np.abs(g - o)
    bound = rtol * (np.abs(o) + rms) + 1e-30
    worst = float(np.max(err / bound)) * rtol
    big = np.abs(o) > rms
    rel_big = float(np.max(err[big] / np.abs(o[big]))) if big.any() else 0.0
    nrm = float(np.max(err)) / max(float(np.max(np.abs(o))), 1e-300)
    if worst > rtol:
        idx = np.unravel_index(int(np.argmax(err / bound)), err.shape)
        raise AssertionError(
            f"{what}: |gpu-oracle| exceeds {rtol}·(|o|+rms) at {idx}: gpu={g[idx]!r} "
            f"oracle={o[idx]!r} rms={rms:.3e} (worst ratio {worst:.3e})")
    return worst, rel_big, nrm


def gpu_fwd(inp, softplus=True, want_state=True):
    y, hs = ss.selscan_fwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"],
                           inp.get("D"), inp.get("z"), inp.get("delta_bias"),
                           softplus=softplus, return_final_state=True)
    return y, hs


def oracle_fwd(inp, channels=None, softplus=True, batches=None):
    """Oracle on all channels, or on a channel subset (channels are
    independent, B and C are shared)."""
    sel_c = slice(None) if channels is None else list(channels)
    sel_b = slice(None) if batches is None else list(batches)

    def bl(t):
        if t is None:
            return None
        t = t[sel_b]
        return t[:, :, sel_c] if channels is not None else t

    def ch(t):
        if t is None:
            return None
        return t[sel_c]

    x = bl(inp["x"])
    args = [to_np(x), to_np(bl(inp["delta"])), to_np(ch(inp["A"])),
            to_np(inp["B"][sel_b]), to_np(inp["C"][sel_b]), to_np(ch(inp.get("D"))),
            to_np(bl(inp.get("z"))), to_np(ch(inp.get("delta_bias")))]
    return oracle.default().fwd(*args, softplus=softplus)


@contextmanager
def forced_chunks(n):
    old = os.environ.get("SELSCAN_CHUNKS")
    os.environ["SELSCAN_CHUNKS"] = str(n)
    try:
        yield
    finally:
        if old is None:
            del os.environ["SELSCAN_CHUNKS"]
        else:
            os.environ["SELSCAN_CHUNKS"] = old


@contextmanager
def env(**kw):
    """Temporarily set (value) or unset (None) environment variables read by
    the library's planner (SELSCAN_PATH, SELSCAN_UNIT, SELSCAN_CHUNKS)."""
    old = {k: os.environ.get(k) for k in kw}
    try:
        for k, v in kw.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = str(v)
        yield
    finally:
        for k, v in old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
