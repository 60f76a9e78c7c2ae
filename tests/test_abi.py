"""The C ABI without a GPU: the library loads, exports every function that
include/*.h declares, and its host-side validation returns the documented
status codes before any CUDA call (CPU only; no kernel is launched)."""
import ctypes
import glob
import os
import re
import shutil
import subprocess

import pytest
from hypothesis import given, settings, strategies as st

import selective_state_space_42_b200 as ss
from selective_state_space_42_b200 import build as ssbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    ssbuild.build()
    return ss.load_library()


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        names |= set(re.findall(r"\b(selscan_\w+)\s*\(", text))
    return sorted(names)


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("selscan_fwd", "selscan_state_update", "selscan_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
        assert n in ss.selscan.SIGNATURES, f"{n} has no binding signature"


def test_only_declared_symbols_are_exported(lib):
    out = os.popen(f"nm -D --defined-only {ss.LIB_PATH}").read()
    exported = set(re.findall(r"\b(selscan_\w+)\b", out))
    assert exported == set(declared_functions())


def test_status_strings(lib):
    for code in [0, -1, -2, -3, -4, -5, -6, -7]:
        s = ss.selscan_status_string(code)
        assert s and s != "unknown status"
    assert ss.selscan_status_string(12345) == "unknown status"


P = 1 << 20  # a fake, aligned, non-null device address (never dereferenced)


def fwd(lib, **kw):
    a = dict(x=P, delta=P + 4096, A=P + 8192, B=P + 12288, C=P + 16384, D=None,
             z=None, delta_bias=None, softplus=1, y=P + 65536, final_state=None,
             batch=0, seqlen=8, dim=4, dstate=16, dtype=1, stream=None)
    a.update(kw)
    return lib.selscan_fwd(a["x"], a["delta"], a["A"], a["B"], a["C"], a["D"], a["z"],
                           a["delta_bias"], a["softplus"], a["y"], a["final_state"],
                           a["batch"], a["seqlen"], a["dim"], a["dstate"], a["dtype"],
                           a["stream"])


def step(lib, **kw):
    a = dict(state=P + 131072, x=P, delta=P + 4096, A=P + 8192, B=P + 12288,
             C=P + 16384, D=None, z=None, delta_bias=None, softplus=1, y=P + 65536,
             batch=0, dim=4, dstate=16, dtype=1, stream=None)
    a.update(kw)
    return lib.selscan_state_update(a["state"], a["x"], a["delta"], a["A"], a["B"],
                                    a["C"], a["D"], a["z"], a["delta_bias"],
                                    a["softplus"], a["y"], a["batch"], a["dim"],
                                    a["dstate"], a["dtype"], a["stream"])


def test_fwd_validation(lib):
    assert fwd(lib) == 0  # batch = 0: nothing to do, no CUDA call
    assert fwd(lib, batch=2, dim=0) == 0
    assert fwd(lib, batch=2, seqlen=0) == 0  # no final_state to clear
    assert fwd(lib, x=None) == 0  # empty tensors may be NULL
    assert fwd(lib, batch=1, x=None) == -1
    assert fwd(lib, batch=1, y=None) == -1
    assert fwd(lib, batch=1, B=None) == -1
    assert fwd(lib, batch=1, A=None) == -1
    assert fwd(lib, dtype=7) == -3
    assert fwd(lib, batch=-1) == -2
    assert fwd(lib, seqlen=-5) == -2
    assert fwd(lib, batch=1 << 30, seqlen=1 << 30, dim=1 << 30) == -2
    assert fwd(lib, dstate=0) == -5
    assert fwd(lib, dstate=257) == -5
    assert fwd(lib, dstate=17) == 0  # batch = 0: nothing to do
    assert fwd(lib, batch=70000, dstate=32) == -2  # wide kernel: batch rows are a grid dimension
    assert fwd(lib, x=P + 1) == -4  # bf16 needs 2-byte alignment
    assert fwd(lib, x=P + 2, dtype=0) == -4  # fp32 needs 4-byte alignment
    assert fwd(lib, A=P + 2) == -4
    assert fwd(lib, batch=1, y=P) == -7  # y == x
    assert fwd(lib, batch=1, y=P + 12288 - 2) == -7  # y runs into B


def test_fwd_from_state_validation(lib):
    def call(**kw):
        a = dict(x=P, delta=P + 4096, A=P + 8192, B=P + 12288, C=P + 16384, D=None,
                 z=None, delta_bias=None, softplus=1, h0=P + 32768, y=P + 65536,
                 final_state=P + 32768, batch=0, seqlen=8, dim=4, dstate=16, dtype=1,
                 stream=None)
        a.update(kw)
        return lib.selscan_fwd_from_state(
            a["x"], a["delta"], a["A"], a["B"], a["C"], a["D"], a["z"], a["delta_bias"],
            a["softplus"], a["h0"], a["y"], a["final_state"], a["batch"], a["seqlen"],
            a["dim"], a["dstate"], a["dtype"], a["stream"])
    assert call() == 0  # batch = 0; the state advanced in place is allowed
    assert call(h0=P + 32770) == -4
    assert call(batch=1, final_state=P + 32768 + 64) == -7  # partial overlap
    assert call(batch=1, y=P + 32768) == -7  # y overlaps the initial state


def test_state_update_validation(lib):
    assert step(lib) == 0
    assert step(lib, state=None) == 0  # batch = 0: empty
    assert step(lib, batch=1, state=None) == -1
    assert step(lib, dtype=-1) == -3
    assert step(lib, dim=-1) == -2
    assert step(lib, dstate=257) == -5
    assert step(lib, state=P + 2) == -4
    assert step(lib, batch=1, y=P + 131072) == -7  # y overlaps the state


def test_binding_rejects_cpu_tensors(lib):
    torch = pytest.importorskip("torch")
    x = torch.zeros(1, 4, 8)
    with pytest.raises(ValueError):
        ss.selscan_fwd(x, x, torch.zeros(8, 16), torch.zeros(1, 4, 16),
                       torch.zeros(1, 4, 16))


def bwd(lib, **kw):
    names = ["x", "delta", "A", "B", "C", "D", "z", "delta_bias", "dy", "dfinal",
             "dx", "ddelta", "dA", "dB", "dC", "dD", "dz", "ddelta_bias"]
    a = {n: P + 4096 * i for i, n in enumerate(names)}
    a.update(D=None, z=None, delta_bias=None, dfinal=None, dz=None, softplus=1,
             batch=0, seqlen=8, dim=0, dstate=16, dtype=1, stream=None)
    a.update(kw)
    return lib.selscan_bwd(a["x"], a["delta"], a["A"], a["B"], a["C"], a["D"], a["z"],
                           a["delta_bias"], a["softplus"], a["dy"], a["dfinal"], a["dx"],
                           a["ddelta"], a["dA"], a["dB"], a["dC"], a["dD"], a["dz"],
                           a["ddelta_bias"], a["batch"], a["seqlen"], a["dim"],
                           a["dstate"], a["dtype"], a["stream"])


def test_bwd_validation(lib):
    """Every check runs before any CUDA call (no GPU here)."""
    assert bwd(lib) == 0  # batch = 0 and dim = 0: no output has an element
    assert bwd(lib, dtype=7) == -3
    assert bwd(lib, batch=-1) == -2
    assert bwd(lib, batch=70000, dim=4) == -2  # batch rows are a grid dimension
    assert bwd(lib, dstate=0) == -5
    assert bwd(lib, dstate=257) == -5  # the gradient takes d_state <= 256
    full = dict(batch=1, dim=4)
    assert bwd(lib, x=None, **full) == -1
    assert bwd(lib, dy=None, **full) == -1
    assert bwd(lib, dx=None, **full) == -1
    assert bwd(lib, dB=None, **full) == -1
    assert bwd(lib, A=None, **full) == -1
    assert bwd(lib, dA=None, **full) == -1
    assert bwd(lib, z=P + 4096 * 40, dz=None, **full) == -1  # dz required with z
    assert bwd(lib, dx=P + 4096 * 10 + 1, **full) == -4
    assert bwd(lib, dA=P + 4096 * 12 + 2, **full) == -4
    assert bwd(lib, dx=P, **full) == -7  # dx == x
    assert bwd(lib, dB=P + 4096 * 3 + 64, **full) == -7  # dB runs into B
    assert bwd(lib, ddelta=P + 4096 * 10, **full) == -7  # two outputs overlap


def test_bwd_workspace_bytes(lib):
    assert lib.selscan_bwd_workspace_bytes(0, 8, 4, 16) == 0
    assert lib.selscan_bwd_workspace_bytes(1, 8, 4, 257) == 0
    # one 16-token tile, one 32-channel tile: checkpoints 4·16·4 B, partials
    # 8·32·4 B, per-channel partials 4·(16 + 2)·4 B, each rounded up to 256 B
    assert lib.selscan_bwd_workspace_bytes(1, 8, 4, 16) == 256 + 1024 + 256 + 256 + 256
    # 17 states: two 16-state groups side by side, so the checkpoints and the
    # dB/dC and dA partials double, and each group writes three float32
    # [1, 8, 4] per-token arrays for the finishing sum
    assert lib.selscan_bwd_workspace_bytes(1, 8, 4, 17) == 512 + 2048 + 512 + 256 + 256 + 768


def test_plans_of_the_workloads(lib):
    """The host planner (no GPU: the SM count falls back to 148) picks one
    pass for the Mamba-2.8B layer, the chunked plan for the 1M-token
    sequence and the wide kernel (one launch, no workspace) above d_state 16."""
    from selective_state_space_42_b200 import workloads as wl  # noqa: F401
    p = ss.selscan_fwd_plan(4, 8192, 5120, 16)
    assert p["launches"] == 1 and p["chunks"] == 8
    p = ss.selscan_fwd_plan(1, 1 << 20, 2048, 16)
    assert p["launches"] == 3 and p["chunks"] > 1 and p["workspace_bytes"] > 0
    p = ss.selscan_fwd_plan(2, 4096, 2048, 128)
    assert p == {"chunks": 1, "launches": 1, "workspace_bytes": 0}
    w = wl.WORKLOADS["mamba130m_layer"]
    p = ss.selscan_fwd_plan(w.batch, w.seqlen, w.dim, w.dstate)
    assert p["launches"] == 1 and p["chunks"] == 2  # 96 groups: enough for one pass
    p = ss.selscan_fwd_plan(1, 8192, 1536, 16)  # 12 groups: chunked
    assert p["launches"] == 3


def ssd(lib, **kw):
    names = ["x", "dt", "A", "B", "C", "D", "z", "dt_bias", "h0", "y", "final"]
    a = {n: P + 4096 * i for i, n in enumerate(names)}
    a.update(D=None, z=None, dt_bias=None, h0=None, final=None, softplus=1, batch=0,
             seqlen=8, nheads=2, headdim=4, dstate=16, dtype=1, ws=None, wsb=0, stream=None)
    a.update(kw)
    return lib.selscan_ssd_fwd(a["x"], a["dt"], a["A"], a["B"], a["C"], a["D"], a["z"],
                               a["dt_bias"], a["softplus"], a["h0"], a["y"], a["final"],
                               a["batch"], a["seqlen"], a["nheads"], a["headdim"],
                               a["dstate"], a["dtype"], a["ws"], a["wsb"], a["stream"])


def test_ssd_validation(lib):
    """Every check of selscan_ssd_fwd runs before any CUDA call (no GPU here)."""
    assert ssd(lib) == 0  # batch = 0: no output has an element
    assert ssd(lib, dtype=7) == -3
    assert ssd(lib, batch=-1) == -2
    assert ssd(lib, seqlen=-1) == -2
    assert ssd(lib, headdim=0) == -2
    assert ssd(lib, headdim=65) == -2  # one head's channels fit one 64-wide tile
    assert ssd(lib, nheads=70000) == -2  # heads are a grid dimension
    assert ssd(lib, dstate=0) == -5
    assert ssd(lib, dstate=129) == -5  # d_state fits one 128-wide tile
    full = dict(batch=1)
    for name in ("x", "dt", "A", "B", "C", "y"):
        assert ssd(lib, **{name: None}, **full) == -1, name
    assert ssd(lib, x=P + 1, **full) == -4  # bf16 element alignment
    assert ssd(lib, A=P + 4096 * 2 + 2, **full) == -4
    assert ssd(lib, ws=P + 4096 * 64 + 16, wsb=1 << 20, **full) == -4  # 256-byte workspace
    assert ssd(lib, y=P, **full) == -7  # y == x
    assert ssd(lib, final=P + 4096 * 3, **full) == -7  # the final state runs into B
    assert ssd(lib, ws=P + 4096 * 64, wsb=16, **full) == -8  # too small
    need = lib.selscan_ssd_workspace_bytes(1, 8, 2, 4, 16)
    assert ssd(lib, ws=P + 4096 * 3, wsb=need, **full) == -7  # workspace runs into B


def test_ssd_workspace_bytes(lib):
    assert lib.selscan_ssd_workspace_bytes(0, 8, 2, 4, 16) == 0
    assert lib.selscan_ssd_workspace_bytes(1, 8, 2, 65, 16) == 0
    assert lib.selscan_ssd_workspace_bytes(1, 8, 2, 4, 129) == 0
    # one 64-token chunk, 2 heads: partial output 8·8·4 B; chunk states and
    # carried states 2·128·64·4 B each; decays 2·4 B; each rounded up to 256 B
    assert lib.selscan_ssd_workspace_bytes(1, 8, 2, 4, 16) == 256 + 65536 + 256 + 65536
    # the tensor-core path (128-token chunks) fits in the float32 path's layout
    assert (lib.selscan_ssd_workspace_bytes(2, 1000, 4, 64, 128)
            >= 2 * 4 * 8 * 32768 * 2)


_BwdOpts = ss.selscan.BwdOptions  # selscan_bwd_options_t


def test_bwd_ex_validation(lib):
    """selscan_bwd_ex: the options are checked before anything runs; with
    batch = 0 and dim = 0 nothing has an element (status 0)."""
    names = ["x", "delta", "A", "B", "C", "D", "z", "delta_bias", "dy", "dfinal",
             "dx", "ddelta", "dA", "dB", "dC", "dD", "dz", "ddelta_bias"]
    a = {n: P + 4096 * i for i, n in enumerate(names)}
    a.update(D=None, z=None, delta_bias=None, dfinal=None, dz=None)

    def call(opts, **kw):
        b = dict(a, batch=0, dim=0, dstate=16)
        b.update(kw)
        return ss.selscan.load_library().selscan_bwd_ex(
            b["x"], b["delta"], b["A"], b["B"], b["C"], b["D"], b["z"], b["delta_bias"], 1,
            b["dy"], b["dfinal"], ctypes.byref(opts) if opts is not None else None, b["dx"],
            b["ddelta"], b["dA"], b["dB"], b["dC"], b["dD"], b["dz"], b["ddelta_bias"],
            b["batch"], 8, b["dim"], b["dstate"], 1, None, 0, None)

    assert call(None) == 0
    assert call(_BwdOpts(bbar_mode=1)) == 0
    assert call(_BwdOpts(bbar_mode=2)) == -2
    assert call(_BwdOpts(conv_width=-1)) == -2
    assert call(_BwdOpts(conv_width=5)) == -2
    assert call(_BwdOpts(bbar_mode=1), dstate=257) == -5  # the gradient takes d_state <= 256
    assert call(_BwdOpts(bbar_mode=1), batch=1, dim=4, x=None) == -1


def test_binding_constants_match_the_header():
    """The binding's copies of the header's limits and status codes."""
    text = open(os.path.join(ROOT, "include", "selscan.h")).read()
    defines = dict(re.findall(r"#define\s+(SELSCAN_\w+)\s+(\d+)", text))
    for name in ("SELSCAN_MAX_DSTATE", "SELSCAN_MAX_DSTATE_BWD"):
        assert int(defines[name]) == getattr(ss.selscan, name), name
    codes = dict((n, int(v)) for n, v in re.findall(r"(SELSCAN_(?:OK|ERR_\w+))\s*=\s*(-?\d+)", text))
    for code, name in ss.selscan.STATUS.items():
        assert codes[name] == code, name


def _ptrs(names, spacing=4096):
    return {n: P + spacing * i for i, n in enumerate(names)}


def test_fwd_conv_validation(lib):
    """selscan_fwd_conv: conv width 1..4, the weight required, alignment, and
    y kept clear of the conv's carried inputs."""
    def call(**kw):
        a = _ptrs(["x_in", "cw", "cb", "ci", "delta", "A", "B", "C", "h0", "y", "final"])
        a.update(cb=None, ci=None, h0=None, final=None, width=4, batch=0, dim=4)
        a.update(kw)
        return lib.selscan_fwd_conv(a["x_in"], a["cw"], a["cb"], a["width"], a["ci"],
                                    a["delta"], a["A"], a["B"], a["C"], None, None, None, 1,
                                    a["h0"], a["y"], a["final"], a["batch"], 8, a["dim"], 16,
                                    1, None)
    assert call() == 0  # batch = 0
    assert call(width=0) == -2
    assert call(width=5) == -2
    assert call(width=-1) == -2
    assert call(batch=1, cw=None) == -1
    assert call(cw=P + 4096 + 2) == -4
    assert call(ci=P + 4096 * 3 + 2) == -4
    assert call(batch=1, ci=P + 4096 * 9 + 32) == -7  # y runs into conv_init


def test_fwd_ex_validation(lib):
    Opts = ss.selscan.FwdOptions

    def call(opts, **kw):
        a = _ptrs(["x", "delta", "A", "B", "C", "y", "h0", "cw", "ci"])
        a.update(batch=0, dim=4, dstate=16)
        a.update(kw)
        return lib.selscan_fwd_ex(a["x"], a["delta"], a["A"], a["B"], a["C"], None, None,
                                  None, 1, ctypes.byref(opts) if opts is not None else None,
                                  a["y"], None, a["batch"], 8, a["dim"], a["dstate"], 1, None)
    assert call(None) == 0
    assert call(Opts(bbar_mode=1)) == 0
    assert call(Opts(bbar_mode=2)) == -2
    assert call(Opts(bbar_mode=-1)) == -2
    assert call(Opts(conv_width=5)) == -2
    assert call(Opts(conv_width=4), batch=1) == -1  # no conv weight
    assert call(Opts(initial_state=P + 4096 * 6 + 2)) == -4
    assert call(Opts(conv_width=4, conv_weight=P + 4096 * 7, conv_init=P + 4096 * 5),
                batch=1) == -7  # y == conv_init
    assert call(Opts(bbar_mode=1), dstate=257) == -5


def test_fwd_noalloc_validation(lib):
    """The same checks as selscan_fwd, and sizes whose chunked plan needs more
    than the fixed array are refused before anything runs."""
    def call(spacing=4096, **kw):
        a = _ptrs(["x", "delta", "A", "B", "C", "y"], spacing)
        a.update(batch=0, seqlen=8, dim=4, dstate=16, dtype=1)
        a.update(kw)
        return lib.selscan_fwd_noalloc(a["x"], a["delta"], a["A"], a["B"], a["C"], None,
                                       None, None, 1, a["y"], None, a["batch"], a["seqlen"],
                                       a["dim"], a["dstate"], a["dtype"], None)
    assert call() == 0
    assert call(dtype=7) == -3
    assert call(batch=-1) == -2
    assert call(dstate=0) == -5
    assert call(batch=1, x=None) == -1
    assert call(x=P + 1) == -4
    assert call(batch=1, y=P) == -7
    need = ss.selscan_fwd_plan(1, 1 << 20, 2048, 16)["workspace_bytes"]
    assert need > ss.SELSCAN_NOALLOC_WORKSPACE_BYTES
    # 4 GiB tensors: the fake addresses sit 8 GiB apart so that none overlap
    assert call(spacing=8 << 30, batch=1, seqlen=1 << 20, dim=2048) == -8


def _bwd_names():
    return ["x", "delta", "A", "B", "C", "D", "z", "delta_bias", "dy", "dfinal", "dx",
            "ddelta", "dA", "dB", "dC", "dD", "dz", "ddelta_bias", "h0", "dh0", "cw", "cb",
            "dcw", "dcb", "ws"]


def _bwd_ptrs(**kw):
    a = _ptrs(_bwd_names())
    a.update(D=None, z=None, delta_bias=None, dfinal=None, dz=None, h0=None, dh0=None,
             cb=None, dcb=None, batch=0, dim=0, dstate=16, wsb=0)
    a.update(kw)
    return a


def test_bwd_workspace_validation(lib):
    """selscan_bwd_workspace takes the caller's buffer: required when a token
    is processed, 256-byte aligned, large enough, and clear of every tensor."""
    def call(**kw):
        a = _bwd_ptrs(**kw)
        return lib.selscan_bwd_workspace(
            a["x"], a["delta"], a["A"], a["B"], a["C"], a["D"], a["z"], a["delta_bias"], 1,
            a["dy"], a["dfinal"], a["dx"], a["ddelta"], a["dA"], a["dB"], a["dC"], a["dD"],
            a["dz"], a["ddelta_bias"], a["batch"], 8, a["dim"], a["dstate"], 1, a["ws"],
            a["wsb"], None)
    need = lib.selscan_bwd_workspace_bytes(1, 8, 4, 16)
    ws = P + (1 << 24)  # far from every tensor
    assert call(ws=None) == 0  # nothing processed: no workspace needed
    full = dict(batch=1, dim=4)
    assert call(ws=None, wsb=need, **full) == -1
    assert call(ws=ws + 16, wsb=need, **full) == -4  # 256-byte alignment
    assert call(ws=ws, wsb=need - 1, **full) == -8
    assert call(ws=P + 4096 * 3, wsb=need, **full) == -7  # runs into B
    assert call(ws=P + 4096 * 13, wsb=need, **full) == -7  # runs into dB


def test_bwd_from_state_validation(lib):
    def call(**kw):
        a = _bwd_ptrs(**kw)
        return lib.selscan_bwd_from_state(
            a["x"], a["delta"], a["A"], a["B"], a["C"], a["D"], a["z"], a["delta_bias"], 1,
            a["h0"], a["dy"], a["dfinal"], a["dx"], a["ddelta"], a["dA"], a["dB"], a["dC"],
            a["dD"], a["dz"], a["ddelta_bias"], a["dh0"], a["batch"], 8, a["dim"],
            a["dstate"], 1, None, 0, None)
    h0, dh0 = P + 4096 * 18, P + 4096 * 19
    assert call(h0=h0, dh0=dh0) == 0  # batch = 0, dim = 0
    assert call(h0=h0, dh0=dh0 + 2) == -4
    assert call(h0=h0 + 2) == -4
    full = dict(batch=1, dim=4)
    assert call(h0=h0, dh0=h0, **full) == -7  # the gradient over its own input
    assert call(h0=P + 4096 * 10, **full) == -7  # the initial state runs into dx
    assert call(dfinal=P + 4096 * 9, dh0=P + 4096 * 9 + 64, **full) == -7
    assert call(dstate=257) == -5


def test_bwd_conv_validation(lib):
    def call(**kw):
        a = _bwd_ptrs(**kw)
        a.setdefault("width", 4)
        return lib.selscan_bwd_conv(
            a["x"], a["cw"], a["cb"], a["width"], a["delta"], a["A"], a["B"], a["C"], a["D"],
            a["z"], a["delta_bias"], 1, a["h0"], a["dy"], a["dfinal"], a["dx"], a["ddelta"],
            a["dA"], a["dB"], a["dC"], a["dD"], a["dz"], a["ddelta_bias"], a["dh0"], a["dcw"],
            a["dcb"], a["batch"], 8, a["dim"], a["dstate"], 1, None, 0, None)
    assert call() == 0
    assert call(width=0) == -2
    assert call(width=5) == -2
    full = dict(batch=1, dim=4)
    assert call(cw=None, **full) == -1
    assert call(dcw=None, **full) == -1
    assert call(dcw=P + 4096 * 22 + 2) == -4
    assert call(dcw=P + 4096 * 20, **full) == -7  # dconv_weight over conv_weight
    assert call(dcb=P + 4096 * 10, **full) == -7  # two outputs overlap


def test_bwd_conv_workspace_bytes(lib):
    f = lib.selscan_bwd_conv_workspace_bytes
    assert f(0, 8, 4, 16) == 0 and f(1, 0, 4, 16) == 0 and f(1, 8, 0, 16) == 0
    assert f(1, 8, 4, 0) == 0 and f(1, 8, 4, 257) == 0
    for shape in ((1, 8, 4, 16), (2, 300, 70, 16), (1, 100, 40, 40)):
        plain = lib.selscan_bwd_workspace_bytes(*shape)
        # besides the scan gradient's workspace: the conv output's float32 gradient
        assert f(*shape) >= plain + shape[0] * shape[1] * shape[2] * 4


def _step_ptrs(**kw):
    a = _ptrs(["state", "cs", "x", "cw", "cb", "delta", "A", "B", "C", "y"])
    a.update(cb=None, batch=0, dim=4, dstate=16, width=4)
    a.update(kw)
    return a


def test_state_update_conv_validation(lib):
    def call(**kw):
        a = _step_ptrs(**kw)
        return lib.selscan_state_update_conv(
            a["state"], a["cs"], a["x"], a["cw"], a["cb"], a["width"], a["delta"], a["A"],
            a["B"], a["C"], None, None, None, 1, a["y"], a["batch"], a["dim"], a["dstate"], 1,
            None)
    assert call() == 0
    assert call(width=0) == -2
    assert call(width=5) == -2
    assert call(batch=1, cs=None) == -1
    assert call(batch=1, cw=None) == -1
    assert call(cs=P + 4096 + 2) == -4
    assert call(batch=1, cs=P + 32) == -7  # conv_state runs into the state
    assert call(batch=1, cs=P + 4096 * 2) == -7  # conv_state over x_in
    assert call(batch=1, y=P + 4096) == -7  # y over conv_state


def test_state_update_ex_validation(lib):
    Opts = ss.selscan.StepOptions

    def call(opts, **kw):
        a = _step_ptrs(**kw)
        return lib.selscan_state_update_ex(
            a["state"], a["x"], a["delta"], a["A"], a["B"], a["C"], None, None, None, 1,
            ctypes.byref(opts) if opts is not None else None, a["y"], a["batch"], a["dim"],
            a["dstate"], 1, None)
    assert call(None) == 0
    assert call(Opts(bbar_mode=1)) == 0
    assert call(Opts(bbar_mode=2)) == -2
    assert call(Opts(conv_width=5)) == -2
    assert call(Opts(conv_width=4), batch=1) == -1  # no conv_state, no weight
    assert call(Opts(bbar_mode=1), dstate=257) == -5


def test_device_status_without_a_gpu(lib):
    assert lib.selscan_device_status(None, 0) == -1
    assert isinstance(ss.selscan_last_cuda_error(), str)
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("a GPU is visible: the status read succeeds there")
    st = ctypes.c_int(7)
    assert lib.selscan_device_status(ctypes.byref(st), 0) == -6  # no device: a CUDA error
    assert ss.selscan_last_cuda_error() != "no error"


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """Without the built library the binding raises: there is no fallback."""
    monkeypatch.setattr(ss.selscan, "_lib", None)
    with pytest.raises(ss.SelscanUnavailable, match="missing"):
        ss.selscan.load_library(str(tmp_path / "libselscan.so"))
    bad = tmp_path / "not_a_library.so"
    bad.write_bytes(b"not an ELF file")
    with pytest.raises(ss.SelscanUnavailable, match="cannot load"):
        ss.selscan.load_library(str(bad))


def test_product_and_oracle_share_no_code():
    """The package and its CUDA sources never import, include or load the
    oracle, and the oracle references none of the CUDA sources: the two sides
    of every parity test are independent."""
    pkg = os.path.join(ROOT, "selective_state_space_42_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if not f.endswith((".py", ".cu", ".cuh", ".h", ".cc", ".cpp")):
                continue
            text = open(os.path.join(dirpath, f), encoding="utf-8").read()
            assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), f
            assert not re.search(r'#include\s+["<][^">]*oracle', text), f
            assert "selscan_oracle" not in text, f
    for f in os.listdir(os.path.join(ROOT, "oracle")):
        if f.endswith((".py", ".c", ".h")):
            text = open(os.path.join(ROOT, "oracle", f), encoding="utf-8").read()
            assert not re.search(r"^\s*(import|from)\s+selective_state_space_42_b200\b",
                                 text, re.M), f
            assert not re.search(r'#include\s+["<][^">]*(selscan\.h|\.cuh)', text), f



@settings(max_examples=300, deadline=None)
@given(batch=st.integers(1, 16), seqlen=st.integers(1, 16384), dim=st.integers(1, 4096),
       dstate=st.integers(1, 256))
def test_plan_invariants_any_size(lib, batch, seqlen, dim, dstate):
    """The host planner (no GPU: 148 SMs assumed) on random sizes, with bf16
    tensors on 16-byte boundaries. It always makes one launch or three; the
    wide kernel (d_state above 16) runs in one pass with no workspace; a
    chunked plan has two or more chunks of at least 256 tokens and holds P and
    H for every chunk; TMA-eligible shapes with at least 60% as many
    (row, 128-channel) groups as SMs take the one-pass plan."""
    p = ss.selscan_fwd_plan(batch, seqlen, dim, dstate)
    assert p["launches"] in (1, 3) and p["chunks"] >= 1
    if dstate > 16:
        assert p == {"chunks": 1, "launches": 1, "workspace_bytes": 0}
        return
    if p["launches"] == 3:
        assert 2 <= p["chunks"] <= max(1, seqlen // 256)
        assert p["workspace_bytes"] >= 2 * batch * p["chunks"] * dim * 16 * 4
    eligible = dim >= 128 and (dim * 2) % 16 == 0 and (dstate * 2) % 16 == 0
    groups = batch * -(-dim // 128)
    if eligible and groups * 5 >= 148 * 3:
        assert p["launches"] == 1
        # the one pass keeps each group's 128 chains' states between chunks
        assert p["workspace_bytes"] >= groups * 128 * 16 * 4


def test_plan_of_empty_sizes(lib):
    for shape in ((0, 8, 4, 16), (2, 0, 4, 16), (2, 8, 0, 16)):
        assert ss.selscan_fwd_plan(*shape) == {"chunks": 0, "launches": 0, "workspace_bytes": 0}


@settings(max_examples=200, deadline=None)
@given(b=st.integers(1, 8), l=st.integers(1, 5000), d=st.integers(1, 3000),
       n=st.integers(1, 256), grow=st.sampled_from(["b", "l", "d", "n"]),
       by=st.integers(1, 300))
def test_gradient_workspace_grows_with_every_size(lib, b, l, d, n, grow, by):
    """More batch rows, tokens, channels or states never need less gradient
    workspace, and it always holds the float32 checkpoints: 16 states per
    chain and 16-state group every 8 tokens."""
    size = dict(b=b, l=l, d=d, n=n)
    bigger = dict(size)
    bigger[grow] = min(bigger[grow] + by, 256) if grow == "n" else bigger[grow] + by
    for f in (lib.selscan_bwd_workspace_bytes, lib.selscan_bwd_conv_workspace_bytes):
        small = f(size["b"], size["l"], size["d"], size["n"])
        large = f(bigger["b"], bigger["l"], bigger["d"], bigger["n"])
        assert 0 < small <= large
        groups = -(-n // 16)
        assert small >= groups * b * -(-l // 8) * d * 16 * 4


@settings(max_examples=200, deadline=None)
@given(b=st.integers(1, 4), l=st.integers(1, 5000), h=st.integers(1, 64),
       p=st.integers(1, 64), n=st.integers(1, 128),
       grow=st.sampled_from(["b", "l", "h", "p", "n"]), by=st.integers(1, 64))
def test_ssd_workspace_grows_with_every_size(lib, b, l, h, p, n, grow, by):
    size = dict(b=b, l=l, h=h, p=p, n=n)
    cap = {"p": 64, "n": 128}
    bigger = dict(size)
    bigger[grow] = min(bigger[grow] + by, cap.get(grow, 1 << 30))
    small = lib.selscan_ssd_workspace_bytes(*size.values())
    large = lib.selscan_ssd_workspace_bytes(*bigger.values())
    assert 0 < small <= large


def test_binding_error_mapping(lib):
    """A nonzero status becomes SelscanError carrying the status and the
    library's text; a CUDA failure appends the CUDA error text."""
    torch = pytest.importorskip("torch")
    ss.selscan._check(0)
    for code, name in ss.selscan.STATUS.items():
        if code == 0:
            continue
        with pytest.raises(ss.SelscanError) as e:
            ss.selscan._check(code)
        assert e.value.status == code and name in str(e.value)
        assert ss.selscan_status_string(code) in str(e.value)
    with pytest.raises(ss.SelscanError, match=re.escape(ss.selscan_last_cuda_error())):
        ss.selscan._check(-6)
    assert ss.selscan._dtype_code(torch.zeros(1)) == ss.SELSCAN_F32
    assert ss.selscan._dtype_code(torch.zeros(1, dtype=torch.bfloat16)) == ss.SELSCAN_BF16
    with pytest.raises(TypeError):
        ss.selscan._dtype_code(torch.zeros(1, dtype=torch.float16))
    with pytest.raises(ValueError, match="required"):
        ss.selscan._ptr(None, "x")
    assert ss.selscan._ptr(None, "z", required=False) is None


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "selscan.h"

int main(void) {
    int64_t chunks = -1, launches = -1, ws = -1;
    int st = selscan_fwd_plan(4, 8192, 5120, 16, &chunks, &launches, &ws);
    printf("%d %lld %lld %lld\n", st, (long long)chunks, (long long)launches, (long long)ws);
    printf("%lld\n", (long long)selscan_bwd_workspace_bytes(1, 8, 4, 16));
    printf("%s\n", selscan_status_string(SELSCAN_ERR_ALIAS));
    /* batch = 0, dim = 0: validated, nothing to do, no CUDA call */
    printf("%d\n", selscan_fwd(0, 0, 0, 0, 0, 0, 0, 0, 1, 0, 0, 0, 8, 0, 16, SELSCAN_BF16, 0));
    /* dim = 4 without A: rejected before any CUDA call */
    printf("%d\n", selscan_fwd(0, 0, 0, 0, 0, 0, 0, 0, 1, 0, 0, 0, 8, 4, 16, SELSCAN_BF16, 0));
    return 0;
}
"""


def test_plain_c_client_links_and_calls(lib, tmp_path):
    """The header compiles as pedantic C99 and a C program links against
    libselscan and calls its host-only entry points: the ABI needs neither
    Python nor C++."""
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    libdir = os.path.dirname(ss.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                    "-L", libdir, "-lselscan", "-Wl,-rpath," + libdir],
                   check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True,
                         timeout=60).stdout.split("\n")
    st, chunks, launches, ws = (int(v) for v in out[0].split())
    assert (st, chunks, launches) == (0, 8, 1) and ws > 0
    assert int(out[1]) == lib.selscan_bwd_workspace_bytes(1, 8, 4, 16)
    assert out[2] == ss.selscan_status_string(-7)
    assert int(out[3]) == 0
    assert int(out[4]) == -1  # SELSCAN_ERR_NULL_ARG
