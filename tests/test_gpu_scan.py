"""GPU parity of selscan_fwd against the float64 oracle, through the C ABI.

Small cases compare every output element; the full-size workloads (the same
plan the benchmark times) compare every token of a deterministic channel
sample. Tolerances: see gpu_helpers.RTOL.
"""
import numpy as np
import pytest
import torch

import selective_state_space_42_b200 as ss
from selective_state_space_42_b200 import workloads as wl

import gpu_helpers as gh
from test_golden import golden_arrays, load_golden

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _cuda(inp):
    return {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}


def _random_A(dim, N, seed):
    g = torch.Generator().manual_seed(seed)
    return (-torch.exp(torch.rand(dim, N, generator=g) * 3.0 - 1.0)).float()


def _check_fwd(inp, rtol, softplus=True, what=""):
    y, hs = gh.gpu_fwd(inp, softplus=softplus)
    torch.cuda.synchronize()
    yo, ho = gh.oracle_fwd(inp, softplus=softplus)
    gh.compare(gh.to_np(y), yo, rtol, what + " y")
    gh.compare(gh.to_np(hs), ho, rtol, what + " final_state")


def test_tiny_f32_full():
    """The tiny fp32 workload, every element, default plan and chunked."""
    w = wl.WORKLOADS["tiny_f32"]
    inp = _cuda(wl.make_scan_inputs(w))
    _check_fwd(inp, 1e-4, what="tiny_f32")
    with gh.forced_chunks(4):
        _check_fwd(inp, 1e-4, what="tiny_f32 chunked")


def test_golden_cases():
    for case in load_golden():
        arrs, y_ref, h_ref = golden_arrays(case)
        dt = torch.float32 if case["dtype"] == "f32" else torch.bfloat16
        inp = {}
        for k, v in arrs.items():
            if v is None:
                inp[k] = None
            else:
                t = torch.from_numpy(v)
                inp[k] = (t.float() if k in ("A", "D", "delta_bias") else t.to(dt)).to(DEV)
        y, hs = gh.gpu_fwd(inp)
        torch.cuda.synchronize()
        rtol = gh.RTOL[case["dtype"]]
        gh.compare(gh.to_np(y), y_ref, rtol, case["name"])
        gh.compare(gh.to_np(hs), h_ref, rtol, case["name"] + " state")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", wl.ragged_shapes(), ids=str)
@pytest.mark.parametrize("variant", ["structA_gate", "randomA_nogate", "randomA_gate_nosoftplus"])
@pytest.mark.parametrize("chunks", [1, 3])
def test_ragged(dtype, shape, variant, chunks):
    batch, L, dim, N = shape
    w = wl.ScanWorkload("ragged", batch, L, dim, N, dtype,
                        gate="nogate" not in variant,
                        seed=1000 + L + dim + N)
    inp = wl.make_scan_inputs(w)
    softplus = "nosoftplus" not in variant
    if variant.startswith("randomA"):
        inp["A"] = _random_A(dim, N, seed=L * 7 + dim)
    if not softplus:
        inp["delta"] = inp["delta"].abs().mul(0.2).to(inp["delta"].dtype)
        inp["delta_bias"] = None
    inp = _cuda(inp)
    with gh.forced_chunks(chunks):
        _check_fwd(inp, gh.RTOL[dtype], softplus=softplus, what=f"{shape} {variant}")


TMA_SHAPES = [(1, 1, 128, 16), (2, 33, 136, 16), (1, 300, 256, 8), (3, 257, 384, 16),
              (2, 1000, 200, 4), (1, 2049, 128, 1), (4, 96, 1024, 16)]
TMA_PATHS = {
    "seq_unit32": dict(SELSCAN_PATH="seq", SELSCAN_UNIT="32", SELSCAN_CHUNKS=None),
    "seq_default": dict(SELSCAN_PATH="seq", SELSCAN_UNIT=None, SELSCAN_CHUNKS=None),
    "chunked3": dict(SELSCAN_PATH="chunked", SELSCAN_UNIT=None, SELSCAN_CHUNKS="3"),
    "chunked_auto": dict(SELSCAN_PATH="chunked", SELSCAN_UNIT=None, SELSCAN_CHUNKS=None),
}


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", TMA_SHAPES, ids=str)
@pytest.mark.parametrize("variant", ["structA_gate", "randomA_nogate"])
@pytest.mark.parametrize("path", list(TMA_PATHS))
def test_tma_paths(dtype, shape, variant, path):
    """The TMA-staged kernel in each of its plans, on ragged channel tiles
    (dim not a multiple of 128), ragged token tiles and d_state 1..16."""
    batch, L, dim, N = shape
    w = wl.ScanWorkload("tma", batch, L, dim, N, dtype, gate=variant.endswith("_gate"),
                        seed=2000 + L + dim + N)
    inp = wl.make_scan_inputs(w)
    if variant.startswith("randomA"):
        inp["A"] = _random_A(dim, N, seed=L * 11 + dim)
    inp = _cuda(inp)
    with gh.env(**TMA_PATHS[path]):
        _check_fwd(inp, gh.RTOL[dtype], what=f"{shape} {variant} {path}")
    assert ss.selscan_device_status() == 0


def test_empty_and_degenerate():
    f32 = torch.float32
    # L = 0: nothing to compute, final state is zero
    x = torch.empty(2, 0, 8, device=DEV)
    A = -torch.ones(8, 4, device=DEV)
    BC = torch.empty(2, 0, 4, device=DEV)
    y, hs = ss.selscan_fwd(x, x, A, BC, BC, return_final_state=True,
                           final_state=torch.full((2, 8, 4), 7.0, device=DEV))
    torch.cuda.synchronize()
    assert y.shape == (2, 0, 8) and torch.all(hs == 0)
    # batch = 0 and dim = 0
    ss.selscan_fwd(torch.empty(0, 5, 8, device=DEV), torch.empty(0, 5, 8, device=DEV), A,
                   torch.empty(0, 5, 4, device=DEV), torch.empty(0, 5, 4, device=DEV))
    ss.selscan_fwd(torch.empty(1, 5, 0, device=DEV), torch.empty(1, 5, 0, device=DEV),
                   torch.empty(0, 4, device=DEV), torch.zeros(1, 5, 4, device=DEV),
                   torch.zeros(1, 5, 4, device=DEV))
    # A = 0, softplus off, delta = 0: Abar = 1 and Δ = 0 -> state stays 0, y = D·x
    x = torch.randn(1, 40, 16, device=DEV)
    y, hs = ss.selscan_fwd(x, torch.zeros_like(x), torch.zeros(16, 16, device=DEV),
                           torch.randn(1, 40, 16, device=DEV),
                           torch.randn(1, 40, 16, device=DEV),
                           D=torch.full((16,), 2.0, device=DEV), softplus=False,
                           return_final_state=True)
    torch.cuda.synchronize()
    assert torch.equal(y, 2.0 * x) and torch.all(hs == 0)
    assert f32 == hs.dtype


def test_errors_raise():
    x = torch.zeros(1, 4, 8, device=DEV, dtype=torch.bfloat16)
    A = -torch.ones(8, 257, device=DEV)
    BC = torch.zeros(1, 4, 257, device=DEV, dtype=torch.bfloat16)
    with pytest.raises(ss.SelscanError) as e:
        ss.selscan_fwd(x, x, A, BC, BC)
    assert e.value.status == -5
    y = torch.zeros_like(x)
    with pytest.raises(ss.SelscanError) as e:  # y aliases x
        ss.selscan_fwd(x, x.clone(), -torch.ones(8, 16, device=DEV),
                       torch.zeros(1, 4, 16, device=DEV, dtype=torch.bfloat16),
                       torch.zeros(1, 4, 16, device=DEV, dtype=torch.bfloat16), y=x)
    assert e.value.status == -7
    del y


def _full_size_sampled(name, stride, chunks=None, batches=None):
    w = wl.WORKLOADS[name]
    inp = wl.make_scan_inputs(w, device=DEV)
    if chunks is None:
        y, hs = gh.gpu_fwd(inp)
    else:
        with gh.forced_chunks(chunks):
            y, hs = gh.gpu_fwd(inp)
    torch.cuda.synchronize()
    chans = wl.channel_subset(w.dim, stride)
    bsel = list(range(w.batch)) if batches is None else batches
    yo, ho = gh.oracle_fwd(inp, channels=chans, batches=bsel)
    yg = gh.to_np(y[bsel][:, :, chans])
    hg = gh.to_np(hs[bsel][:, chans, :])
    r1 = gh.compare(yg, yo, gh.RTOL[w.dtype], name + " y (sampled)")
    r2 = gh.compare(hg, ho, gh.RTOL[w.dtype], name + " final_state (sampled)")
    del inp, y, hs
    torch.cuda.empty_cache()
    return r1, r2


def test_mamba130m_layer_sampled():
    _full_size_sampled("mamba130m_layer", 64)


def test_mamba2p8b_layer_sampled():
    """The benchmark's workload, in the benchmark's launch configuration."""
    _full_size_sampled("mamba2p8b_layer", 160)


def test_mamba2p8b_layer_expA_sampled():
    """The benchmark's workload with the pages' A = −exp(log(1..16)) in float32,
    a few ulps off the integers: within the ladder test's bound, so it takes
    the power-ladder decay of (n+1)·A[d, 0]."""
    _full_size_sampled("mamba2p8b_layer_expA", 160)


def test_mamba2p8b_layer_trainedA_sampled():
    """The benchmark's workload with a general A (−exp(log(n+1) + 0.1·N(0,1))
    per channel and state): the general decay, one exp per state, part of
    them on the FMA pipe."""
    _full_size_sampled("mamba2p8b_layer_trainedA", 160)


@pytest.mark.parametrize("a_init", ["exp_log", "random"])
def test_general_A_final_state_tight(a_init):
    """General A with bf16 I/O: y is rounded to bf16, but the float32 final
    state carries the error of the decay factors themselves (MUFU ex2 and the
    degree-4 polynomial, 2.7e-6), so it is held to 1e-3."""
    w = wl.ScanWorkload("genA", 2, 2048, 256, 16, "bf16", gate=True, seed=41,
                        a_init="exp_log")
    inp = _cuda(wl.make_scan_inputs(w))
    if a_init == "random":
        inp["A"] = _random_A(w.dim, w.dstate, 42).to(DEV)
    y, hs = gh.gpu_fwd(inp)
    torch.cuda.synchronize()
    yo, ho = gh.oracle_fwd(inp)
    gh.compare(gh.to_np(y), yo, gh.RTOL["bf16"], "general A y")
    gh.compare(gh.to_np(hs), ho, 1e-3, "general A final_state")


def test_mamba2p8b_layer_chunked_sampled():
    _full_size_sampled("mamba2p8b_layer", 512, chunks=4, batches=[0, 3])


def test_long_1m_sampled():
    """One 1M-token sequence: chunk carry across many chunks, state continuity
    over the whole length."""
    _full_size_sampled("long_1m", 512)


def test_generic_path_forced_on_bench_shape_sampled():
    """The generic kernels on the benchmark's workload (planner override)."""
    with gh.env(SELSCAN_PATH="generic"):
        _full_size_sampled("mamba2p8b_layer", 1024, batches=[0, 3])


def test_no_device_wait_gave_up():
    assert ss.selscan_device_status(clear=True) == 0


def test_cross_entry_fwd_then_decode():
    """fwd over [0, L1) then L − L1 decode steps == fwd over [0, L)."""
    w = wl.ScanWorkload("xentry", 2, 96, 320, 16, "f32", gate=True, seed=77)
    inp = _cuda(wl.make_scan_inputs(w))
    y_full, h_full = gh.gpu_fwd(inp)
    L1 = 50
    pre = {k: (v[:, :L1].contiguous() if k in ("x", "delta", "z", "B", "C") else v)
           for k, v in inp.items()}
    _, h = gh.gpu_fwd(pre)
    ys = []
    for t in range(L1, w.seqlen):
        ys.append(ss.selscan_state_update(
            h, inp["x"][:, t].contiguous(), inp["delta"][:, t].contiguous(), inp["A"],
            inp["B"][:, t].contiguous(), inp["C"][:, t].contiguous(), inp["D"],
            inp["z"][:, t].contiguous(), inp["delta_bias"]))
    torch.cuda.synchronize()
    y_dec = torch.stack(ys, dim=1)
    gh.compare(gh.to_np(y_dec), gh.to_np(y_full[:, L1:]), 1e-4, "decode vs fwd y")
    gh.compare(gh.to_np(h), gh.to_np(h_full), 1e-4, "decode vs fwd state")
    assert np.isfinite(gh.to_np(h)).all()
