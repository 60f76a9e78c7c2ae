"""GPU parity of the zero-order-hold input term (Bbar = (exp(Δ·A) − 1)/A·B,
C ABI selscan_fwd_ex / selscan_state_update_ex) against the oracle's ZOH
mode, which is pinned against the matrix exponential formula."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_42_b200 as ss
from selective_state_space_42_b200 import workloads as wl

import gpu_helpers as gh

pytestmark = pytest.mark.gpu
DEV = "cuda"
ZOH = oracle.BBAR_ZOH


def _inputs(batch, L, dim, N, dtype, seed, A_kind):
    w = wl.ScanWorkload("zoh", batch, L, dim, N, dtype, gate=True, seed=seed)
    inp = wl.make_scan_inputs(w)
    g = torch.Generator().manual_seed(seed + 3)
    if A_kind == "random":
        inp["A"] = -torch.rand(dim, N, generator=g) * 4 - 0.1
    elif A_kind == "with_zeros":
        A = -torch.rand(dim, N, generator=g) * 4
        A[::3, ::2] = 0.0  # the Δ·B limit of the ZOH term
        inp["A"] = A
    return inp


def _oracle(inp, h0=None):
    n = gh.to_np
    return oracle.default().fwd(n(inp["x"]), n(inp["delta"]), n(inp["A"]), n(inp["B"]),
                                n(inp["C"]), n(inp["D"]), n(inp["z"]), n(inp["delta_bias"]),
                                bbar=ZOH, h0=None if h0 is None else n(h0))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(1, 1, 8, 16), (2, 77, 130, 16), (1, 300, 40, 7),
                                   (3, 64, 256, 16)], ids=str)
@pytest.mark.parametrize("A_kind", ["structured", "random", "with_zeros"])
def test_zoh_scan(dtype, shape, A_kind):
    batch, L, dim, N = shape
    inp = _inputs(batch, L, dim, N, dtype, 5000 + L + dim, A_kind)
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    y, hf = ss.selscan_fwd(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["z"],
                           d["delta_bias"], bbar="zoh", return_final_state=True)
    torch.cuda.synchronize()
    yo, ho = _oracle(inp)
    gh.compare(gh.to_np(y), yo, gh.RTOL[dtype], f"{shape} {A_kind} y")
    gh.compare(gh.to_np(hf), ho, gh.RTOL[dtype], f"{shape} {A_kind} final state")


def test_zoh_chunked_with_initial_state():
    inp = _inputs(1, 2000, 96, 16, "f32", 5100, "random")
    g = torch.Generator().manual_seed(5101)
    h0 = torch.randn(1, 96, 16, generator=g)
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    with gh.env(SELSCAN_PATH=None, SELSCAN_CHUNKS="5", SELSCAN_UNIT=None):
        y, hf = ss.selscan_fwd(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["z"],
                               d["delta_bias"], bbar="zoh", initial_state=h0.to(DEV),
                               return_final_state=True)
        torch.cuda.synchronize()
    yo, ho = _oracle(inp, h0)
    gh.compare(gh.to_np(y), yo, gh.RTOL["f32"], "chunked zoh y")
    gh.compare(gh.to_np(hf), ho, gh.RTOL["f32"], "chunked zoh final state")


def test_zoh_differs_from_delta_term():
    """The two input terms give different results on the same inputs (so the
    mode switch is not ignored), and agree as Δ·A → 0."""
    inp = _inputs(1, 50, 64, 16, "f32", 5200, "random")
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    args = (d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["z"], d["delta_bias"])
    y_delta = ss.selscan_fwd(*args)
    y_zoh = ss.selscan_fwd(*args, bbar="zoh")
    torch.cuda.synchronize()
    assert (y_delta - y_zoh).abs().max() > 1e-3
    small = {**d, "A": d["A"] * 1e-6}
    y1 = ss.selscan_fwd(small["x"], small["delta"], small["A"], small["B"], small["C"],
                        small["D"], small["z"], small["delta_bias"])
    y2 = ss.selscan_fwd(small["x"], small["delta"], small["A"], small["B"], small["C"],
                        small["D"], small["z"], small["delta_bias"], bbar="zoh")
    torch.cuda.synchronize()
    gh.compare(gh.to_np(y2), gh.to_np(y1).astype(np.float64), 1e-4, "zoh -> delta as A -> 0")


@pytest.mark.parametrize("N", [16, 7])
def test_zoh_decode_steps(N):
    """Decode steps with the ZOH term against the oracle's one-token scan from
    the previous state, step after step."""
    batch, dim, steps = 3, 70, 8
    inp = _inputs(batch, steps, dim, N, "f32", 5300 + N, "random")
    g = torch.Generator().manual_seed(5301)
    state = (torch.randn(batch, dim, N, generator=g) * 0.1)
    ref = state.clone()
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    sd = state.to(DEV)
    for t in range(steps):
        tok = {k: d[k][:, t].contiguous() for k in ("x", "delta", "z", "B", "C")}
        y = ss.selscan_state_update(sd, tok["x"], tok["delta"], d["A"], tok["B"], tok["C"],
                                    d["D"], tok["z"], d["delta_bias"], bbar="zoh")
        one = {k: (v[:, t:t + 1] if v is not None and v.dim() == 3 else v)
               for k, v in inp.items()}
        yo, ho = _oracle(one, ref)
        ref = torch.from_numpy(ho)
        torch.cuda.synchronize()
        gh.compare(gh.to_np(y), yo[:, 0], gh.RTOL["f32"], f"step {t} y")
        gh.compare(gh.to_np(sd), ho, gh.RTOL["f32"], f"step {t} state")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("plan", ["seq_unit64", "chunked3"])
@pytest.mark.parametrize("A_kind", ["structured", "random", "with_zeros"])
def test_zoh_tma_plans(dtype, plan, A_kind):
    """The ZOH term on the TMA-staged kernel (dim a multiple of 128, aligned
    rows): the one-pass plan with state hand-off and the chunked plan, over
    several tiles and a ragged tail."""
    env = {"seq_unit64": dict(SELSCAN_PATH="seq", SELSCAN_UNIT="64", SELSCAN_CHUNKS=None),
           "chunked3": dict(SELSCAN_PATH="chunked", SELSCAN_UNIT=None, SELSCAN_CHUNKS="3")}[plan]
    inp = _inputs(2, 1000, 384, 16, dtype, 5200, A_kind)
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    with gh.env(**env):
        y, hf = ss.selscan_fwd(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["z"],
                               d["delta_bias"], bbar="zoh", return_final_state=True)
        torch.cuda.synchronize()
    yo, ho = _oracle(inp)
    gh.compare(gh.to_np(y), yo, gh.RTOL[dtype], f"{plan} {A_kind} y")
    gh.compare(gh.to_np(hf), ho, gh.RTOL[dtype], f"{plan} {A_kind} final state")
