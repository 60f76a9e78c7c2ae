"""The hot path inside CUDA graphs: decode steps, the scan (persistent TMA
plan, workspace allocated on the stream), its gradient and the tensor-core
SSD form are captured with torch.cuda.CUDAGraph and replayed; every replay
reproduces the eager results bit for bit (the kernels are deterministic)."""
import pytest
import torch

import selective_state_space_42_b200 as ss
from selective_state_space_42_b200 import workloads as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _capture(fn):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        out = fn()
    return g, out


def test_decode_steps_in_a_graph():
    w = wl.DecodeWorkload("graph", 8, 384, 16, 4, "bf16", True, 31)
    state0 = wl.make_decode_state(w, device=DEV)
    A, Dv, bias = wl.make_decode_params(w, device=DEV)
    steps = [wl.make_decode_step(w, s, device=DEV) for s in range(4)]

    def run(state, ys):
        for s, y in zip(steps, ys):
            ss.selscan_state_update(state, s["x"], s["delta"], A, s["B"], s["C"], Dv, s["z"],
                                    bias, y=y)

    se = state0.clone()
    ye = [torch.empty(8, 384, device=DEV, dtype=torch.bfloat16) for _ in range(4)]
    run(se, ye)
    sg = state0.clone()
    yg = [torch.empty_like(y) for y in ye]
    g, _ = _capture(lambda: run(sg, yg))
    sg.copy_(state0)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(sg, se)
    for a, b in zip(yg, ye):
        assert torch.equal(a, b)
    g.replay()  # a second replay continues from the advanced state
    run(se, ye)
    torch.cuda.synchronize()
    assert torch.equal(sg, se)


def test_scan_and_gradient_in_a_graph():
    w = wl.ScanWorkload("graph", 2, 1024, 512, 16, "bf16", gate=True, seed=32)
    inp = wl.make_scan_inputs(w, device=DEV)
    args = (inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["z"],
            inp["delta_bias"])
    dy = torch.randn(2, 1024, 512, device=DEV).to(torch.bfloat16)
    ye, he = ss.selscan_fwd(*args, return_final_state=True)
    ge = ss.selscan_bwd(*args, dy=dy)
    yg = torch.empty_like(ye)
    hg = torch.empty_like(he)

    def body():
        ss.selscan_fwd(*args, y=yg, final_state=hg)
        return ss.selscan_bwd(*args, dy=dy)

    g, grads = _capture(body)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(yg, ye) and torch.equal(hg, he)
    for k, v in ge.items():
        if v is not None:
            assert torch.equal(grads[k], v), k
    assert ss.selscan_fwd_plan(2, 1024, 512, 16)["launches"] >= 1


def test_ssd_in_a_graph():
    w = wl.SsdWorkload("graph", 2, 640, 4, 64, 128, "bf16", gate=True, seed=33)
    inp = wl.make_ssd_inputs(w, device=DEV)

    def call(y=None, fs=None):
        return ss.selscan_ssd_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                                  z=inp["z"], dt_bias=inp["dt_bias"], y=y, final_state=fs,
                                  return_final_state=True)

    ye, he = call()
    yg, hg = torch.empty_like(ye), torch.empty_like(he)
    g, _ = _capture(lambda: call(yg, hg))
    for _ in range(2):
        yg.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(yg, ye) and torch.equal(hg, he)
    assert ss.selscan_device_status() == 0
