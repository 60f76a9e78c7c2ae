"""GPU parity of selscan_state_update (the in-place single-token decode step)
against the oracle's recurrence, through the C ABI, plus exact layout and
indexing checks of the [batch, dim, dstate] state."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_42_b200 as ss
from selective_state_space_42_b200 import workloads as wl

import gpu_helpers as gh

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _step(state, inp, params, softplus=True):
    A, Dv, bias = params
    return ss.selscan_state_update(state, inp["x"], inp["delta"], A, inp["B"], inp["C"],
                                   Dv, inp.get("z"), bias, softplus=softplus)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(1, 1, 1), (3, 37, 16), (5, 130, 7), (2, 64, 4),
                                   (4, 3, 16), (7, 1, 16), (3, 9, 16)],
                         ids=str)
@pytest.mark.parametrize("gate", [True, False])
def test_small_steps_every_element(dtype, shape, gate):
    batch, dim, N = shape
    w = wl.DecodeWorkload("small", batch, dim, N, 20, dtype, gate, seed=500 + dim)
    state = wl.make_decode_state(w).to(DEV)
    A, Dv, bias = (t.to(DEV) for t in wl.make_decode_params(w))
    if N != 16:
        g = torch.Generator().manual_seed(600 + dim)
        A = (-torch.rand(dim, N, generator=g) * 4 - 0.1).to(DEV)
    ref = gh.to_np(state)
    orc = oracle.default()
    ys, yos, sts, refs = [], [], [], []
    for s in range(w.steps):
        inp = {k: (None if v is None else v.to(DEV)) for k, v in wl.make_decode_step(w, s).items()}
        y = _step(state, inp, (A, Dv, bias))
        yo, ref = orc.state_update(ref, gh.to_np(inp["x"]), gh.to_np(inp["delta"]),
                                   gh.to_np(A), gh.to_np(inp["B"]), gh.to_np(inp["C"]),
                                   gh.to_np(Dv), gh.to_np(inp.get("z")), gh.to_np(bias))
        torch.cuda.synchronize()
        ys.append(gh.to_np(y))
        yos.append(yo)
        sts.append(gh.to_np(state))
        refs.append(ref.copy())
    # every element of every step; the rms floor is taken over the trajectory
    gh.compare(np.stack(ys), np.stack(yos), gh.RTOL[dtype], "y trajectory")
    gh.compare(np.stack(sts), np.stack(refs), gh.RTOL[dtype], "state trajectory")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_unaligned_bc(dtype):
    """B and C starting one element past an 8-byte (bf16) or 16-byte (f32)
    boundary: the step must give the same values as the oracle (the vector
    loads are not usable there)."""
    batch, dim, N = 3, 70, 16
    w = wl.DecodeWorkload("unaligned", batch, dim, N, 3, dtype, True, seed=77)
    state = wl.make_decode_state(w).to(DEV)
    A, Dv, bias = (t.to(DEV) for t in wl.make_decode_params(w))
    ref = gh.to_np(state)
    orc = oracle.default()
    for s in range(w.steps):
        inp = {k: (None if v is None else v.to(DEV)) for k, v in wl.make_decode_step(w, s).items()}
        for key in ("B", "C"):
            big = torch.empty(batch * N + 1, dtype=inp[key].dtype, device=DEV)
            view = big[1:].view(batch, N)
            view.copy_(inp[key])
            inp[key] = view
            assert view.data_ptr() % 8 != 0
        y = _step(state, inp, (A, Dv, bias))
        yo, ref = orc.state_update(ref, gh.to_np(inp["x"]), gh.to_np(inp["delta"]),
                                   gh.to_np(A), gh.to_np(inp["B"]), gh.to_np(inp["C"]),
                                   gh.to_np(Dv), gh.to_np(inp.get("z")), gh.to_np(bias))
        torch.cuda.synchronize()
        gh.compare(gh.to_np(y), yo, gh.RTOL[dtype], f"y step {s}")
        gh.compare(gh.to_np(state), ref, gh.RTOL[dtype], f"state step {s}")


def test_decode_workload_1000_steps_sampled():
    """The decode workload: [256, 5120, 16] state, 1000 consecutive steps on
    the GPU; y checked at every step and the state at steps 1, 10, 100, 1000
    on a deterministic sample of batch rows and channels."""
    w = wl.DECODE
    state = wl.make_decode_state(w, device=DEV)
    A, Dv, bias = wl.make_decode_params(w, device=DEV)
    rows = sorted({0, 1, 127, w.batch - 1} | set(range(0, w.batch, 32)))
    chans = wl.channel_subset(w.dim, 128)
    ref = gh.to_np(state[rows][:, chans])
    orc = oracle.default()
    An, Dn, bn = gh.to_np(A[chans]), gh.to_np(Dv[chans]), gh.to_np(bias[chans])
    for s in range(w.steps):
        inp = wl.make_decode_step(w, s, device=DEV)
        y = _step(state, inp, (A, Dv, bias))
        yo, ref = orc.state_update(
            ref, gh.to_np(inp["x"][rows][:, chans]), gh.to_np(inp["delta"][rows][:, chans]),
            An, gh.to_np(inp["B"][rows]), gh.to_np(inp["C"][rows]), Dn,
            gh.to_np(inp["z"][rows][:, chans]), bn)
        gh.compare(gh.to_np(y[rows][:, chans]), yo, 2e-2, f"decode step {s} y")
        if s + 1 in (1, 10, 100, 1000):
            gh.compare(gh.to_np(state[rows][:, chans]), ref, 2e-2, f"decode state {s + 1}")


def test_layout_bit_exact():
    """A = 0 (Abar = 1 exactly) and x = 0 leave the state bit-identical; a
    one-hot x at (b0, d0) with B one-hot at n0 changes exactly
    state[b0, d0, n0], by exactly Δ·B·x computed in float32."""
    batch, dim, N = 6, 300, 16
    g = torch.Generator().manual_seed(9)
    st0 = torch.randn(batch, dim, N, generator=g)
    state = st0.clone().to(DEV)
    A = torch.zeros(dim, N, device=DEV)
    delta = (torch.rand(batch, dim, generator=g) * 0.9 + 0.1).to(DEV)
    Cm = torch.randn(batch, N, generator=g).to(DEV)
    ss.selscan_state_update(state, torch.zeros(batch, dim, device=DEV), delta, A,
                            torch.randn(batch, N, generator=g).to(DEV), Cm, softplus=False)
    torch.cuda.synchronize()
    assert torch.equal(state.cpu(), st0)
    b0, d0, n0 = 4, 211, 13
    x = torch.zeros(batch, dim, device=DEV)
    x[b0, d0] = 1.5
    Bo = torch.zeros(batch, N, device=DEV)
    Bo[b0, n0] = -0.75
    ss.selscan_state_update(state, x, delta, A, Bo, Cm, softplus=False)
    torch.cuda.synchronize()
    got = state.cpu()
    changed = (got != st0).nonzero().tolist()
    assert changed == [[b0, d0, n0]]
    dt = delta[b0, d0].cpu()
    expect = torch.tensor(st0[b0, d0, n0].item(), dtype=torch.float32) + \
        (dt * 1.5) * torch.tensor(-0.75)
    assert got[b0, d0, n0].item() == expect.item()


def test_fwd_final_state_feeds_decode_layout():
    """final_state written by selscan_fwd is read back by the decode step in
    the same [batch, dim, dstate] order: with A = 0 and x = 0 the step returns
    y = C·state exactly as float64 math on that state says (to fp32)."""
    batch, L, dim, N = 2, 33, 130, 16
    w = wl.ScanWorkload("layout", batch, L, dim, N, "f32", gate=False, seed=31)
    inp = {k: (None if v is None else v.to(DEV)) for k, v in wl.make_scan_inputs(w).items()}
    _, hs = gh.gpu_fwd(inp)
    Cm = torch.randn(batch, N, device=DEV)
    y = ss.selscan_state_update(hs.clone(), torch.zeros(batch, dim, device=DEV),
                                torch.zeros(batch, dim, device=DEV),
                                torch.zeros(dim, N, device=DEV),
                                torch.zeros(batch, N, device=DEV), Cm, softplus=False)
    torch.cuda.synchronize()
    expect = np.einsum("bdn,bn->bd", gh.to_np(hs), gh.to_np(Cm))
    gh.compare(gh.to_np(y), expect, 1e-5, "C·state")
