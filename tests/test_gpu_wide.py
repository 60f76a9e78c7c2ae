"""GPU parity of the scan and the decode step for d_state 17..256 (the
wide-state kernel: each chain's states split over several lanes) against the
oracle, which takes any d_state."""
import pytest
import torch

import oracle
import selective_state_space_42_b200 as ss
from selective_state_space_42_b200 import workloads as wl

import gpu_helpers as gh

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(batch, L, dim, N, dtype, seed, A_kind, gate=True):
    w = wl.ScanWorkload("wide", batch, L, dim, N, dtype, gate=gate, seed=seed)
    inp = wl.make_scan_inputs(w)
    g = torch.Generator().manual_seed(seed + 1)
    if A_kind == "random":
        inp["A"] = -torch.rand(dim, N, generator=g) * 4 - 0.1
    elif A_kind == "per_channel":  # one scalar per channel, as in the Mamba-2 heads
        inp["A"] = (-torch.rand(dim, 1, generator=g) * 2 - 0.05).repeat(1, N).contiguous()
    return inp


def _oracle(inp, h0=None, bbar=oracle.BBAR_DELTA):
    n = gh.to_np
    return oracle.default().fwd(n(inp["x"]), n(inp["delta"]), n(inp["A"]), n(inp["B"]),
                                n(inp["C"]), n(inp["D"]), n(inp["z"]), n(inp["delta_bias"]),
                                h0=None if h0 is None else n(h0), bbar=bbar)


def _gpu(inp, **kw):
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    return ss.selscan_fwd(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["z"],
                          d["delta_bias"], return_final_state=True, **kw)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [17, 32, 64, 100, 128, 256])
@pytest.mark.parametrize("A_kind", ["structured", "per_channel", "random"])
def test_wide_scan(dtype, N, A_kind):
    inp = _inputs(2, 37, 70, N, dtype, 6000 + N, A_kind)
    y, hf = _gpu(inp)
    torch.cuda.synchronize()
    yo, ho = _oracle(inp)
    gh.compare(gh.to_np(y), yo, gh.RTOL[dtype], f"N={N} {A_kind} y")
    gh.compare(gh.to_np(hf), ho, gh.RTOL[dtype], f"N={N} {A_kind} final state")


@pytest.mark.parametrize("N", [48, 256])
def test_wide_options(N):
    """Initial state, no gate, ZOH term and the conv front end on the wide
    kernel."""
    inp = _inputs(2, 50, 40, N, "f32", 6100 + N, "random", gate=False)
    g = torch.Generator().manual_seed(6101)
    h0 = torch.randn(2, 40, N, generator=g) * 0.3
    y, hf = _gpu(inp, initial_state=h0.to(DEV))
    yz, hz = _gpu(inp, initial_state=h0.to(DEV), bbar="zoh")
    torch.cuda.synchronize()
    yo, ho = _oracle(inp, h0)
    gh.compare(gh.to_np(y), yo, gh.RTOL["f32"], "h0 y")
    gh.compare(gh.to_np(hf), ho, gh.RTOL["f32"], "h0 final state")
    yzo, hzo = _oracle(inp, h0, bbar=oracle.BBAR_ZOH)
    gh.compare(gh.to_np(yz), yzo, gh.RTOL["f32"], "zoh y")
    gh.compare(gh.to_np(hz), hzo, gh.RTOL["f32"], "zoh final state")
    cw = torch.randn(40, 4, generator=g) * 0.5
    cb = torch.randn(40, generator=g) * 0.1
    yc, hc = _gpu(inp, conv_weight=cw.to(DEV), conv_bias=cb.to(DEV))
    torch.cuda.synchronize()
    xc = oracle.default().causal_conv1d(gh.to_np(inp["x"]), gh.to_np(cw), gh.to_np(cb))
    conv_inp = dict(inp)
    conv_inp["x"] = torch.from_numpy(xc)
    yco, hco = _oracle(conv_inp)
    gh.compare(gh.to_np(yc), yco, gh.RTOL["f32"], "conv y")
    gh.compare(gh.to_np(hc), hco, gh.RTOL["f32"], "conv final state")


def test_wide_head_layer_sampled():
    """A Mamba-2-sized layer run through the selective scan: 2 × 2048 tokens,
    2048 channels (32 heads of 64), d_state 128, one A per channel; a channel
    sample against the oracle on those channels."""
    inp = _inputs(2, 2048, 2048, 128, "bf16", 6200, "per_channel")
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    y, hf = ss.selscan_fwd(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["z"],
                           d["delta_bias"], return_final_state=True)
    torch.cuda.synchronize()
    chans = list(wl.channel_subset(2048, 64))
    yo, ho = gh.oracle_fwd(inp, channels=chans)
    gh.compare(gh.to_np(y[:, :, chans]), yo, gh.RTOL["bf16"], "wide layer y")
    gh.compare(gh.to_np(hf[:, chans]), ho, gh.RTOL["bf16"], "wide layer state")


@pytest.mark.parametrize("N", [64, 256])
def test_wide_decode_steps(N):
    batch, dim, steps = 3, 50, 6
    inp = _inputs(batch, steps, dim, N, "f32", 6300 + N, "random")
    g = torch.Generator().manual_seed(6301)
    state = torch.randn(batch, dim, N, generator=g) * 0.1
    ref = gh.to_np(state)
    sd = state.to(DEV)
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    orc = oracle.default()
    n = gh.to_np
    for t in range(steps):
        tok = {k: d[k][:, t].contiguous() for k in ("x", "delta", "z", "B", "C")}
        y = ss.selscan_state_update(sd, tok["x"], tok["delta"], d["A"], tok["B"], tok["C"],
                                    d["D"], tok["z"], d["delta_bias"])
        yo, ref = orc.state_update(ref, n(inp["x"][:, t]), n(inp["delta"][:, t]), n(inp["A"]),
                                   n(inp["B"][:, t]), n(inp["C"][:, t]), n(inp["D"]),
                                   n(inp["z"][:, t]), n(inp["delta_bias"]))
        torch.cuda.synchronize()
        gh.compare(gh.to_np(y), yo, gh.RTOL["f32"], f"N={N} step {t} y")
        gh.compare(gh.to_np(sd), ref, gh.RTOL["f32"], f"N={N} step {t} state")
