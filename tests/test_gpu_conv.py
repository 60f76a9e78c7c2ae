"""GPU parity of selscan_fwd_conv (causal depthwise conv + SiLU fused in
front of the scan) against the oracle's conv followed by the oracle's scan,
in every launch plan, and continuation of a sequence across two calls."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_42_b200 as ss
from selective_state_space_42_b200 import workloads as wl

import gpu_helpers as gh

pytestmark = pytest.mark.gpu
DEV = "cuda"

PATHS = {
    "generic": dict(SELSCAN_PATH="generic", SELSCAN_UNIT=None, SELSCAN_CHUNKS=None),
    "generic_chunked": dict(SELSCAN_PATH="generic", SELSCAN_UNIT=None, SELSCAN_CHUNKS="3"),
    "seq_unit32": dict(SELSCAN_PATH="seq", SELSCAN_UNIT="32", SELSCAN_CHUNKS=None),
    "seq_default": dict(SELSCAN_PATH="seq", SELSCAN_UNIT=None, SELSCAN_CHUNKS=None),
    "chunked3": dict(SELSCAN_PATH="chunked", SELSCAN_UNIT=None, SELSCAN_CHUNKS="3"),
}
SHAPES = [(1, 1, 128, 16), (2, 300, 136, 16), (1, 257, 256, 8), (3, 96, 40, 16),
          (2, 70, 384, 16)]


def _inputs(batch, L, dim, N, dtype, K, seed, with_init=False):
    w = wl.ScanWorkload("conv", batch, L, dim, N, dtype, gate=True, seed=seed)
    inp = wl.make_scan_inputs(w)
    g = torch.Generator().manual_seed(seed + 9)
    conv = dict(w=torch.randn(dim, K, generator=g) * 0.5,
                b=torch.randn(dim, generator=g) * 0.1,
                init=(torch.randn(batch, dim, 3, generator=g).to(inp["x"].dtype).float()
                      if with_init else None))
    return inp, conv


def _oracle(inp, conv, h0=None, channels=None):
    """The oracle's conv (over the 3 initial tokens followed by x_in, first 3
    outputs dropped) and then the oracle's scan."""
    n = gh.to_np
    sel = slice(None) if channels is None else list(channels)
    x_in = n(inp["x"][:, :, sel])
    if conv["init"] is not None:
        init = np.transpose(n(conv["init"][:, sel]), (0, 2, 1))  # [batch, 3, dim]
        x_full = np.concatenate([init, x_in], axis=1)
    else:
        x_full = x_in
    orc = oracle.default()
    xc = orc.causal_conv1d(x_full, n(conv["w"][sel]), n(conv["b"][sel]), silu=True)
    if conv["init"] is not None:
        xc = xc[:, 3:]

    def bl(t):
        return None if t is None else n(t[:, :, sel])

    def ch(t):
        return None if t is None else n(t[sel])

    return orc.fwd(xc, bl(inp["delta"]), ch(inp["A"]), n(inp["B"]), n(inp["C"]), ch(inp["D"]),
                   bl(inp["z"]), ch(inp["delta_bias"]),
                   h0=None if h0 is None else n(h0[:, sel]))


def _gpu(inp, conv, h0=None):
    d = {k: (None if v is None else v.to(DEV).contiguous()) for k, v in inp.items()}
    c = {k: (None if v is None else v.to(DEV).contiguous()) for k, v in conv.items()}
    return ss.selscan_fwd(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["z"],
                          d["delta_bias"], initial_state=h0, conv_weight=c["w"],
                          conv_bias=c["b"], conv_init=c["init"], return_final_state=True)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", SHAPES, ids=str)
@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("K", [1, 4])
def test_conv_every_plan(dtype, shape, path, K):
    batch, L, dim, N = shape
    inp, conv = _inputs(batch, L, dim, N, dtype, K, seed=4000 + L + dim + K)
    with gh.env(**PATHS[path]):
        y, hf = _gpu(inp, conv)
        torch.cuda.synchronize()
    yo, ho = _oracle(inp, conv)
    gh.compare(gh.to_np(y), yo, gh.RTOL[dtype], f"{shape} {path} K={K} y")
    gh.compare(gh.to_np(hf), ho, gh.RTOL[dtype], f"{shape} {path} K={K} final state")
    assert ss.selscan_device_status() == 0


@pytest.mark.parametrize("K", [2, 3])
@pytest.mark.parametrize("path", ["generic", "seq_unit32", "chunked3"])
def test_conv_widths_with_init(K, path):
    inp, conv = _inputs(2, 200, 256, 16, "f32", K, seed=4100 + K, with_init=True)
    with gh.env(**PATHS[path]):
        y, hf = _gpu(inp, conv)
        torch.cuda.synchronize()
    yo, ho = _oracle(inp, conv)
    gh.compare(gh.to_np(y), yo, gh.RTOL["f32"], f"K={K} {path} y")
    gh.compare(gh.to_np(hf), ho, gh.RTOL["f32"], f"K={K} {path} final state")


def test_conv_sequence_continues_across_calls():
    """Tokens [0, L1) and then [L1, L) with the first call's final state as
    initial state and its last 3 conv inputs as conv_init equal one call over
    all L tokens."""
    inp, conv = _inputs(2, 500, 256, 16, "bf16", 4, seed=4200)
    L1 = 221

    def part(lo, hi):
        return {k: (v[:, lo:hi] if v is not None and v.dim() == 3 else v)
                for k, v in inp.items()}

    y1, h1 = _gpu(part(0, L1), conv)
    conv2 = dict(conv)
    conv2["init"] = inp["x"][:, L1 - 3:L1].float().permute(0, 2, 1).contiguous()
    y2, h2 = _gpu(part(L1, 500), conv2, h0=h1)
    torch.cuda.synchronize()
    yo, ho = _oracle(inp, conv)
    gh.compare(np.concatenate([gh.to_np(y1), gh.to_np(y2)], axis=1), yo, gh.RTOL["bf16"],
               "continued y")
    gh.compare(gh.to_np(h2), ho, gh.RTOL["bf16"], "continued final state")


def test_conv_bench_shape_sampled():
    """The Mamba-2.8B layer shape with a width-4 conv in front, in the launch
    plan the scan takes there; channels are independent, so a channel sample
    is checked against the oracle on those channels."""
    w = wl.WORKLOADS["mamba2p8b_layer"]
    inp = wl.make_scan_inputs(w, device=DEV)
    g = torch.Generator(device=DEV).manual_seed(77)
    conv = dict(w=torch.randn(w.dim, 4, generator=g, device=DEV) * 0.5,
                b=torch.randn(w.dim, generator=g, device=DEV) * 0.1, init=None)
    y, hf = _gpu(inp, conv)
    torch.cuda.synchronize()
    chans = wl.channel_subset(w.dim, 64)
    yo, ho = _oracle(inp, conv, channels=chans)
    gh.compare(gh.to_np(y[:, :, list(chans)]), yo, gh.RTOL["bf16"], "bench conv y")
    gh.compare(gh.to_np(hf[:, list(chans)]), ho, gh.RTOL["bf16"], "bench conv state")
    assert ss.selscan_device_status() == 0


@pytest.mark.parametrize("N", [16, 7])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_conv_trajectory(N, dtype):
    """Decode steps with the conv in front: y, the SSM state and the conv
    window after every step against the oracle's conv over the window and
    the tokens, followed by its recurrent step."""
    batch, dim, K, steps = 3, 70, 4, 12
    w = wl.ScanWorkload("dconv", batch, steps, dim, N, dtype, gate=True, seed=4300 + N)
    inp = wl.make_scan_inputs(w)
    g = torch.Generator().manual_seed(4301 + N)
    cw = torch.randn(dim, K, generator=g) * 0.5
    cb = torch.randn(dim, generator=g) * 0.1
    cs0 = torch.randn(batch, dim, 3, generator=g).to(inp["x"].dtype).float()
    h0 = torch.randn(batch, dim, N, generator=g) * 0.1
    if N != 16:
        inp["A"] = -torch.rand(dim, N, generator=g) * 4 - 0.1
    # oracle: conv over [window, tokens], then the recurrence step by step
    orc = oracle.default()
    n = gh.to_np
    x_full = np.concatenate([np.transpose(n(cs0), (0, 2, 1)), n(inp["x"])], axis=1)
    xc = orc.causal_conv1d(x_full, n(cw), n(cb), silu=True)[:, 3:]
    ref = n(h0)
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    state, cstate = h0.to(DEV).clone(), cs0.to(DEV).clone()
    cwd, cbd = cw.to(DEV), cb.to(DEV)
    for t in range(steps):
        tok = {k: d[k][:, t].contiguous() for k in ("x", "delta", "z", "B", "C")}
        y = ss.selscan_state_update(state, tok["x"], tok["delta"], d["A"], tok["B"], tok["C"],
                                    d["D"], tok["z"], d["delta_bias"], conv_state=cstate,
                                    conv_weight=cwd, conv_bias=cbd)
        yo, ref = orc.state_update(ref, xc[:, t], n(inp["delta"][:, t]), n(inp["A"]),
                                   n(inp["B"][:, t]), n(inp["C"][:, t]), n(inp["D"]),
                                   n(inp["z"][:, t]), n(inp["delta_bias"]))
        torch.cuda.synchronize()
        gh.compare(gh.to_np(y), yo, gh.RTOL[dtype], f"step {t} y")
        gh.compare(gh.to_np(state), ref, gh.RTOL[dtype], f"step {t} state")
        want_cs = x_full[:, t + 1:t + 4].transpose(0, 2, 1)
        assert np.array_equal(gh.to_np(cstate), want_cs), f"step {t} conv window"


def test_prefill_then_decode_with_conv():
    """selscan_fwd_conv over L tokens, then decode steps with the conv window
    taken from the last 3 inputs, equal selscan_fwd_conv over all tokens."""
    batch, dim, N, L, k = 2, 256, 16, 300, 6
    inp, conv = _inputs(batch, L + k, dim, N, "f32", 4, seed=4400)
    pre = {kk: (v[:, :L] if v is not None and v.dim() == 3 else v) for kk, v in inp.items()}
    _, hf = _gpu(pre, conv)
    state = hf.clone()
    cstate = inp["x"][:, L - 3:L].float().permute(0, 2, 1).contiguous().to(DEV)
    d = {kk: (None if v is None else v.to(DEV)) for kk, v in inp.items()}
    ys = []
    for t in range(L, L + k):
        tok = {kk: d[kk][:, t].contiguous() for kk in ("x", "delta", "z", "B", "C")}
        ys.append(ss.selscan_state_update(state, tok["x"], tok["delta"], d["A"], tok["B"],
                                          tok["C"], d["D"], tok["z"], d["delta_bias"],
                                          conv_state=cstate, conv_weight=conv["w"].to(DEV),
                                          conv_bias=conv["b"].to(DEV)))
    torch.cuda.synchronize()
    yo, ho = _oracle(inp, conv)
    got = np.stack([gh.to_np(v) for v in ys], axis=1)
    gh.compare(got, yo[:, L:], gh.RTOL["f32"], "decode after prefill y")
    gh.compare(gh.to_np(state), ho, gh.RTOL["f32"], "decode after prefill state")
