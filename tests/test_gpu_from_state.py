"""GPU parity of selscan_fwd_from_state (the scan started from a given state)
against the oracle's scan with an initial state, in every launch plan, plus
continuation identities: a sequence split in two, the state advanced in place,
and decode steps followed by a scan."""
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
    "chunked3": dict(SELSCAN_PATH="chunked", SELSCAN_UNIT=None, SELSCAN_CHUNKS="3"),
}
SHAPES = [(1, 1, 128, 16), (2, 300, 136, 16), (1, 257, 256, 8), (3, 96, 40, 16)]


def _inputs(batch, L, dim, N, dtype, seed):
    w = wl.ScanWorkload("h0", batch, L, dim, N, dtype, gate=True, seed=seed)
    inp = wl.make_scan_inputs(w)
    g = torch.Generator().manual_seed(seed + 5)
    h0 = torch.randn(batch, dim, N, generator=g)
    return inp, h0


def _oracle(inp, h0):
    n = gh.to_np
    return oracle.default().fwd(n(inp["x"]), n(inp["delta"]), n(inp["A"]), n(inp["B"]),
                                n(inp["C"]), n(inp["D"]), n(inp["z"]), n(inp["delta_bias"]),
                                h0=n(h0))


def _gpu(inp, h0, final_state=None):
    d = {k: (None if v is None else v.to(DEV).contiguous()) for k, v in inp.items()}
    return ss.selscan_fwd(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["z"],
                          d["delta_bias"], initial_state=h0, final_state=final_state,
                          return_final_state=True)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", SHAPES, ids=str)
@pytest.mark.parametrize("path", list(PATHS))
def test_initial_state_every_plan(dtype, shape, path):
    batch, L, dim, N = shape
    inp, h0 = _inputs(batch, L, dim, N, dtype, seed=3000 + L + dim)
    with gh.env(**PATHS[path]):
        y, hf = _gpu(inp, h0.to(DEV))
        torch.cuda.synchronize()
    yo, ho = _oracle(inp, h0)
    gh.compare(gh.to_np(y), yo, gh.RTOL[dtype], f"{shape} {path} y")
    gh.compare(gh.to_np(hf), ho, gh.RTOL[dtype], f"{shape} {path} final state")
    assert ss.selscan_device_status() == 0


def test_split_sequence_continues():
    """Scanning tokens [0, L1) and then [L1, L) from the first call's final
    state gives the whole scan's outputs (both against the oracle)."""
    inp, _ = _inputs(2, 700, 256, 16, "bf16", seed=31)
    L1 = 333
    first = {k: (v[:, :L1] if v is not None and v.dim() == 3 and k not in ("A",) else v)
             for k, v in inp.items()}
    second = {k: (v[:, L1:] if v is not None and v.dim() == 3 and k not in ("A",) else v)
              for k, v in inp.items()}
    y1, h1 = _gpu(first, None)
    y2, h2 = _gpu(second, h1)
    torch.cuda.synchronize()
    yo, ho = _oracle(inp, None)
    gh.compare(np.concatenate([gh.to_np(y1), gh.to_np(y2)], axis=1), yo, gh.RTOL["bf16"],
               "split y")
    gh.compare(gh.to_np(h2), ho, gh.RTOL["bf16"], "split final state")


def test_state_advanced_in_place():
    inp, h0 = _inputs(2, 150, 136, 16, "f32", seed=32)
    state = h0.to(DEV).clone()
    y, hf = _gpu(inp, state, final_state=state)
    torch.cuda.synchronize()
    assert hf.data_ptr() == state.data_ptr()
    yo, ho = _oracle(inp, h0)
    gh.compare(gh.to_np(y), yo, gh.RTOL["f32"], "in-place y")
    gh.compare(gh.to_np(state), ho, gh.RTOL["f32"], "in-place state")


def test_no_tokens_copies_the_state():
    inp, h0 = _inputs(2, 0, 64, 16, "bf16", seed=33)
    y, hf = _gpu(inp, h0.to(DEV))
    torch.cuda.synchronize()
    assert y.numel() == 0 and torch.equal(hf.cpu(), h0)


def test_decode_steps_then_scan():
    """A state advanced by selscan_state_update for 5 tokens, then a scan of
    the next 200 tokens from it, equals the scan of all 205 tokens."""
    batch, dim, N, k, L = 2, 256, 16, 5, 200
    inp, _ = _inputs(batch, k + L, dim, N, "f32", seed=34)
    d = {kk: (None if v is None else v.to(DEV)) for kk, v in inp.items()}
    state = torch.zeros(batch, dim, N, device=DEV)
    ys = []
    for t in range(k):
        ys.append(ss.selscan_state_update(state, d["x"][:, t].contiguous(),
                                          d["delta"][:, t].contiguous(), d["A"],
                                          d["B"][:, t].contiguous(), d["C"][:, t].contiguous(),
                                          d["D"], d["z"][:, t].contiguous(), d["delta_bias"]))
    rest = {kk: (v[:, k:].contiguous() if v is not None and v.dim() == 3 else v)
            for kk, v in inp.items()}
    y2, hf = _gpu(rest, state)
    torch.cuda.synchronize()
    yo, ho = _oracle(inp, None)
    got = np.concatenate([np.stack([gh.to_np(v) for v in ys], axis=1), gh.to_np(y2)], axis=1)
    gh.compare(got, yo, gh.RTOL["f32"], "decode then scan y")
    gh.compare(gh.to_np(hf), ho, gh.RTOL["f32"], "decode then scan final state")
