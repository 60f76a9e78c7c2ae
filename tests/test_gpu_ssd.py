"""GPU parity of selscan_ssd_fwd (the scan with one scalar A per head, in
chunked matrix form) against the oracle's scan with the heads' Δ, A, D and
bias broadcast to their channels."""
import numpy as np
import pytest
import torch

import oracle
import selective_state_space_42_b200 as ss
from selective_state_space_42_b200 import workloads as wl

import gpu_helpers as gh

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(batch, L, H, P, N, dtype, seed, gate=True):
    g = torch.Generator().manual_seed(seed)
    dt_ = wl.DTYPES[dtype]
    D = H * P
    inp = dict(
        x=torch.randn(batch, L, D, generator=g).to(dt_),
        dt=(0.5 * torch.randn(batch, L, H, generator=g)).to(dt_),
        z=torch.randn(batch, L, D, generator=g).to(dt_) if gate else None,
        B=torch.randn(batch, L, N, generator=g).to(dt_),
        C=torch.randn(batch, L, N, generator=g).to(dt_),
        A=-(torch.rand(H, generator=g) * 3.5 + 0.5),
        Dh=1.0 + 0.1 * torch.randn(H, generator=g),
        dt_bias=torch.log(torch.expm1(1e-3 + (1e-1 - 1e-3) * torch.rand(H, generator=g,
                                                                         dtype=torch.float64))
                          ).float(),
    )
    return inp


def _oracle(inp, P, h0=None):
    n = gh.to_np
    H = inp["A"].shape[0]
    N = inp["B"].shape[2]
    rep = lambda v: np.repeat(n(v), P, axis=-1)  # noqa: E731  heads -> channels
    A_full = np.repeat(n(inp["A"])[:, None], P, axis=0).repeat(N, axis=1)
    return oracle.default().fwd(n(inp["x"]), rep(inp["dt"]), A_full, n(inp["B"]), n(inp["C"]),
                                rep(inp["Dh"]), None if inp["z"] is None else n(inp["z"]),
                                rep(inp["dt_bias"]), h0=None if h0 is None else n(h0))


def _gpu(inp, h0=None):
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    return ss.selscan_ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], D=d["Dh"], z=d["z"],
                              dt_bias=d["dt_bias"], initial_state=h0,
                              return_final_state=True)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(1, 1, 1, 1, 1), (2, 100, 3, 64, 16), (1, 200, 2, 64, 128),
                                   (2, 65, 4, 32, 64), (1, 1000, 2, 64, 64),
                                   (1, 130, 5, 7, 33)], ids=str)
def test_ssd_matches_scan(dtype, shape):
    batch, L, H, P, N = shape
    inp = _inputs(batch, L, H, P, N, dtype, seed=7000 + L + H + N)
    y, hf = _gpu(inp)
    torch.cuda.synchronize()
    yo, ho = _oracle(inp, P)
    gh.compare(gh.to_np(y), yo, gh.RTOL[dtype], f"{shape} y")
    gh.compare(gh.to_np(hf), ho, gh.RTOL[dtype], f"{shape} final state")


def test_ssd_initial_state_and_no_gate():
    inp = _inputs(2, 300, 3, 64, 64, "f32", seed=7100, gate=False)
    g = torch.Generator().manual_seed(7101)
    h0 = torch.randn(2, 3 * 64, 64, generator=g)
    y, hf = _gpu(inp, h0.to(DEV))
    torch.cuda.synchronize()
    yo, ho = _oracle(inp, 64, h0)
    gh.compare(gh.to_np(y), yo, gh.RTOL["f32"], "h0 y")
    gh.compare(gh.to_np(hf), ho, gh.RTOL["f32"], "h0 final state")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_ssd_long_sequence_from_a_state(dtype):
    """More chunks than the carry stages its decays for at a time (258 chunks
    of 128 tokens), from an initial state."""
    H, P, N = 2, 16, 16
    inp = _inputs(1, 33000, H, P, N, dtype, seed=7150)
    g = torch.Generator().manual_seed(7151)
    h0 = torch.randn(1, H * P, N, generator=g)
    y, hf = _gpu(inp, h0.to(DEV))
    torch.cuda.synchronize()
    yo, ho = _oracle(inp, P, h0)
    gh.compare(gh.to_np(y), yo, gh.RTOL[dtype], "long y")
    gh.compare(gh.to_np(hf), ho, gh.RTOL[dtype], "long final state")


@pytest.mark.parametrize("L,H", [(2048, 32), (4096, 37)], ids=["32-heads", "37-heads"])
def test_ssd_equals_wide_scan_on_a_head_layer(L, H):
    """A Mamba-2-sized layer (2 × L tokens, H heads of 64, d_state 128): the
    chunked form against the recurrence of the wide-state scan kernel with
    the same inputs broadcast to channels, and a channel sample against the
    oracle. The state kernel groups 4 heads per CTA for the first shape and
    3 for the second, whose last group holds one head."""
    inp = _inputs(2, L, H, 64, 128, "bf16", seed=7200 + H)
    y, hf = _gpu(inp)
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    rep = lambda v: v.repeat_interleave(64, dim=-1).contiguous()  # noqa: E731
    A_full = d["A"].repeat_interleave(64)[:, None].repeat(1, 128).contiguous()
    yw, hw = ss.selscan_fwd(d["x"], rep(d["dt"]), A_full, d["B"], d["C"], rep(d["Dh"]), d["z"],
                            rep(d["dt_bias"]), return_final_state=True)
    torch.cuda.synchronize()
    gh.compare(gh.to_np(y), gh.to_np(yw), 2e-2, "ssd vs recurrence y")
    gh.compare(gh.to_np(hf), gh.to_np(hw), 2e-2, "ssd vs recurrence state")
    chans = list(wl.channel_subset(H * 64, 64))
    n = gh.to_np
    heads = [c // 64 for c in chans]
    A_s = np.repeat(n(inp["A"])[heads][:, None], 128, axis=1)
    yo, ho = oracle.default().fwd(n(inp["x"][:, :, chans]), n(inp["dt"][:, :, heads]), A_s,
                                  n(inp["B"]), n(inp["C"]), n(inp["Dh"])[heads],
                                  n(inp["z"][:, :, chans]), n(inp["dt_bias"])[heads])
    gh.compare(gh.to_np(y[:, :, chans]), yo, gh.RTOL["bf16"], "ssd layer y")
    gh.compare(gh.to_np(hf[:, chans]), ho, gh.RTOL["bf16"], "ssd layer state")


def _misaligned(t):
    """A copy of t whose data starts one element past a 16-byte boundary."""
    buf = torch.empty(t.numel() + 8, dtype=t.dtype, device=t.device)
    out = buf[1:1 + t.numel()].view(t.shape)
    out.copy_(t)
    return out


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_ssd_options(dtype):
    """Initial state without the gate, softplus off (positive Δ), no D and no
    dt_bias, on 3 chunks of the bf16 path (2 of 64 + 1 of the f32 path)."""
    inp = _inputs(2, 300, 3, 64, 128, dtype, seed=7300, gate=False)
    g = torch.Generator().manual_seed(7301)
    h0 = torch.randn(2, 3 * 64, 128, generator=g) * 0.3
    y, hf = _gpu(inp, h0.to(DEV))
    torch.cuda.synchronize()
    yo, ho = _oracle(inp, 64, h0)
    gh.compare(gh.to_np(y), yo, gh.RTOL[dtype], "h0 no gate y")
    gh.compare(gh.to_np(hf), ho, gh.RTOL[dtype], "h0 no gate final state")

    inp2 = dict(inp)
    inp2["dt"] = (inp["dt"].float().abs() * 0.2 + 0.01).to(inp["dt"].dtype)
    inp2["Dh"] = torch.zeros_like(inp["Dh"])
    inp2["dt_bias"] = torch.zeros_like(inp["dt_bias"])
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp2.items()}
    y2, h2 = ss.selscan_ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], softplus=False,
                                return_final_state=True)
    torch.cuda.synchronize()
    n = gh.to_np
    A_full = np.repeat(n(inp2["A"])[:, None], 64, axis=0).repeat(128, axis=1)
    yo2, ho2 = oracle.default().fwd(n(inp2["x"]), np.repeat(n(inp2["dt"]), 64, axis=-1),
                                    A_full, n(inp2["B"]), n(inp2["C"]), None, None, None,
                                    softplus=False)
    gh.compare(gh.to_np(y2), yo2, gh.RTOL[dtype], "no softplus, D, bias y")
    gh.compare(gh.to_np(h2), ho2, gh.RTOL[dtype], "no softplus, D, bias final state")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_ssd_steep_decay_heads(dtype):
    """Heads whose decay over a 128-token chunk leaves the float32 range of
    2^(Acum_i − Acum_j) factored as 2^Acum_i · 2^(−Acum_j) (|A|·Δ large) next
    to heads where it does not: the per-element decay path and the factored
    one in the same calls, with an initial state so that C·h_in counts."""
    inp = _inputs(2, 300, 5, 64, 128, dtype, seed=7700)
    inp["A"] = torch.tensor([-0.5, -30.0, -1.0, -40.0, -12.0])
    inp["dt_bias"] = torch.zeros(5)
    g = torch.Generator().manual_seed(7701)
    h0 = torch.randn(2, 5 * 64, 128, generator=g) * 0.3
    y, hf = _gpu(inp, h0.to(DEV))
    torch.cuda.synchronize()
    yo, ho = _oracle(inp, 64, h0)
    gh.compare(gh.to_np(y), yo, gh.RTOL[dtype], "steep decay y")
    gh.compare(gh.to_np(hf), ho, gh.RTOL[dtype], "steep decay final state")


@pytest.mark.parametrize("L", [127, 128, 129, 256, 257])
def test_ssd_chunk_edges(L):
    """Sequence lengths at the 128-token chunk edges of the tensor-core path
    (and 64-token edges of the float32 one)."""
    for dtype in ("bf16", "f32"):
        inp = _inputs(1, L, 2, 64, 64, dtype, seed=7400 + L)
        y, hf = _gpu(inp)
        torch.cuda.synchronize()
        yo, ho = _oracle(inp, 64)
        gh.compare(gh.to_np(y), yo, gh.RTOL[dtype], f"L={L} {dtype} y")
        gh.compare(gh.to_np(hf), ho, gh.RTOL[dtype], f"L={L} {dtype} final state")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_ssd_misaligned_rows(dtype):
    """x, z, y, B and C one element off a 16-byte boundary: the element-wise
    staging and store paths instead of the 16-byte copies."""
    inp = _inputs(2, 150, 2, 64, 32, dtype, seed=7500)
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    for k in ("x", "z", "B", "C"):
        d[k] = _misaligned(d[k])
    y = _misaligned(torch.zeros_like(d["x"]))
    _, hf = ss.selscan_ssd_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], D=d["Dh"], z=d["z"],
                               dt_bias=d["dt_bias"], y=y, return_final_state=True)
    torch.cuda.synchronize()
    yo, ho = _oracle(inp, 64)
    gh.compare(gh.to_np(y), yo, gh.RTOL[dtype], "misaligned y")
    gh.compare(gh.to_np(hf), ho, gh.RTOL[dtype], "misaligned final state")


def test_ssd_rejects_unsupported_sizes():
    x = torch.zeros(1, 4, 2 * 65, device=DEV, dtype=torch.bfloat16)
    dt = torch.zeros(1, 4, 2, device=DEV, dtype=torch.bfloat16)
    A = -torch.ones(2, device=DEV)
    B = torch.zeros(1, 4, 16, device=DEV, dtype=torch.bfloat16)
    with pytest.raises(ss.SelscanError):
        ss.selscan_ssd_fwd(x, dt, A, B, B)  # headdim 65
    x = torch.zeros(1, 4, 2 * 64, device=DEV, dtype=torch.bfloat16)
    B = torch.zeros(1, 4, 129, device=DEV, dtype=torch.bfloat16)
    with pytest.raises(ss.SelscanError):
        ss.selscan_ssd_fwd(x, dt, A, B, B)  # d_state 129
    assert ss.selscan_device_status() == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_ssd_matches_matrix_form(dtype):
    """Against the semiseparable matrix form written out in float64 (the
    dense (L ◦ S)·diag(Δ)·x per head), with an initial state, 2 batch rows
    and 3 chunks of the tensor-core path."""
    from oracle import ssd_matrix
    inp = _inputs(2, 300, 3, 64, 128, dtype, seed=7600)
    g = torch.Generator().manual_seed(7601)
    h0 = torch.randn(2, 3 * 64, 128, generator=g) * 0.3
    y, hf = _gpu(inp, h0.to(DEV))
    torch.cuda.synchronize()
    n = gh.to_np
    yo, ho = ssd_matrix.ssd_matrix_form(n(inp["x"]), n(inp["dt"]), n(inp["A"]), n(inp["B"]),
                                        n(inp["C"]), n(inp["Dh"]), n(inp["z"]),
                                        n(inp["dt_bias"]), h0=n(h0))
    gh.compare(gh.to_np(y), yo, gh.RTOL[dtype], "matrix form y")
    gh.compare(gh.to_np(hf), ho, gh.RTOL[dtype], "matrix form final state")
