"""GPU parity of selscan_bwd (the gradient of the scan) against the float64
oracle's reverse sweep, through the C ABI."""
import pytest
import torch

import oracle
import selective_state_space_42_b200 as ss
from selective_state_space_42_b200 import workloads as wl

import gpu_helpers as gh

pytestmark = pytest.mark.gpu
DEV = "cuda"

GRADS = ("dx", "ddelta", "dz", "dA", "dB", "dC", "dD", "ddelta_bias")


def _inputs(batch, L, dim, N, dtype, gate, seed, structured=True, dfinal=True):
    w = wl.ScanWorkload("bwd", batch, L, dim, N, dtype, gate=gate, seed=seed)
    inp = wl.make_scan_inputs(w)
    if not structured:
        g = torch.Generator().manual_seed(seed + 1)
        inp["A"] = -torch.rand(dim, N, generator=g) * 4 - 0.1
    g = torch.Generator().manual_seed(seed + 2)
    dy = torch.randn(batch, L, dim, generator=g).to(inp["x"].dtype)
    df = torch.randn(batch, dim, N, generator=g) if dfinal else None
    return inp, dy, df


def _gpu_bwd(inp, dy, df, softplus=True):
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    return ss.selscan_bwd(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["z"],
                          d["delta_bias"], softplus=softplus, dy=dy.to(DEV),
                          dfinal_state=None if df is None else df.to(DEV))


def _oracle_bwd(inp, dy, df, softplus=True, channels=None):
    sel = slice(None) if channels is None else list(channels)

    def bl(t):
        return None if t is None else gh.to_np(t[:, :, sel])

    def ch(t):
        return None if t is None else gh.to_np(t[sel])

    return oracle.default().bwd(
        bl(inp["x"]), bl(inp["delta"]), ch(inp["A"]), gh.to_np(inp["B"]), gh.to_np(inp["C"]),
        ch(inp["D"]), bl(inp["z"]), ch(inp["delta_bias"]), softplus=softplus, dy=bl(dy),
        dfinal=None if df is None else gh.to_np(df[:, sel]))


def _compare_all(g, o, dtype, what, names=GRADS):
    rtol = gh.RTOL[dtype]
    for k in names:
        if o.get(k) is None:
            assert g.get(k) is None, f"{what}: {k} should be absent"
            continue
        gh.compare(gh.to_np(g[k]), o[k], rtol, f"{what} {k}")


SHAPES = [(1, 1, 1, 1), (2, 31, 33, 16), (1, 40, 64, 16), (3, 17, 5, 4), (2, 50, 70, 7),
          (1, 300, 40, 16), (2, 16, 32, 16), (1, 257, 96, 8)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", SHAPES, ids=str)
@pytest.mark.parametrize("gate", [True, False])
def test_small_every_element(dtype, shape, gate):
    batch, L, dim, N = shape
    inp, dy, df = _inputs(batch, L, dim, N, dtype, gate, seed=100 + L + dim)
    g = _gpu_bwd(inp, dy, df)
    torch.cuda.synchronize()
    _compare_all(g, _oracle_bwd(inp, dy, df), dtype, f"{shape}")


# Shapes whose rows are whole 16-byte chunks in both dtypes, so the two-lane
# kernel takes them: ragged last tiles, channel tiles with one warp partly or
# wholly past the channels, fewer than 16 states.
PAIR_SHAPES = [(2, 37, 48, 16), (2, 61, 24, 16), (1, 46, 40, 4), (3, 9, 8, 8), (1, 8, 64, 16)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", PAIR_SHAPES, ids=str)
@pytest.mark.parametrize("gate", [True, False])
@pytest.mark.parametrize("structured", [True, False])
def test_chunked_rows_every_element(dtype, shape, gate, structured):
    inp, dy, df = _inputs(*shape, dtype, gate, seed=41, structured=structured)
    g = _gpu_bwd(inp, dy, df)
    torch.cuda.synchronize()
    _compare_all(g, _oracle_bwd(inp, dy, df), dtype,
                 f"{shape} {dtype} gate={gate} structured={structured}")


@pytest.mark.parametrize("structured", [True, False])
@pytest.mark.parametrize("softplus", [True, False])
def test_variants(structured, softplus):
    inp, dy, df = _inputs(2, 100, 48, 16, "f32", True, seed=7, structured=structured,
                          dfinal=not softplus)
    if not softplus:  # Δ = delta + bias itself: keep it positive
        inp["delta"] = inp["delta"].abs() + 0.05
        inp["delta_bias"] = torch.full_like(inp["delta_bias"], 0.01)
    g = _gpu_bwd(inp, dy, df, softplus=softplus)
    torch.cuda.synchronize()
    _compare_all(g, _oracle_bwd(inp, dy, df, softplus=softplus), "f32",
                 f"structured={structured} softplus={softplus}")


def test_medium_130m_shape():
    """A Mamba-130M-shaped layer cut to 2 × 512 tokens × 1536 channels, every
    element of every gradient."""
    inp, dy, df = _inputs(2, 512, 1536, 16, "bf16", True, seed=11)
    g = _gpu_bwd(inp, dy, df)
    torch.cuda.synchronize()
    _compare_all(g, _oracle_bwd(inp, dy, df), "bf16", "130m-shaped")


@pytest.mark.parametrize("dim", [100, 96])
def test_deterministic(dim):
    inp, dy, df = _inputs(2, 200, dim, 16, "bf16", True, seed=12)
    g1 = _gpu_bwd(inp, dy, df)
    g2 = _gpu_bwd(inp, dy, df)
    torch.cuda.synchronize()
    for k in GRADS:
        assert torch.equal(g1[k], g2[k]), k


def test_empty_and_degenerate():
    # no tokens: float32 gradients are zero, token gradients empty
    inp, dy, df = _inputs(2, 0, 8, 16, "bf16", True, seed=13)
    g = _gpu_bwd(inp, dy, df)
    torch.cuda.synchronize()
    for k in ("dA", "dD", "ddelta_bias"):
        assert torch.count_nonzero(g[k]) == 0, k
    assert g["dx"].numel() == 0 and g["dB"].numel() == 0
    # no channels: dB and dC are zero
    w = wl.ScanWorkload("nodim", 2, 5, 0, 16, "bf16", gate=True, seed=14)
    inp = wl.make_scan_inputs(w)
    dy = torch.zeros(2, 5, 0, dtype=torch.bfloat16)
    g = _gpu_bwd(inp, dy, None)
    torch.cuda.synchronize()
    assert g["dB"].shape == (2, 5, 16) and torch.count_nonzero(g["dB"]) == 0
    assert torch.count_nonzero(g["dC"]) == 0


def test_bench_shape_sampled_and_identities():
    """The Mamba-2.8B-shaped layer (4 × 8192 × 5120, N = 16, bf16, gated):
    per-channel gradients on a channel sample against the oracle on those
    channels (channels are independent chains), and the channel sums dB, dC
    through identities that hold at any size:
        Σ dC·C = Σ dy·(y − D·x·silu(z)),   Σ dB·B = Σ dC·C + Σ dfinal·h_final
    (h0 = 0; y and h_final from the GPU forward)."""
    w = wl.WORKLOADS["mamba2p8b_layer"]
    inp = wl.make_scan_inputs(w, device=DEV)
    g = torch.Generator(device=DEV).manual_seed(99)
    dy = torch.randn(w.batch, w.seqlen, w.dim, generator=g, device=DEV).to(torch.bfloat16)
    df = torch.randn(w.batch, w.dim, w.dstate, generator=g, device=DEV)
    grads = ss.selscan_bwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                           inp["z"], inp["delta_bias"], dy=dy, dfinal_state=df)
    y, hf = ss.selscan_fwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                           inp["z"], inp["delta_bias"], return_final_state=True)
    torch.cuda.synchronize()
    chans = wl.channel_subset(w.dim, 64)
    o = _oracle_bwd(inp, dy, df, channels=chans)
    sel = list(chans)
    for k in ("dx", "ddelta", "dz"):
        gh.compare(gh.to_np(grads[k][:, :, sel]), o[k], gh.RTOL["bf16"], f"bench {k}")
    for k in ("dA", "dD", "ddelta_bias"):
        gh.compare(gh.to_np(grads[k][sel]), o[k], gh.RTOL["bf16"], f"bench {k}")
    f64 = torch.float64
    x, z = inp["x"].to(f64), inp["z"].to(f64)
    ylin = y.to(f64) - inp["D"].to(f64) * x * (z * torch.sigmoid(z))
    lhs_c = float((grads["dC"].to(f64) * inp["C"].to(f64)).sum())
    rhs_c = float((dy.to(f64) * ylin).sum())
    assert abs(lhs_c - rhs_c) <= 2e-2 * (abs(rhs_c) + float((dy.to(f64) * ylin).abs().sum()) / 1e3), \
        (lhs_c, rhs_c)
    lhs_b = float((grads["dB"].to(f64) * inp["B"].to(f64)).sum())
    rhs_b = lhs_c + float((df.to(f64) * hf.to(f64)).sum())
    assert abs(lhs_b - rhs_b) <= 1e-3 * (abs(rhs_b) + abs(lhs_c)), (lhs_b, rhs_b)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("structured", [True, False])
def test_checkpoints_from_the_forward_kernel(dtype, structured, monkeypatch):
    """The checkpoints written by the TMA-staged forward kernel (its one-pass
    plan forced on a small shape, ragged last tile, with an initial state)
    against the oracle, and against the gradient kernel's own forward sweep."""
    inp, dy, df = _inputs(2, 301, 256, 16, dtype, True, seed=51, structured=structured)
    g = torch.Generator().manual_seed(52)
    h0 = torch.randn(2, 256, 16, generator=g)
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}

    def run():
        return ss.selscan_bwd(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["z"],
                              d["delta_bias"], dy=dy.to(DEV), dfinal_state=df.to(DEV),
                              initial_state=h0.to(DEV))

    monkeypatch.setenv("SELSCAN_PATH", "seq")
    assert ss.selscan_fwd_plan(2, 301, 256, 16)["launches"] == 1  # the one-pass plan
    got = run()
    monkeypatch.setenv("SELSCAN_BWD_OWN_SWEEP", "1")
    own = run()
    torch.cuda.synchronize()
    n = gh.to_np
    o = oracle.default().bwd(n(inp["x"]), n(inp["delta"]), n(inp["A"]), n(inp["B"]), n(inp["C"]),
                             n(inp["D"]), n(inp["z"]), n(inp["delta_bias"]), h0=n(h0), dy=n(dy),
                             dfinal=n(df))
    _compare_all(got, o, dtype, "forward-kernel checkpoints", names=GRADS + ("dh0",))
    _compare_all(own, o, dtype, "own forward sweep", names=GRADS + ("dh0",))


def test_long_sequence_sampled():
    """The 1M-token layer (1 × 1,048,576 × 2048, N = 16, bf16, gated): 131,072
    8-token tiles per chain, checkpoint and partial buffers of several GB;
    per-channel gradients on a channel sample against the oracle."""
    w = wl.WORKLOADS["long_1m"]
    inp = wl.make_scan_inputs(w, device=DEV)
    g = torch.Generator(device=DEV).manual_seed(98)
    dy = torch.randn(w.batch, w.seqlen, w.dim, generator=g, device=DEV).to(torch.bfloat16)
    df = torch.randn(w.batch, w.dim, w.dstate, generator=g, device=DEV)
    grads = ss.selscan_bwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                           inp["z"], inp["delta_bias"], dy=dy, dfinal_state=df)
    torch.cuda.synchronize()
    assert ss.selscan_device_status() == 0
    chans = wl.channel_subset(w.dim, 256)
    o = _oracle_bwd(inp, dy, df, channels=chans)
    sel = list(chans)
    for k in ("dx", "ddelta", "dz"):
        gh.compare(gh.to_np(grads[k][:, :, sel]), o[k], gh.RTOL["bf16"], f"long {k}")
    for k in ("dA", "dD", "ddelta_bias"):
        gh.compare(gh.to_np(grads[k][sel]), o[k], gh.RTOL["bf16"], f"long {k}")
    for k in ("dB", "dC"):
        assert torch.isfinite(grads[k]).all(), k


@pytest.mark.parametrize("shape,path", [((2, 77, 70), None), ((2, 301, 256), "seq")],
                         ids=["own-sweep", "forward-kernel-checkpoints"])
def test_library_allocated_workspace_matches(shape, path, monkeypatch):
    """selscan_bwd (workspace allocated on the stream by the library) and
    selscan_bwd_workspace (torch-allocated workspace) give identical results,
    also where the workspace holds the forward kernel's checkpoint-pass
    region (one-pass plan forced)."""
    if path:
        monkeypatch.setenv("SELSCAN_PATH", path)
    inp, dy, df = _inputs(*shape, 16, "bf16", True, seed=15)
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    args = (d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["z"], d["delta_bias"])
    g1 = ss.selscan_bwd(*args, dy=dy.to(DEV), dfinal_state=df.to(DEV))
    g2 = ss.selscan_bwd(*args, dy=dy.to(DEV), dfinal_state=df.to(DEV),
                        allocate_in_library=True)
    torch.cuda.synchronize()
    for k in GRADS:
        assert torch.equal(g1[k], g2[k]), k


def test_workspace_too_small_is_rejected():
    inp, dy, _ = _inputs(1, 20, 40, 16, "bf16", False, seed=16)
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    lib = ss.load_library()
    need = ss.selscan_bwd_workspace_bytes(1, 20, 40, 16)
    ws = torch.empty(need, device=DEV, dtype=torch.uint8)
    outs = [torch.empty_like(d["x"]), torch.empty_like(d["x"]),
            torch.empty(40, 16, device=DEV), torch.empty(1, 20, 16, device=DEV),
            torch.empty(1, 20, 16, device=DEV)]
    st = lib.selscan_bwd_workspace(
        d["x"].data_ptr(), d["delta"].data_ptr(), d["A"].data_ptr(), d["B"].data_ptr(),
        d["C"].data_ptr(), None, None, None, 1, dy.to(DEV).data_ptr(), None,
        outs[0].data_ptr(), outs[1].data_ptr(), outs[2].data_ptr(), outs[3].data_ptr(),
        outs[4].data_ptr(), None, None, None, 1, 20, 40, 16, 1, ws.data_ptr(), need - 1,
        None)
    assert st == -8


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dim", [70, 48])
def test_initial_state_gradient(dtype, dim):
    """The gradient of the scan started from a given state: every gradient,
    the initial state's included, against the oracle (70 channels: rows that
    are not whole 16-byte chunks; 48: the two-lane kernel)."""
    inp, dy, df = _inputs(2, 90, dim, 16, dtype, True, seed=17)
    g = torch.Generator().manual_seed(18)
    h0 = torch.randn(2, dim, 16, generator=g)
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    got = ss.selscan_bwd(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["z"],
                         d["delta_bias"], dy=dy.to(DEV), dfinal_state=df.to(DEV),
                         initial_state=h0.to(DEV))
    torch.cuda.synchronize()
    n = gh.to_np
    o = oracle.default().bwd(n(inp["x"]), n(inp["delta"]), n(inp["A"]), n(inp["B"]),
                             n(inp["C"]), n(inp["D"]), n(inp["z"]), n(inp["delta_bias"]),
                             h0=n(h0), dy=n(dy), dfinal=n(df))
    _compare_all(got, o, dtype, "from state", names=GRADS + ("dh0",))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("K", [4, 2])
@pytest.mark.parametrize("shape", [(2, 90, 70), (1, 1100, 40)], ids=str)
def test_conv_gradient(dtype, K, shape):
    """The gradient through the causal conv + SiLU in front of the scan
    (selscan_bwd_conv) against the oracle's scan gradient at the conv output
    followed by its conv gradient."""
    batch, L, dim = shape
    inp, dy, df = _inputs(batch, L, dim, 16, dtype, True, seed=19 + K)
    g = torch.Generator().manual_seed(20 + K)
    cw = torch.randn(dim, K, generator=g) * 0.5
    cb = torch.randn(dim, generator=g) * 0.1
    h0 = torch.randn(batch, dim, 16, generator=g)
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    got = ss.selscan_bwd(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["z"],
                         d["delta_bias"], dy=dy.to(DEV), dfinal_state=df.to(DEV),
                         initial_state=h0.to(DEV), conv_weight=cw.to(DEV),
                         conv_bias=cb.to(DEV))
    torch.cuda.synchronize()
    n = gh.to_np
    orc = oracle.default()
    xc = orc.causal_conv1d(n(inp["x"]), n(cw), n(cb))
    o = orc.bwd(xc, n(inp["delta"]), n(inp["A"]), n(inp["B"]), n(inp["C"]), n(inp["D"]),
                n(inp["z"]), n(inp["delta_bias"]), h0=n(h0), dy=n(dy), dfinal=n(df))
    dx_in, dw, dcb = orc.causal_conv1d_bwd(n(inp["x"]), n(cw), n(cb), o["dx"])
    o.update(dx=dx_in, dconv_weight=dw, dconv_bias=dcb)
    _compare_all(got, o, dtype, f"conv K={K}",
                 names=GRADS + ("dh0", "dconv_weight", "dconv_bias"))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("structured", [True, False])
@pytest.mark.parametrize("shape", [(2, 37, 40, 16), (1, 130, 33, 7)], ids=str)
def test_zoh_gradient(dtype, structured, shape):
    """The gradient of the ZOH input term (C ABI selscan_bwd_ex) against the
    oracle's, every element; one A entry of 0 exercises the c → Δ limit."""
    batch, L, dim, N = shape
    inp, dy, df = _inputs(batch, L, dim, N, dtype, True, seed=900 + L, structured=structured)
    if not structured:
        inp["A"][3, 1] = 0.0
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    g = ss.selscan_bwd(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["z"],
                       d["delta_bias"], dy=dy.to(DEV), dfinal_state=df.to(DEV), bbar="zoh")
    torch.cuda.synchronize()
    n = gh.to_np
    o = oracle.default().bwd(n(inp["x"]), n(inp["delta"]), n(inp["A"]), n(inp["B"]),
                             n(inp["C"]), n(inp["D"]), n(inp["z"]), n(inp["delta_bias"]),
                             dy=n(dy), dfinal=n(df), bbar=oracle.BBAR_ZOH)
    _compare_all(g, o, dtype, f"zoh {shape}")


def test_zoh_gradient_with_state_and_conv():
    """ZOH together with the initial state and the conv front end."""
    inp, dy, df = _inputs(2, 45, 24, 16, "f32", True, seed=950, structured=False)
    g0 = torch.Generator().manual_seed(951)
    h0 = torch.randn(2, 24, 16, generator=g0) * 0.3
    cw = torch.randn(24, 4, generator=g0) * 0.5
    cb = torch.randn(24, generator=g0) * 0.1
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    g = ss.selscan_bwd(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["z"],
                       d["delta_bias"], dy=dy.to(DEV), dfinal_state=df.to(DEV),
                       initial_state=h0.to(DEV), conv_weight=cw.to(DEV), conv_bias=cb.to(DEV),
                       bbar="zoh")
    torch.cuda.synchronize()
    n = gh.to_np
    orc = oracle.default()
    xc = orc.causal_conv1d(n(inp["x"]), n(cw), n(cb))
    o = orc.bwd(xc, n(inp["delta"]), n(inp["A"]), n(inp["B"]), n(inp["C"]), n(inp["D"]),
                n(inp["z"]), n(inp["delta_bias"]), h0=n(h0), dy=n(dy), dfinal=n(df),
                bbar=oracle.BBAR_ZOH)
    for k in ("ddelta", "dz", "dA", "dB", "dC", "dD", "ddelta_bias", "dh0"):
        gh.compare(gh.to_np(g[k]), o[k], gh.RTOL["f32"], f"zoh+conv {k}")
    # dx is w.r.t. the conv's input: the oracle's conv backward of the scan's dx
    dxin, dw, dcb = orc.causal_conv1d_bwd(n(inp["x"]), n(cw), n(cb), o["dx"])
    gh.compare(gh.to_np(g["dx"]), dxin, gh.RTOL["f32"], "zoh+conv dx_in")
    gh.compare(gh.to_np(g["dconv_weight"]), dw, gh.RTOL["f32"], "zoh+conv dconv_weight")
    gh.compare(gh.to_np(g["dconv_bias"]), dcb, gh.RTOL["f32"], "zoh+conv dconv_bias")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [17, 32, 64, 100, 256])
@pytest.mark.parametrize("structured", [True, False])
def test_wide_state_gradient(dtype, N, structured):
    """d_state above 16: the chains are walked once per group of 16 states and
    the per-token sums over the groups carried in float32; every element
    against the oracle (which takes any d_state)."""
    inp, dy, df = _inputs(2, 37, 40, N, dtype, True, seed=1100 + N, structured=structured)
    g = _gpu_bwd(inp, dy, df)
    torch.cuda.synchronize()
    _compare_all(g, _oracle_bwd(inp, dy, df), dtype, f"N={N}")


def test_wide_state_gradient_with_options():
    """d_state 48 with the initial state, the conv front end and the ZOH term."""
    N = 48
    inp, dy, df = _inputs(2, 45, 24, N, "f32", True, seed=1200, structured=False)
    g0 = torch.Generator().manual_seed(1201)
    h0 = torch.randn(2, 24, N, generator=g0) * 0.3
    cw = torch.randn(24, 4, generator=g0) * 0.5
    cb = torch.randn(24, generator=g0) * 0.1
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    n = gh.to_np
    orc = oracle.default()
    xc = orc.causal_conv1d(n(inp["x"]), n(cw), n(cb))
    for bbar, mode in (("delta", oracle.BBAR_DELTA), ("zoh", oracle.BBAR_ZOH)):
        g = ss.selscan_bwd(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["z"],
                           d["delta_bias"], dy=dy.to(DEV), dfinal_state=df.to(DEV),
                           initial_state=h0.to(DEV), conv_weight=cw.to(DEV),
                           conv_bias=cb.to(DEV), bbar=bbar)
        torch.cuda.synchronize()
        o = orc.bwd(xc, n(inp["delta"]), n(inp["A"]), n(inp["B"]), n(inp["C"]), n(inp["D"]),
                    n(inp["z"]), n(inp["delta_bias"]), h0=n(h0), dy=n(dy), dfinal=n(df),
                    bbar=mode)
        for k in ("ddelta", "dz", "dA", "dB", "dC", "dD", "ddelta_bias", "dh0"):
            gh.compare(gh.to_np(g[k]), o[k], gh.RTOL["f32"], f"N={N} {bbar} {k}")
        dxin, dw, dcb = orc.causal_conv1d_bwd(n(inp["x"]), n(cw), n(cb), o["dx"])
        gh.compare(gh.to_np(g["dx"]), dxin, gh.RTOL["f32"], f"N={N} {bbar} dx_in")
        gh.compare(gh.to_np(g["dconv_weight"]), dw, gh.RTOL["f32"], f"N={N} {bbar} dconv_weight")
        gh.compare(gh.to_np(g["dconv_bias"]), dcb, gh.RTOL["f32"], f"N={N} {bbar} dconv_bias")


def test_wide_state_gradient_layer_sampled():
    """A Mamba-2-sized layer (2 × 2048 tokens, 2048 channels, d_state 128):
    the gradient of a channel sample against the oracle on those channels
    (the channels are independent), and dC, a sum over all channels, by the
    identity Σ dC·C = Σ dy·(y − D·x·silu(z)) (y − D·x·silu(z) is linear and
    homogeneous in C; no final-state gradient)."""
    w = wl.ScanWorkload("wide_bwd", 2, 2048, 2048, 128, "bf16", gate=True, seed=1300)
    inp = wl.make_scan_inputs(w)
    g0 = torch.Generator().manual_seed(1301)
    dy = torch.randn(2, 2048, 2048, generator=g0).to(torch.bfloat16)
    g = _gpu_bwd(inp, dy, None)
    torch.cuda.synchronize()
    chans = list(wl.channel_subset(2048, 64))
    o = _oracle_bwd(inp, dy, None, channels=chans)
    for k in ("dx", "ddelta", "dz"):
        gh.compare(gh.to_np(g[k][:, :, chans]), o[k], gh.RTOL["bf16"], f"layer {k}")
    for k in ("dA", "dD", "ddelta_bias"):
        gh.compare(gh.to_np(g[k][chans]), o[k], gh.RTOL["bf16"], f"layer {k}")
    d = {k: (None if v is None else v.to(DEV)) for k, v in inp.items()}
    y = ss.selscan_fwd(d["x"], d["delta"], d["A"], d["B"], d["C"], d["D"], d["z"],
                       d["delta_bias"])
    zz = d["z"].double()
    rest = y.double() - d["D"].double() * d["x"].double() * zz * torch.sigmoid(zz)
    rhs = float((dy.to(DEV).double() * rest).sum())
    lhs = float((g["dC"].double() * d["C"].double()).sum())
    assert abs(lhs - rhs) <= 2e-2 * abs(rhs), (lhs, rhs)
