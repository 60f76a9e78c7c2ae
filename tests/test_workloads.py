"""The seeded input generators and the algorithmic byte counts behind the
roofline figures, on CPU: the generators are deterministic and draw what their
docstrings state, and every per-call byte count equals the summed sizes of the
tensors that call must read and write, counted from real tensors."""
import math

import pytest
import torch
from hypothesis import given, settings, strategies as st

from selective_state_space_42_b200 import workloads as wl


def _nb(*ts):
    return sum(t.numel() * t.element_size() for t in ts if t is not None)


@pytest.mark.parametrize("gate", [True, False])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_forward_bytes_are_the_tensors_it_moves(gate, dtype):
    w = wl.ScanWorkload("t", 2, 24, 40, 16, dtype, gate=gate, seed=1)
    i = wl.make_scan_inputs(w)
    y = torch.empty_like(i["x"])
    final = torch.empty(w.batch, w.dim, w.dstate)
    want = _nb(i["x"], i["delta"], i["z"], i["B"], i["C"], i["A"], i["D"], i["delta_bias"],
               y, final)
    assert w.algorithmic_bytes() == want


@pytest.mark.parametrize("gate", [True, False])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_gradient_bytes_are_the_tensors_it_moves(gate, dtype):
    """In: x, delta, z, dy, B, C, A, D, delta_bias and the final state's
    gradient; out: dx, ddelta, dz, dB, dC (float32), dA, dD, ddelta_bias."""
    w = wl.ScanWorkload("t", 2, 24, 40, 16, dtype, gate=gate, seed=1)
    i = wl.make_scan_inputs(w)
    dy = torch.empty_like(i["x"])
    dfinal = torch.empty(w.batch, w.dim, w.dstate)
    grads = [torch.empty_like(i["x"]), torch.empty_like(i["delta"]),
             None if i["z"] is None else torch.empty_like(i["z"]),
             torch.empty(i["B"].shape), torch.empty(i["C"].shape),
             torch.empty_like(i["A"]), torch.empty_like(i["D"]),
             torch.empty_like(i["delta_bias"])]
    want = _nb(i["x"], i["delta"], i["z"], dy, i["B"], i["C"], i["A"], i["D"],
               i["delta_bias"], dfinal, *grads)
    assert w.backward_algorithmic_bytes() == want


@pytest.mark.parametrize("gate", [True, False])
def test_decode_bytes_are_the_tensors_it_moves(gate):
    """The state is read and written; x, delta, z in and y out; B, C per row."""
    w = wl.DecodeWorkload("t", 3, 40, 16, 1, "bf16", gate=gate, seed=2)
    st = wl.make_decode_state(w)
    A, D, bias = wl.make_decode_params(w)
    s = wl.make_decode_step(w, 0)
    y = torch.empty_like(s["x"])
    want = 2 * _nb(st) + _nb(s["x"], s["delta"], s["z"] if gate else None, s["B"], s["C"],
                             A, D, bias, y)
    assert w.algorithmic_bytes_per_step() == want


@pytest.mark.parametrize("gate", [True, False])
def test_ssd_bytes_are_the_tensors_it_moves(gate):
    w = wl.SsdWorkload("t", 2, 50, 3, 8, 16, "bf16", gate=gate, seed=3)
    i = wl.make_ssd_inputs(w)
    y = torch.empty_like(i["x"])
    final = torch.empty(w.batch, w.dim, w.dstate)
    want = _nb(i["x"], i["dt"], i["z"], i["B"], i["C"], i["A"], i["D"], i["dt_bias"], y,
               final)
    assert w.algorithmic_bytes() == want


def test_ssd_flops_count_each_chunk_product_once():
    """One chunk of q tokens per head: C·Bᵀ is q×q×N multiply-adds, M·X
    q×q×P, C·h_in q×N×P and Bᵀ·(w∘X) N×q×P; a ragged last chunk counts
    its own length."""
    w = wl.SsdWorkload("t", 1, 200, 1, 8, 16, "bf16", gate=False, seed=3)

    def per_chunk(q, N=16, P=8):
        return 2 * (q * q * N + q * q * P + q * N * P + N * q * P)
    assert w.algorithmic_flops(128) == per_chunk(128) + per_chunk(72)
    assert w.algorithmic_flops(64) == 3 * per_chunk(64) + per_chunk(8)


def test_generators_are_deterministic_and_seeded():
    w = wl.ScanWorkload("t", 2, 30, 20, 16, "bf16", gate=True, seed=11)
    a, b = wl.make_scan_inputs(w), wl.make_scan_inputs(w)
    for k in a:
        assert torch.equal(a[k], b[k]), k
    c = wl.make_scan_inputs(w.scaled(seed=12))
    assert not torch.equal(a["x"], c["x"])
    s0, s1 = (wl.make_decode_step(wl.DECODE, k) for k in (0, 1))
    assert not torch.equal(s0["x"], s1["x"])


def test_generators_draw_the_stated_distributions():
    """A[d, n] = −(n+1); softplus(delta_bias) in [1e-3, 1e-1]; x, z, B, C
    standard normal and delta 0.5·N(0, 1) (moments of each tensor); SSD
    heads' A in −[0.5, 4]."""
    w = wl.ScanWorkload("t", 2, 512, 256, 16, "f32", gate=True, seed=5)
    i = wl.make_scan_inputs(w)
    assert torch.equal(i["A"], -torch.arange(1, 17, dtype=torch.float32).repeat(256, 1))
    sp = torch.nn.functional.softplus(i["delta_bias"].double())
    assert float(sp.min()) >= 1e-3 * (1 - 1e-5) and float(sp.max()) <= 1e-1 * (1 + 1e-5)
    for k, sd in (("x", 1.0), ("z", 1.0), ("delta", 0.5), ("B", 1.0), ("C", 1.0)):
        v = i[k].double()
        n = v.numel()
        assert abs(float(v.mean())) < 5 * sd / math.sqrt(n), k
        assert abs(float(v.std()) / sd - 1) < 0.02, k
    assert abs(float(i["D"].mean()) - 1.0) < 0.05
    tiny = wl.make_scan_inputs(wl.WORKLOADS["tiny_f32"])
    assert torch.equal(tiny["D"], torch.ones(64)) and tiny["z"] is None
    s = wl.make_ssd_inputs(wl.SsdWorkload("t", 1, 8, 64, 4, 16, "bf16", True, 6))
    assert float(s["A"].max()) <= -0.5 and float(s["A"].min()) >= -4.0


def test_bench_workload_byte_counts():
    """The per-call figures the roofline lines divide by."""
    assert wl.WORKLOADS["mamba2p8b_layer"].algorithmic_bytes() == 1_345_953_792
    assert wl.WORKLOADS["mamba2p8b_layer"].backward_algorithmic_bytes() == 2_357_149_696
    assert wl.WORKLOADS["mamba130m_layer"].backward_algorithmic_bytes() == 356_474_880
    assert wl.DECODE.algorithmic_bytes_per_step() == 178_642_944
    assert wl.SSD.algorithmic_bytes() == 107_479_424
    assert wl.SSD.algorithmic_flops() == 21_474_836_480  # 2·32 heads·32 chunks·10.5 MFLOP


@settings(max_examples=200, deadline=None)
@given(dim=st.integers(1, 10_000), stride=st.integers(1, 512))
def test_channel_subset_covers_the_edges(dim, stride):
    """The channels the full-size parity tests sample: sorted, distinct, in
    range, always the first, second and last channel, and every stride-th."""
    s = list(wl.channel_subset(dim, stride))
    assert s == sorted(set(s)) and all(0 <= c < dim for c in s)
    assert {0, min(1, dim - 1), dim - 1} <= set(s)
    assert set(range(0, dim, stride)) <= set(s)


def test_ragged_shapes_span_tiles_with_tails():
    """The small parity shapes include lengths and widths that are not
    multiples of the kernels' 32-token and 32/128-channel tiles."""
    shapes = wl.ragged_shapes()
    assert shapes
    assert any(s[1] % 32 for s in shapes) and any(s[2] % 32 for s in shapes)
    assert any(s[1] > 32 for s in shapes) and any(s[2] > 128 for s in shapes)


def test_a_initialisations():
    """The three A recipes: −(n+1) exactly; the pages' −exp(log(n+1)) within
    2^−21 of it (the kernels' ladder bound); the trained-like A negative and
    off the ladder by far more than that bound."""
    ladder = wl.a_matrix(8, 16, "ladder")
    assert torch.equal(ladder, -torch.arange(1, 17, dtype=torch.float32).repeat(8, 1))
    pages = wl.a_matrix(8, 16, "exp_log")
    assert float(((pages - ladder).abs() / ladder.abs()).max()) <= 2.0 ** -21
    trained = wl.a_matrix(8, 16, "trained")
    assert bool((trained < 0).all())
    assert float(((trained - ladder).abs() / ladder.abs()).min()) > 2.0 ** -21
    assert torch.equal(trained, wl.a_matrix(8, 16, "trained"))  # seeded
