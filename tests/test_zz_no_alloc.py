"""selscan_fwd_noalloc: the selective scan for callers that cannot allocate
device memory while they run (their device memory belongs to another
allocator, an allocation could stall a latency-critical loop, or stream-ordered
memory pools are unavailable). Its chunk workspace is a fixed array inside the
library instead of a stream-ordered allocation. It runs the same plan and the
same kernels as selscan_fwd on the same inputs, so its results must be
bit-identical to selscan_fwd's.

The array is laid out three ways, one per plan, and each is exercised here:
the one-pass TMA plan (tickets, hand-over flags and handed-over states), the
chunked TMA plan (tickets, chunk aggregates and carried states) and the
generic kernels' chunked plan (aggregates and states only).

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import pytest
import torch

import selective_state_space_42_b200 as ss
from selective_state_space_42_b200 import workloads as wl

import gpu_helpers as gh

pytestmark = pytest.mark.gpu
DEV = "cuda"
F32 = 4

# (workload, expected plan); selscan_fwd_plan reports the plan of 16-byte
# aligned bf16 tensors, and the fp32 shape below takes the same generic plan
# (dim < 128 rules out the TMA kernel for either dtype).
CASES = {
    # one pass, 1024-token units handed from chunk to chunk: 2 units per group
    "tma_one_pass": wl.ScanWorkload("noalloc_seq", 4, 2048, 5120, 16, "bf16", gate=True,
                                    seed=21),
    # few groups: aggregates -> carry -> rescan
    "tma_chunked": wl.ScanWorkload("noalloc_chunked", 2, 3000, 384, 16, "bf16", gate=True,
                                   seed=11),
    # generic kernels (fp32, 96 channels): aggregates -> carry -> rescan
    "generic_chunked": wl.ScanWorkload("noalloc_generic", 1, 4096, 96, 16, "f32", gate=True,
                                       seed=31),
}


def _cuda_inputs(w):
    return {k: (None if v is None else v.to(DEV))
            for k, v in wl.make_scan_inputs(w).items()}


def _check_plan(name, w):
    plan = ss.selscan_fwd_plan(w.batch, w.seqlen, w.dim, w.dstate)
    assert 0 < plan["workspace_bytes"] <= ss.SELSCAN_NOALLOC_WORKSPACE_BYTES
    if name == "tma_one_pass":
        assert plan["launches"] == 1 and plan["chunks"] == 2
    elif name == "tma_chunked":
        assert plan["launches"] == 3 and plan["chunks"] > 1
        # 256 bytes of counters, then P and H: [batch][chunks][dim][16] each
        assert plan["workspace_bytes"] == 256 + 2 * w.batch * plan["chunks"] * w.dim * 16 * F32
    else:
        assert plan["launches"] == 3 and plan["chunks"] > 1
        # no counters: P and H only
        assert plan["workspace_bytes"] == 2 * w.batch * plan["chunks"] * w.dim * 16 * F32


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_matches_selscan_fwd_on_two_calls_in_a_row(name):
    w = CASES[name]
    _check_plan(name, w)
    for seed in (w.seed, w.seed + 1):  # the second call finds the first call's contents
        inp = _cuda_inputs(w.scaled(seed=seed))
        args = (inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                inp["z"], inp["delta_bias"])
        y_ref, h_ref = ss.selscan_fwd(*args, softplus=True, return_final_state=True)
        y = torch.empty_like(inp["x"])
        h = torch.empty(w.batch, w.dim, w.dstate, device=DEV, dtype=torch.float32)
        ss.selscan_fwd_noalloc(*args, softplus=True, y=y, final_state=h)
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref), f"{name}: noalloc y differs (seed {seed})"
        assert torch.equal(h, h_ref), f"{name}: noalloc final state differs (seed {seed})"
    assert ss.selscan_device_status() == 0


def test_noalloc_rejects_sizes_beyond_its_workspace():
    w = wl.ScanWorkload("noalloc_big", 1, 32768, 2048, 16, "bf16", gate=False, seed=13)
    with gh.forced_chunks(128):
        plan = ss.selscan_fwd_plan(w.batch, w.seqlen, w.dim, w.dstate)
        assert plan["workspace_bytes"] > ss.SELSCAN_NOALLOC_WORKSPACE_BYTES
        inp = _cuda_inputs(w)
        with pytest.raises(ss.SelscanError) as e:
            ss.selscan_fwd_noalloc(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"],
                                   inp["D"], None, inp["delta_bias"])
        assert e.value.status == -8
    torch.cuda.synchronize()
