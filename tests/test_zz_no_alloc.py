"""selscan_fwd_noalloc: the selective scan for callers that cannot allocate
device memory while they run (their device memory belongs to another
allocator, an allocation could stall a latency-critical loop, or stream-ordered
memory pools are unavailable). Its chunk workspace is a fixed array inside the
library instead of a stream-ordered allocation; its results must match
selscan_fwd's.

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

# a shape whose launch plan is chunked, so the fixed workspace is used
SHAPE = wl.ScanWorkload("noalloc", 2, 3000, 384, 16, "bf16", gate=True, seed=11)


def _cuda_inputs(w):
    return {k: (None if v is None else v.to(DEV))
            for k, v in wl.make_scan_inputs(w).items()}


def test_noalloc_matches_selscan_fwd_on_two_calls_in_a_row():
    w = SHAPE
    plan = ss.selscan_fwd_plan(w.batch, w.seqlen, w.dim, w.dstate)
    assert plan["chunks"] > 1
    assert 0 < plan["workspace_bytes"] <= ss.SELSCAN_NOALLOC_WORKSPACE_BYTES
    for seed in (11, 12):  # the second call finds the first call's workspace contents
        inp = _cuda_inputs(w.scaled(seed=seed))
        args = (inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                inp["z"], inp["delta_bias"])
        y_ref, h_ref = ss.selscan_fwd(*args, softplus=True, return_final_state=True)
        y = torch.empty_like(inp["x"])
        h = torch.empty(w.batch, w.dim, w.dstate, device=DEV, dtype=torch.float32)
        ss.selscan_fwd_noalloc(*args, softplus=True, y=y, final_state=h)
        torch.cuda.synchronize()
        gh.compare(gh.to_np(y), gh.to_np(y_ref), gh.RTOL["bf16"], f"noalloc y (seed {seed})")
        gh.compare(gh.to_np(h), gh.to_np(h_ref), gh.RTOL["bf16"],
                   f"noalloc final state (seed {seed})")


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
