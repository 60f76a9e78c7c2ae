"""A bounded device-side wait that runs out, made to run out on purpose.

The one-pass plan hands each unit's final state to the next chunk through a
flag in global memory; the successor waits for it with a wait bounded by
%globaltimer (SELSCAN_TIMEOUT_MS). The test hook SELSCAN_TEST_SKIP_RELEASE
makes the units of one chunk skip that flag, so every successor's wait runs
out. Nothing faults: the waiting CTA records code 1 in the library's sticky
device word, raises the launch's abort word so that every other CTA leaves
its next wait, and the launch ends normally. The context stays usable: the
next call on it gives the same bits as a clean run.
"""
import time

import pytest
import torch

import selective_state_space_42_b200 as ss
from selective_state_space_42_b200 import workloads as wl

import gpu_helpers as gh

pytestmark = pytest.mark.gpu
DEV = "cuda"

# one-pass plan, 64-token units: 2 batch rows x 2 tiles x 4 chunks = 16 units,
# all resident at once
PLAN = dict(SELSCAN_PATH="seq", SELSCAN_UNIT="64", SELSCAN_CHUNKS=None)
W = wl.ScanWorkload("waitfail", 2, 256, 256, 16, "bf16", gate=True, seed=91)


def _run(inp):
    y, h = ss.selscan_fwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                          inp["z"], inp["delta_bias"], softplus=True,
                          return_final_state=True)
    torch.cuda.synchronize()
    return y, h


def test_flag_wait_runs_out_and_context_survives():
    inp = {k: (None if v is None else v.to(DEV)) for k, v in wl.make_scan_inputs(W).items()}
    assert ss.selscan_device_status(clear=True) == 0
    with gh.env(**PLAN, SELSCAN_TEST_SKIP_RELEASE=None, SELSCAN_TIMEOUT_MS=None):
        plan = ss.selscan_fwd_plan(W.batch, W.seqlen, W.dim, W.dstate)
        assert plan["launches"] == 1 and plan["chunks"] == 4
        y_ref, h_ref = _run(inp)
    assert ss.selscan_device_status() == 0

    # chunk 0 publishes nothing: the chunk-1 units' waits run out after 20 ms
    with gh.env(**PLAN, SELSCAN_TEST_SKIP_RELEASE="0", SELSCAN_TIMEOUT_MS="20"):
        t0 = time.perf_counter()
        _run(inp)  # returns, and the synchronize inside reports no CUDA error
        elapsed = time.perf_counter() - t0
    assert ss.selscan_device_status(clear=True) == 1  # code 1: a predecessor-flag wait
    assert elapsed < 2.0  # the abort word stopped the other CTAs; nothing hung

    with gh.env(**PLAN, SELSCAN_TEST_SKIP_RELEASE=None, SELSCAN_TIMEOUT_MS=None):
        y, h = _run(inp)
    assert torch.equal(y, y_ref) and torch.equal(h, h_ref)
    assert ss.selscan_device_status() == 0
