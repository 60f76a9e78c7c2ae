"""Run a fixed number of launches of one kernel on a named workload.

Meant to sit under a profiler (one kernel, a few launches, nothing else on
the device) and to give quick CUDA-event timings without one:

    python -m selective_state_space_42_b200.profile_case scan mamba2p8b_layer --launches 2
    python -m selective_state_space_42_b200.profile_case decode --launches 3
    python -m selective_state_space_42_b200.profile_case bwd mamba2p8b_layer --launches 2
    python -m selective_state_space_42_b200.profile_case bwd mamba2p8b_layer --seqlen 1024
    python -m selective_state_space_42_b200.profile_case ssd --launches 3
    python -m selective_state_space_42_b200.profile_case decode --launches 4 --flushed 3

``scan`` calls selscan_fwd on a scan workload; ``bwd`` calls selscan_bwd on
it (with a seeded dy and final-state gradient); ``decode`` calls
selscan_state_update on the decode workload; ``ssd`` calls selscan_ssd_fwd
on the Mamba-2-shaped head workload. With ``--time`` it also prints
the median CUDA-event time per launch, cold (a 512 MiB buffer is written
between launches, which evicts L2) and back to back, as one JSON line.
``--flushed N`` adds N launches after the back-to-back ones, each after a
512 MiB write (for DRAM counters of launches that find L2 full of another
buffer's dirty lines).
"""
from __future__ import annotations

import argparse
import dataclasses
import json

import torch

from . import selscan as ss
from . import workloads as wl


def _workload(name: str, seqlen: int | None):
    w = wl.WORKLOADS[name]
    return w if seqlen is None else dataclasses.replace(w, seqlen=seqlen)


def _scan_case(name: str, seqlen: int | None = None):
    w = _workload(name, seqlen)
    inp = wl.make_scan_inputs(w, device="cuda")
    y = torch.empty_like(inp["x"])
    fs = torch.empty(w.batch, w.dim, w.dstate, device="cuda") if w.final_state else None

    def launch(_i: int) -> None:
        ss.selscan_fwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                       inp["z"], inp["delta_bias"], softplus=w.softplus, y=y,
                       final_state=fs)

    return launch, w.algorithmic_bytes()


def _bwd_case(name: str, seqlen: int | None = None):
    w = _workload(name, seqlen)
    inp = wl.make_scan_inputs(w, device="cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(w.seed + 1000)
    dy = torch.randn(w.batch, w.seqlen, w.dim, generator=g, device="cuda").to(inp["x"].dtype)
    dfinal = torch.randn(w.batch, w.dim, w.dstate, generator=g, device="cuda")

    def launch(_i: int) -> None:
        ss.selscan_bwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                       inp["z"], inp["delta_bias"], softplus=w.softplus, dy=dy,
                       dfinal_state=dfinal)

    return launch, w.backward_algorithmic_bytes()


def _decode_case():
    w = wl.DECODE
    state = wl.make_decode_state(w, device="cuda")
    A, Dv, bias = wl.make_decode_params(w, device="cuda")
    steps = [wl.make_decode_step(w, s, device="cuda") for s in range(8)]
    y = torch.empty(w.batch, w.dim, device="cuda", dtype=wl.DTYPES[w.dtype])

    def launch(i: int) -> None:
        s = steps[i % len(steps)]
        ss.selscan_state_update(state, s["x"], s["delta"], A, s["B"], s["C"], Dv, s["z"],
                                bias, y=y)

    return launch, w.algorithmic_bytes_per_step()


def _ssd_case():
    w = wl.SSD
    inp = wl.make_ssd_inputs(w, device="cuda")
    y = torch.empty_like(inp["x"])
    fs = torch.empty(w.batch, w.dim, w.dstate, device="cuda")

    def launch(_i: int) -> None:
        ss.selscan_ssd_fwd(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], D=inp["D"],
                           z=inp["z"], dt_bias=inp["dt_bias"], y=y, final_state=fs)

    return launch, w.algorithmic_bytes()


def _median(v):
    v = sorted(v)
    return v[len(v) // 2]


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("kernel", choices=["scan", "bwd", "decode", "ssd"])
    ap.add_argument("workload", nargs="?", default="mamba2p8b_layer",
                    help="scan workload name (ignored for decode)")
    ap.add_argument("--launches", type=int, default=2)
    ap.add_argument("--time", action="store_true")
    ap.add_argument("--flushed", type=int, default=0,
                    help="launches after the back-to-back ones, each after a 512 MiB write")
    ap.add_argument("--seqlen", type=int, default=None,
                    help="scan and bwd: the workload cut (or grown) to this many tokens")
    args = ap.parse_args(argv)

    if args.kernel == "scan":
        launch, nbytes = _scan_case(args.workload, args.seqlen)
    elif args.kernel == "bwd":
        launch, nbytes = _bwd_case(args.workload, args.seqlen)
    elif args.kernel == "ssd":
        launch, nbytes = _ssd_case()
    else:
        launch, nbytes = _decode_case()
    for i in range(args.launches):
        launch(i)
    if args.flushed > 0:
        buf = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
        for i in range(args.flushed):
            buf.zero_()
            launch(args.launches + i)
        del buf
    torch.cuda.synchronize()
    out = {"kernel": args.kernel, "launches": args.launches,
           "workload": {"decode": wl.DECODE.name, "ssd": wl.SSD.name}.get(args.kernel,
                                                                          args.workload),
           "seqlen": args.seqlen, "algorithmic_bytes": nbytes}
    if args.time:
        flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
        cold = []
        for i in range(20):
            flush.zero_()
            # device-side spin so that the launch is queued before e0 fires:
            # the interval holds the kernels, not the host's launch time
            torch.cuda._sleep(2_000_000)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            launch(i)
            e1.record()
            torch.cuda.synchronize()
            cold.append(e0.elapsed_time(e1))
        n = 100
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(n):
            launch(i)
        e1.record()
        torch.cuda.synchronize()
        b2b = e0.elapsed_time(e1) / n
        cold_ms = _median(cold)
        out.update(cold_ms=cold_ms, cold_GBps=nbytes / cold_ms / 1e6, b2b_ms=b2b,
                   b2b_GBps=nbytes / b2b / 1e6)
    status = ss.selscan_device_status()
    out["device_status"] = status
    print(json.dumps(out), flush=True)
    return 0 if status == 0 else 1


if __name__ == "__main__":
    raise SystemExit(main())
