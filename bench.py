#!/usr/bin/env python
"""Benchmark of the selective scan (libselscan) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl selscan|reference]

One step = one selscan_fwd call over one batch of the Mamba-2.8B-shaped layer
(batch 4, L 8192, d_inner 5120, d_state 16; bf16 x/delta/z/B/C, fp32 state,
softplus and silu gate on, final state returned). Inputs are synthetic and
seeded, and stay resident in HBM; at 1.35 GB per step they are ~10x the L2,
so no L2 flush is needed between steps.

Prints ONE JSON line (rank 0). Under torchrun each rank runs its own replica
(independent batches: weak scaling, no collective on the data path); time is
the max over ranks of the CUDA-event time of the K timed steps.

--impl reference times the float64 CPU oracle (the only reference there is)
on a bounded sample of the same workload, on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "selective-scan elems (B·L·D·N)/s"
UNIT = "elems/s"
WORKLOAD = "mamba2p8b_layer"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["selscan", "reference"], default="selscan")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target duration of the oracle CPU-baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    return ap.parse_args()


PROFILE = os.path.join(ROOT, "profiles", "scan_tma_mamba2p8b_layer.md")
KERNEL_SOURCES = ["scan_tma.cu", "tma_util.cuh", "selscan_device.cuh"]


def profiled_traffic():
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel sources changed since that capture (sha256 recorded beside it)."""
    import hashlib
    try:
        text = open(PROFILE).read()
    except OSError:
        return None
    want = traffic = None
    for line in text.splitlines():
        if line.startswith("kernel_sources_sha256:"):
            want = line.split(":", 1)[1].strip()
        if line.startswith("traffic_bytes_per_launch:"):
            traffic = int(line.split(":", 1)[1].strip())
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "selective_state_space_42_b200", "csrc")
    for f in KERNEL_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return traffic if want == h.hexdigest() else None


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def tensor_peak() -> float:
    """Dense bf16 TFLOP/s for a kernel timed alone (the measured burst figure,
    else the pool's earlier measurement)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"])
    except Exception:
        return 1590.0


# ---- clocks sampled during the timed region -----------------------------------
class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self._reader = threading.Thread(target=self._read, daemon=True)
        self._reader.start()
        time.sleep(0.6)  # nvidia-smi start-up

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons, n = [], None, set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        for ts, line in self.lines:
            if self.t0 is None or ts < self.t0 or ts > self.t1 + 0.15:
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                sm.append(float(parts[2]))
                mx = float(parts[3])
            except ValueError:
                continue
            n += 1
            for name, v in zip(names, parts[6:10]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": n}


# ---- CPU baseline: the float64 oracle on a bounded sample ------------------------
def _oracle_args(inp, rows, nch):
    """Host float64 copies of batch rows `rows` and channels 0..nch-1."""
    import torch
    sel = list(rows)
    bl = lambda t: None if t is None else t[sel][:, :, :nch].to("cpu", torch.float64).numpy()  # noqa
    ch = lambda t: t[:nch].to("cpu", torch.float64).numpy()  # noqa
    return (bl(inp["x"]), bl(inp["delta"]), ch(inp["A"]),
            inp["B"][sel].to("cpu", torch.float64).numpy(),
            inp["C"][sel].to("cpu", torch.float64).numpy(), ch(inp["D"]),
            bl(inp.get("z")), ch(inp["delta_bias"]))


def _sample_channels(w, rate, seconds, cores, rows=1):
    per_channel = rows * w.seqlen * w.dstate
    n = int(rate * seconds / per_channel)
    if n >= cores:
        n = n // cores * cores
    return max(1, min(w.dim, n))


def oracle_sample(w, inp, target_s, cores):
    """The one sample definition shared by `cpu_baseline` and the reference
    arm: the workload's batch rows in order, all of their tokens; channels
    0..n-1 of row 0 when one row takes longer than target_s seconds on
    `cores` threads, else whole rows, repeated when the whole workload is
    shorter. Sized from a short probe. Returns (oracle args, passes,
    elements per pass, description)."""
    import oracle
    orc = oracle.default()
    # the probe's inputs are prepared, and its threads started once, outside
    # the timed call: the rate is the oracle's own
    probe = min(w.dim, 4 * max(cores, 8))
    pargs = _oracle_args(inp, (0,), probe)
    orc.fwd(*pargs, softplus=True, threads=cores)
    t = time.perf_counter()
    orc.fwd(*pargs, softplus=True, threads=cores)
    rate = probe * w.seqlen * w.dstate / max(time.perf_counter() - t, 1e-9)
    row_s = w.dim * w.seqlen * w.dstate / rate
    if row_s >= target_s:
        rows, nch, reps = 1, _sample_channels(w, rate, target_s, cores), 1
        what = f"batch row 0, channels 0..{nch - 1} of {w.dim}"
    else:
        rows, nch = min(w.batch, max(1, int(target_s / row_s))), w.dim
        reps = max(1, int(round(target_s / (rows * row_s)))) if rows == w.batch else 1
        what = (f"batch rows 0..{rows - 1} of {w.batch}, all {w.dim} channels"
                + (f", {reps} passes" if reps > 1 else ""))
    desc = (f"{w.name}: {what}, all {w.seqlen} tokens, d_state {w.dstate}; "
            f"float64 oracle, OpenMP over channels")
    return (_oracle_args(inp, tuple(range(rows)), nch), reps,
            rows * nch * w.seqlen * w.dstate, desc)


def oracle_cpu_baseline(inp, w, target_s):
    """The oracle, as it stands, timed on the host cores on the shared sample
    (oracle_sample) of the workload; scan elements per second."""
    import oracle
    orc = oracle.default()
    cores = oracle.default_threads()
    args, reps, per_pass, desc = oracle_sample(w, inp, target_s, cores)
    t = time.perf_counter()
    for _ in range(reps):
        orc.fwd(*args, softplus=True, threads=cores)
    dt = time.perf_counter() - t
    el = reps * per_pass
    return {"value": el / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{desc}: {el:.3e} scan elements in {dt:.2f} s"}


def run_reference(args):
    """--impl reference: the oracle timed on the host cores; each step is the
    same bounded sample as the GPU arm's cpu_baseline (oracle_sample)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    from selective_state_space_42_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    cores = oracle.default_threads()
    inp = wl.make_scan_inputs(w, device="cpu")
    orc = oracle.default()
    per_step_s = min(args.cpu_seconds, 150.0 / max(args.steps + args.warmup, 1))
    a, reps, per_pass, desc = oracle_sample(w, inp, per_step_s, cores)
    times = []
    for i in range(args.warmup + args.steps):
        t = time.perf_counter()
        for _ in range(reps):
            orc.fwd(*a, softplus=True, threads=cores)
        if i >= args.warmup:
            times.append(time.perf_counter() - t)
    total = sum(times)
    elems = len(times) * reps * per_pass
    value = elems / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / max(len(times), 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(w, 1),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores,
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_block(w, world):
    return {"workload": w.name, "batch_per_gpu": w.batch, "seqlen": w.seqlen,
            "d_inner": w.dim, "d_state": w.dstate, "io_dtype": w.dtype,
            "state_dtype": "f32", "gate": w.gate, "delta_softplus": w.softplus,
            "final_state": w.final_state, "A": "-(n+1)",
            "parallelism": f"replicas x{world}" if world > 1 else "single",
            "l2": "no flush: inputs (1.35 GB/step) >> 126 MB L2"}


# ---- multi-rank helpers (host logic; tested with gloo on CPU) ------------------
def rank_seed(w, rank: int) -> int:
    """Each rank draws its own independent batch (weak scaling)."""
    return w.seed + 1000 * rank


def max_over_ranks(value: float, dist, device) -> float:
    """Max of a per-rank float over all ranks (every rank gets it)."""
    import torch
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(elements_per_rank: int, world: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: all ranks' elements over the slowest rank's time."""
    return elements_per_rank * world * steps / (max_ms / 1e3)


# ---- the GPU arm ---------------------------------------------------------------
def smi_id(torch, dev, local):
    """nvidia-smi id of a torch device: its PCI bus id when torch exposes it."""
    p = torch.cuda.get_device_properties(dev)
    try:
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except AttributeError:
        return str(local)


HOLD_CYCLES = 2_000_000  # device clock cycles (~1 ms at 1.965 GHz)


def time_calls(torch, stream, fn, n, flush=None):
    """CUDA-event time of one call in ms: the mean of n back-to-back calls,
    and (with `flush`, a buffer larger than L2 written before each call) the
    median of 10 calls each after an L2-evicting write."""
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    b2b = e0.elapsed_time(e1) / n
    if flush is None:
        return b2b, None
    cold = []
    for _ in range(10):
        flush.zero_()
        # ~1 ms of device-side spinning after the flush, so that the call is
        # already queued when the start event fires: the interval then holds
        # the call's device time, not the host's time to launch it
        torch.cuda._sleep(HOLD_CYCLES)
        c0 = torch.cuda.Event(enable_timing=True)
        c1 = torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        fn()
        c1.record(stream)
        torch.cuda.synchronize()
        cold.append(c0.elapsed_time(c1))
    return b2b, sorted(cold)[len(cold) // 2]


def extra_legs(args, torch, ss, wl, dev, stream, peak, over_ranks):
    """Other workloads of the path, timed the same way (not part of the
    headline metric): the other scan shapes, the general-A and ZOH variants
    of the headline shape, its gradient, the decode step and the SSD layer."""
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    out = {}

    def scan_leg(name, n, bbar="delta", ref_ms=None):
        w = wl.WORKLOADS[name]
        inp = wl.make_scan_inputs(w, device=dev)
        y = torch.empty_like(inp["x"])
        fs = torch.empty(w.batch, w.dim, w.dstate, device=dev, dtype=torch.float32)

        def call():
            ss.selscan_fwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                           inp["z"], inp["delta_bias"], softplus=True, y=y, final_state=fs,
                           stream=stream, bbar=bbar)
        b2b, cold = time_calls(torch, stream, call, n, flush)
        b2b, cold = over_ranks(b2b), over_ranks(cold)
        nb = w.algorithmic_bytes()
        leg = {"workload": name, "bytes_per_call": nb, "elements_per_call": w.elements,
               "us_back_to_back": b2b * 1e3, "us_after_l2_flush": cold * 1e3,
               "elems_per_s": w.elements / (b2b / 1e3),
               "GBps_back_to_back": nb / b2b / 1e6, "frac_back_to_back": nb / b2b / 1e6 / peak,
               "plan": ss.selscan_fwd_plan(w.batch, w.seqlen, w.dim, w.dstate)}
        if ref_ms is not None:
            leg["time_vs_headline_shape"] = b2b / ref_ms
        del inp, y, fs
        return leg, b2b

    out["mamba130m_layer"], _ = scan_leg("mamba130m_layer", 200)
    out["long_1m"], _ = scan_leg("long_1m", 5)
    ref = args.headline_ms
    out["pages_A"], _ = scan_leg("mamba2p8b_layer_expA", 100, ref_ms=ref)
    out["pages_A"]["A"] = ("-exp(log(n+1)) in float32 (within a few ulps of (n+1)*A[d,0]: "
                           "power-ladder decay)")
    out["general_A"], _ = scan_leg("mamba2p8b_layer_trainedA", 100, ref_ms=ref)
    out["general_A"]["A"] = "-exp(log(n+1) + 0.1*N(0,1)) per (d, n) in float32: general decay"
    out["zoh"], _ = scan_leg("mamba2p8b_layer", 50, bbar="zoh", ref_ms=ref)
    out["zoh"]["input_term"] = "(exp(delta*A)-1)/A*B*x"

    # the gradient of the headline shape (dy and a final-state gradient in;
    # dx, ddelta, dz, dA, dB, dC, dD, ddelta_bias out)
    gw = wl.WORKLOADS["mamba2p8b_layer"]
    ginp = wl.make_scan_inputs(gw, device=dev)
    gg = torch.Generator(device=dev)
    gg.manual_seed(gw.seed + 1000)
    gdy = torch.randn(gw.batch, gw.seqlen, gw.dim, generator=gg, device=dev).to(ginp["x"].dtype)
    gdf = torch.randn(gw.batch, gw.dim, gw.dstate, generator=gg, device=dev)

    def grad_call():
        ss.selscan_bwd(ginp["x"], ginp["delta"], ginp["A"], ginp["B"], ginp["C"], ginp["D"],
                       ginp["z"], ginp["delta_bias"], softplus=True, dy=gdy, dfinal_state=gdf,
                       stream=stream)
    b2b, cold = time_calls(torch, stream, grad_call, 10, flush)
    b2b, cold = over_ranks(b2b), over_ranks(cold)
    gnb = gw.backward_algorithmic_bytes()
    out["gradient"] = {
        "workload": gw.name, "bytes_per_call": gnb, "elements_per_call": gw.elements,
        "us_back_to_back": b2b * 1e3, "us_after_l2_flush": cold * 1e3,
        "GBps_back_to_back": gnb / b2b / 1e6, "frac_back_to_back": gnb / b2b / 1e6 / peak,
        "time_vs_headline_shape": b2b / ref,
        "kernels": "scan_bwd_pairs_kernel + bwd_reduce_bc_kernel + bwd_reduce_params_kernel"}
    del ginp, gdy, gdf

    # the decode step (one token in place on the [256, 5120, 16] state); the
    # after-flush time is the headline: back to back the 84 MB state stays in L2
    dw = wl.DECODE
    dstate_t = wl.make_decode_state(dw, device=dev)
    dA, dDv, dbias = wl.make_decode_params(dw, device=dev)
    dsteps = [wl.make_decode_step(dw, s, device=dev) for s in range(4)]
    k = [0]

    def decode():
        t = dsteps[k[0] % len(dsteps)]
        k[0] += 1
        ss.selscan_state_update(dstate_t, t["x"], t["delta"], dA, t["B"], t["C"], dDv, t["z"],
                                dbias, stream=stream)
    b2b, cold = time_calls(torch, stream, decode, 200, flush)
    b2b, cold = over_ranks(b2b), over_ranks(cold)
    nb = dw.algorithmic_bytes_per_step()
    out["decode_step"] = {
        "workload": dw.name, "bytes_per_step": nb,
        "us": cold * 1e3, "GBps": nb / cold / 1e6, "frac": nb / cold / 1e6 / peak,
        "timing": "after an L2-evicting write",
        "us_back_to_back": b2b * 1e3, "GBps_back_to_back": nb / b2b / 1e6,
        "kernel": "state_update_vec_kernel<bf16, gate>"}

    # the Mamba-2-shaped SSD layer (one scalar A per head, chunked form on
    # the tensor cores)
    sw = wl.SSD
    sinp = wl.make_ssd_inputs(sw, device=dev)
    sy = torch.empty_like(sinp["x"])
    sfs = torch.empty(sw.batch, sw.dim, sw.dstate, device=dev)

    def ssd_call():
        ss.selscan_ssd_fwd(sinp["x"], sinp["dt"], sinp["A"], sinp["B"], sinp["C"], D=sinp["D"],
                           z=sinp["z"], dt_bias=sinp["dt_bias"], y=sy, final_state=sfs,
                           stream=stream)
    b2b, cold = time_calls(torch, stream, ssd_call, 50, flush)
    b2b, cold = over_ranks(b2b), over_ranks(cold)
    out["ssd_layer"] = {
        "workload": sw.name, "bytes_per_call": sw.algorithmic_bytes(),
        "flops_per_call": sw.algorithmic_flops(),
        "us_back_to_back": b2b * 1e3, "us_after_l2_flush": cold * 1e3,
        "GBps_back_to_back": sw.algorithmic_bytes() / b2b / 1e6,
        "TFLOPs_back_to_back": sw.algorithmic_flops() / b2b / 1e9,
        "frac_hbm_back_to_back": sw.algorithmic_bytes() / b2b / 1e6 / peak,
        "frac_tensor_back_to_back": sw.algorithmic_flops() / b2b / 1e9 / tensor_peak()}
    del flush
    return out


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    import selective_state_space_42_b200 as ss
    from selective_state_space_42_b200 import workloads as wl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", device_id=dev,
                                timeout=datetime.timedelta(seconds=120))
    ss.load_library()

    w = wl.WORKLOADS[args.workload]
    plan = ss.selscan_fwd_plan(w.batch, w.seqlen, w.dim, w.dstate)
    inp = wl.make_scan_inputs(w.scaled(seed=rank_seed(w, rank)), device=dev)
    y = torch.empty_like(inp["x"])
    fs = torch.empty(w.batch, w.dim, w.dstate, device=dev, dtype=torch.float32)
    stream = torch.cuda.current_stream(dev)

    def step():
        ss.selscan_fwd(inp["x"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                       inp["z"], inp["delta_bias"], softplus=True, y=y, final_state=fs,
                       stream=stream)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)

    sampler = None if args.no_clocks else ClockSampler(smi_id(torch, dev, local))
    if sampler:
        sampler.start()
    barrier()
    torch.cuda.synchronize(dev)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    if sampler:
        sampler.mark_start()
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.mark_end()
    barrier()
    ms = ev0.elapsed_time(ev1)
    clocks = sampler.stop() if sampler else None
    ms = max_over_ranks(ms, dist if world > 1 else None, dev)
    args.headline_ms = ms / args.steps

    # end to end through the public call: pinned host inputs -> device ->
    # selscan_fwd -> y and final state back to pinned host memory, every
    # step. Two buffer sets on three streams, as a streaming caller would run
    # it: step i + 1's inputs go up while step i computes and step i − 1's
    # outputs come down (PCIe carries both directions at once).
    names = ["x", "delta", "z", "B", "C"]
    host = {k: inp[k].to("cpu").pin_memory() for k in names}
    nbuf = 2
    y_h = [torch.empty(y.shape, dtype=y.dtype, pin_memory=True) for _ in range(nbuf)]
    fs_h = [torch.empty(fs.shape, dtype=fs.dtype, pin_memory=True) for _ in range(nbuf)]
    dbuf = [{k: torch.empty_like(inp[k]) for k in names} for _ in range(nbuf)]
    ybuf = [y, torch.empty_like(y)]
    fsbuf = [fs, torch.empty_like(fs)]
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    up_done = [torch.cuda.Event() for _ in range(nbuf)]
    comp_done = [torch.cuda.Event() for _ in range(nbuf)]
    down_done = [torch.cuda.Event() for _ in range(nbuf)]
    for e in comp_done + down_done:
        e.record(stream)
    k_step = [0]

    def e2e_step():
        j = k_step[0] % nbuf
        k_step[0] += 1
        s_up.wait_event(comp_done[j])      # the last call that read this input set is done
        with torch.cuda.stream(s_up):
            for k in names:
                dbuf[j][k].copy_(host[k], non_blocking=True)
            up_done[j].record(s_up)
        stream.wait_event(up_done[j])
        stream.wait_event(down_done[j])    # this y / final-state set has been read back
        ss.selscan_fwd(dbuf[j]["x"], dbuf[j]["delta"], inp["A"], dbuf[j]["B"], dbuf[j]["C"],
                       inp["D"], dbuf[j]["z"], inp["delta_bias"], softplus=True, y=ybuf[j],
                       final_state=fsbuf[j], stream=stream)
        comp_done[j].record(stream)
        s_down.wait_event(comp_done[j])
        with torch.cuda.stream(s_down):
            y_h[j].copy_(ybuf[j], non_blocking=True)
            fs_h[j].copy_(fsbuf[j], non_blocking=True)
            down_done[j].record(s_down)

    e2e_step()
    torch.cuda.synchronize(dev)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_up.wait_event(e0)
    s_down.wait_event(e0)
    for _ in range(args.e2e_steps):
        e2e_step()
    stream.wait_stream(s_down)
    stream.wait_stream(s_up)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist if world > 1 else None, dev)
    h2d = sum(host[k].numel() * host[k].element_size() for k in names)
    d2h = y_h[0].numel() * y_h[0].element_size() + fs_h[0].numel() * fs_h[0].element_size()

    peak, peak_kind = peaks()
    legs = extra_legs(args, torch, ss, wl, dev, stream, peak,
                      lambda v: max_over_ranks(v, dist if world > 1 else None, dev))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_cpu_baseline(inp, w, args.cpu_seconds)

    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    if rank != 0:
        return 0

    value = job_rate(w.elements, world, args.steps, ms)
    per_launch_s = ms / 1e3 / args.steps
    alg_bytes = w.algorithmic_bytes()
    achieved = alg_bytes / per_launch_s / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded N(0,1) inputs, Mamba-2.8B layer shapes, no weights)",
        "config": config_block(w, world),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind,
                     "frac_of_8TBps": achieved / 8000.0,
                     "algorithmic_bytes_per_launch": alg_bytes,
                     "kernel": "scan_tma_kernel<bf16, gate, seq, softplus> (two lanes per chain)",
                     "traffic": profiled_traffic()},
        "e2e": {"value": job_rate(w.elements, world, args.e2e_steps, e2e_ms),
                "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms / args.e2e_steps},
        **legs,
        "gpu_launches": args.steps * plan["launches"],
        "plan": plan,
        "cpu_baseline": cpu,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
