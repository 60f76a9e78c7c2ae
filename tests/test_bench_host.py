"""Host-side logic of bench.py on CPU: the parsing of the clock samples taken
during the timed region, the check that ties the recorded DRAM traffic to the
kernel sources it was captured from, the default launch arguments, and the
reference arm (the float64 oracle timed on the host cores, rank 0 only)."""
import json
import os
import shutil
import subprocess
import sys

import pytest

import bench


class _FakeSmi:
    """Stands in for the nvidia-smi child process once its lines are read."""

    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _line(sm, mx=1965, reasons=("Not Active",) * 4):
    # timestamp, index, clocks.sm, clocks.max.sm, power.draw, active mask, 4 reasons
    return ", ".join(["2026/01/01 00:00:00.000", "0", str(sm), str(mx), "812.5", "0x0"]
                     + list(reasons))


def _sampler(lines, t0=10.0, t1=20.0):
    s = bench.ClockSampler(0)
    s.proc = _FakeSmi()
    s.lines = lines
    s.t0, s.t1 = t0, t1
    return s


def test_clock_median_uses_only_the_timed_window():
    lines = [(5.0, _line(345)),                     # before the window
             (11.0, _line(1900)), (12.0, _line(1950)), (13.0, _line(1800)),
             (20.1, _line(1965)),                   # inside the 0.15 s grace
             (25.0, _line(210))]                    # after the window
    out = _sampler(lines).stop()
    assert out["samples"] == 4
    assert out["sm_mhz"] == pytest.approx((1900 + 1950) / 2)
    assert out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == []


def test_clock_reasons_are_named():
    act = ("Not Active", "Not Active", "Active", "Active")
    lines = [(11.0, _line(1300, reasons=act)), (12.0, _line(1310))]
    out = _sampler(lines).stop()
    assert out["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"]
    hw = ("Active", "Not Active", "Not Active", "Not Active")
    assert _sampler([(11.0, _line(1965, reasons=hw))]).stop()["reasons"] == ["hw_slowdown"]


def test_clock_lines_that_do_not_parse_are_skipped():
    lines = [(11.0, "[N/A], 0"), (12.0, _line("[N/A]")), (13.0, _line(1700))]
    out = _sampler(lines).stop()
    assert out["samples"] == 1 and out["sm_mhz"] == 1700.0


def test_clock_without_samples_reports_none():
    out = _sampler([(1.0, _line(1900))]).stop()
    assert out["sm_mhz"] is None and out["samples"] == 0
    assert bench.ClockSampler(0).stop() is None  # nvidia-smi never started


def _copy_tree(tmp_path):
    csrc = tmp_path / "selective_state_space_42_b200" / "csrc"
    csrc.mkdir(parents=True)
    real = os.path.join(os.path.dirname(bench.__file__), "selective_state_space_42_b200", "csrc")
    for f in bench.KERNEL_SOURCES:
        shutil.copy(os.path.join(real, f), csrc / f)
    (tmp_path / "profiles").mkdir()
    return csrc


def _hash(csrc):
    import hashlib
    h = hashlib.sha256()
    for f in bench.KERNEL_SOURCES:
        h.update((csrc / f).read_bytes())
    return h.hexdigest()


def test_traffic_is_reported_only_for_the_sources_it_was_captured_on(tmp_path, monkeypatch):
    csrc = _copy_tree(tmp_path)
    prof = tmp_path / "profiles" / "scan.md"
    prof.write_text("# summary\nkernel_sources_sha256: %s\ntraffic_bytes_per_launch: 1234567\n"
                    % _hash(csrc))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "PROFILE", str(prof))
    assert bench.profiled_traffic() == 1234567
    with open(csrc / bench.KERNEL_SOURCES[0], "a") as f:
        f.write("\n// changed\n")
    assert bench.profiled_traffic() is None


def test_traffic_without_a_record_is_none(tmp_path, monkeypatch):
    _copy_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "PROFILE", str(tmp_path / "profiles" / "absent.md"))
    assert bench.profiled_traffic() is None
    prof = tmp_path / "profiles" / "nohash.md"
    prof.write_text("traffic_bytes_per_launch: 99\n")
    monkeypatch.setattr(bench, "PROFILE", str(prof))
    assert bench.profiled_traffic() is None


def test_committed_profile_carries_a_traffic_record():
    text = open(bench.PROFILE).read()
    keys = {ln.split(":", 1)[0] for ln in text.splitlines() if ":" in ln}
    assert {"kernel_sources_sha256", "traffic_bytes_per_launch"} <= keys


def test_default_launch_is_one_gpu_with_enough_warmup(monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py"])
    a = bench.parse_args()
    assert a.gpus == 1 and a.impl == "selscan"
    assert a.warmup >= 3 and a.steps >= 1


def test_job_rate_counts_every_rank():
    # 2 ranks x 10 steps x 1e9 elements in 4 ms (the slowest rank)
    assert bench.job_rate(10**9, 2, 10, 4.0) == pytest.approx(5e12)


def _run_bench(extra_env, *argv):
    env = dict(os.environ)
    env.update(extra_env)
    root = os.path.dirname(os.path.abspath(bench.__file__))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), *argv], env=env,
                         capture_output=True, text=True, timeout=300, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    return [json.loads(ln) for ln in out.stdout.splitlines() if ln.startswith("{")]


def test_reference_arm_prints_one_line_in_the_contract():
    """--impl reference times the float64 oracle on the host cores and prints
    one JSON line with the metric, unit and config of the GPU arm."""
    lines = _run_bench({"RANK": "0", "OMP_NUM_THREADS": "2"}, "--impl", "reference",
                       "--workload", "tiny_f32", "--steps", "2", "--warmup", "1",
                       "--cpu-seconds", "0.05")
    assert len(lines) == 1
    j = lines[0]
    assert j["impl"] == "reference" and j["metric"] == bench.METRIC and j["unit"] == bench.UNIT
    assert j["steps"] == 2 and j["warmup"] == 1 and j["higher_is_better"] is True
    assert j["value"] > 0 and j["ms_per_step"] > 0 and j["dtype"] == "f64"
    assert j["config"]["workload"] == "tiny_f32"
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == j["value"] and cb["cores"] >= 1
    assert "tiny_f32" in cb["sample"]
    assert j["e2e"] == {"value": j["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_runs_on_rank_zero_only():
    lines = _run_bench({"RANK": "1", "WORLD_SIZE": "2"}, "--impl", "reference",
                       "--workload", "tiny_f32", "--steps", "2", "--warmup", "1")
    assert lines == []


def test_cpu_sample_size_is_bounded():
    """The oracle's CPU-baseline sample: at least one channel, never more than
    the workload has, and a whole number of rounds of the host's threads when
    it is at least one round, so no thread idles in the timed pass."""
    from selective_state_space_42_b200 import workloads as wl
    w = wl.WORKLOADS["mamba2p8b_layer"]
    per_ch = w.seqlen * w.dstate
    for rate in (1e3, 1e6, 3e8, 1e9, 1e15):
        for seconds in (0.01, 10.0):
            for cores in (1, 8, 48):
                n = bench._sample_channels(w, rate, seconds, cores)
                assert 1 <= n <= w.dim
                if cores <= int(rate * seconds / per_ch) < w.dim:
                    assert n % cores == 0


def test_cpu_baseline_and_reference_share_one_sample():
    """cpu_baseline and the reference arm draw their sample from the same
    definition: a channel subset of batch row 0 for a short budget, whole
    rows (and repeated passes) for a long one; the elements it reports match
    the arrays it hands to the oracle."""
    from selective_state_space_42_b200 import workloads as wl
    w = wl.ScanWorkload("sample", 3, 64, 96, 16, "f32", gate=True, seed=3)
    inp = wl.make_scan_inputs(w)
    short = bench.oracle_sample(w, inp, 1e-9, 2)
    args, reps, per_pass, desc = short
    assert reps == 1 and args[0].shape[0] == 1 and args[0].shape[2] < w.dim
    assert per_pass == args[0].shape[0] * args[0].shape[2] * w.seqlen * w.dstate
    assert "batch row 0, channels 0.." in desc
    args, reps, per_pass, desc = bench.oracle_sample(w, inp, 1e3, 2)
    assert args[0].shape == (w.batch, w.seqlen, w.dim) and reps >= 1
    assert per_pass == w.elements
    cb = bench.oracle_cpu_baseline(inp, w, 1e-9)
    assert cb["kind"] == "oracle" and cb["value"] > 0 and "channels 0.." in cb["sample"]
