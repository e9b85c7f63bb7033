"""Host-side pieces of bench.py (CPU only): the clock-sample summary that
decides whether a timed run is kept, and the oracle reference arm."""
import datetime
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class _Finished:
    def poll(self):
        return 0


def _summary_of(lines, t0, t1):
    s = bench.ClockSampler(0)
    try:
        with open(s.path, "w") as f:
            f.write("\n".join(lines) + "\n")
        s.proc = _Finished()               # stands in for a finished nvidia-smi process
        s.t0, s.t1 = t0, t1
        return s.summary()
    finally:
        os.remove(s.path)


def _row(ts, sm, reasons=("Not Active",) * 4):
    # timestamp, index, clocks.sm, clocks.max.sm, power.draw, active mask, 4 reason flags
    return ", ".join([ts.strftime("%Y/%m/%d %H:%M:%S.%f")[:-3], "0", str(sm), "1965", "900.5",
                      "0x0000000000000004", *reasons])


def test_clock_summary_keeps_samples_inside_the_timed_region():
    t0 = datetime.datetime(2026, 1, 1, 12, 0, 0)
    t1 = t0 + datetime.timedelta(seconds=1)
    lines = [_row(t0 - datetime.timedelta(seconds=3), 345),            # before: ignored
             _row(t0 + datetime.timedelta(milliseconds=10), 1950),
             _row(t0 + datetime.timedelta(milliseconds=500), 1845,
                  ("Not Active", "Not Active", "Not Active", "Active")),
             _row(t0 + datetime.timedelta(milliseconds=900), 1965),
             _row(t1 + datetime.timedelta(seconds=5), 210),            # after: ignored
             "garbage line"]
    out = _summary_of(lines, t0, t1)
    assert out["samples"] == 3
    assert out["sm_mhz"] == 1950
    assert out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"]


def test_clock_summary_reports_throttle_reasons_by_name():
    t0 = datetime.datetime(2026, 1, 1, 12, 0, 0)
    lines = [_row(t0, 1500, ("Active", "Not Active", "Active", "Not Active"))]
    out = _summary_of(lines, t0, t0)
    assert out["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_without_samples():
    t0 = datetime.datetime(2026, 1, 1, 12, 0, 0)
    out = _summary_of([], t0, t0)
    assert out["sm_mhz"] is None and out["reasons"] == ["no samples"]


def test_reference_arm_prints_one_json_line():
    """`bench.py --impl reference` times the oracle on this host's cores and
    prints the contract's line with impl, cpu_baseline and e2e."""
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_sampler_left_running_is_killed_at_exit():
    """A run that raises between start() and stop() must not leave an endless
    sampler behind: the exit hook kills it and removes the sample file."""
    s = bench.ClockSampler(0)
    s.proc = subprocess.Popen(["sleep", "60"])     # stands in for nvidia-smi -lms
    assert os.path.exists(s.path) and s.proc.poll() is None
    s._cleanup()
    assert s.proc.poll() is not None and not os.path.exists(s.path)
    s._cleanup()                                   # a second call (the real exit) is harmless
