"""The benchmark's one-line JSON contract, on the tiny workload: the GPU arm's
line carries the metric, timing, roofline, end-to-end, clocks, launch count
and CPU-oracle baseline; the reference arm (the oracle, on the host, so that
test needs no GPU) prints the same metric with impl "reference"."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args):
    r = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    return json.loads(lines[0])


@pytest.mark.gpu
def test_gpu_arm_line():
    d = run_bench("--workload", "tiny", "--steps", "5", "--warmup", "3", "--e2e-steps", "2", "--cpu-budget", "1")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks",
                "cpu_baseline"):
        assert key in d, key
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["n_gpus"] == 1 and d["steps"] == 5
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["dtype"] == "bf16"
    assert d["config"]["workload"] == "tiny"
    rl = d["roofline"]
    assert rl["bound"] == "hbm" and rl["unit"] == "GB/s" and rl["peak"] > 0 and rl["achieved"] > 0
    assert abs(rl["frac"] - rl["achieved"] / rl["peak"]) < 1e-3
    e2e = d["e2e"]
    assert e2e["value"] > 0 and e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] == 4 * 5
    assert d["graph"]["ms_per_step"] > 0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["cores"] >= 1 and cb["sample"]


def test_reference_arm_line():
    d = run_bench("--impl", "reference", "--workload", "tiny", "--steps", "3", "--warmup", "3")
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_clock_summary_and_note():
    """The clock record of a run (host logic, canned samples): only samples
    inside the timed window count when there are any; the reasons are the
    union of the samples' reasons; the one-line note of --table / --variants
    reports the median and the reasons."""
    sys.path.insert(0, ROOT)
    import bench

    class Canned(bench.ClockSampler):
        def __init__(self, samples):
            self.samples, self.max_mhz, self.source = samples, 1965.0, "canned"

        def stop(self):
            pass

    s = Canned([(0.5, 1965.0, [], 200.0), (1.0, 1800.0, ["sw_power_cap"], 500.0), (2.0, 1700.0, [], 480.0),
                (9.0, 1000.0, ["hw_slowdown"], 100.0)])
    c = s.summary(0.9, 2.1)
    assert c["samples"] == 2 and c["in_timed_window"] is True
    assert c["sm_mhz"] == 1750.0 and c["sm_mhz_min"] == 1700.0 and c["sm_mhz_max"] == 1800.0
    assert c["reasons"] == ["sw_power_cap"] and c["power_w_max"] == 500.0
    outside = s.summary(3.0, 4.0)  # no sample inside: every sample counts, flagged as such
    assert outside["samples"] == 4 and outside["in_timed_window"] is False
    assert outside["reasons"] == ["hw_slowdown", "sw_power_cap"]
    note = bench.clock_note(s)
    assert "median 1750 MHz" in note and "hw_slowdown" in note and "4 samples" in note
    assert "not sampled" in bench.clock_note(Canned([]))
