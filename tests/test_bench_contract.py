"""bench.py's reference arm (the oracle on the host cores) prints one JSON
line with the keys the benchmark contract fixes; it needs no GPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True and d["data"] == "synthetic"
    assert d["config"]["workload"] == "cogvideox2b_block_linears"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_clock_window_median_reasons_and_widening():
    """The clock record beside each timed figure: the median SM clock of the
    nvidia-smi samples inside the window, the union of the active throttle
    reasons, and, for a window shorter than the sampling interval, the
    samples of the 100 ms around it (marked as widened)."""
    sys.path.insert(0, ROOT)
    import bench
    cs = bench.ClockSampler(0)
    cs.samples = [(10.00, 1965.0, 1965.0, set()), (10.02, 1950.0, 1965.0, {"sw_power_cap"}),
                  (10.04, 1800.0, 1965.0, set()), (10.50, 1500.0, 1965.0, {"hw_slowdown"})]
    w = cs.window(9.99, 10.05)
    assert w == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "samples": 3, "reasons": ["sw_power_cap"]}
    w = cs.window(10.43, 10.44)          # no sample inside: widened by 100 ms on each side
    assert w["samples"] == 1 and w["sm_mhz"] == 1500.0 and w["window_widened_ms"] == 100
    assert w["reasons"] == ["hw_slowdown"]
    assert cs.window(20.0, 20.01) is None
    assert cs.window()["samples"] == 4   # no bounds: every sample


def test_clock_sampler_without_nvidia_smi(monkeypatch):
    """Where nvidia-smi cannot start, sampling yields no record instead of
    failing the run."""
    sys.path.insert(0, ROOT)
    import bench

    def no_smi(*a, **k):
        raise OSError("no nvidia-smi")
    monkeypatch.setattr(bench.subprocess, "Popen", no_smi)
    cs = bench.ClockSampler(0)
    cs.start()
    cs.stop()
    assert cs.samples == [] and cs.window(0.0, 1.0) is None
