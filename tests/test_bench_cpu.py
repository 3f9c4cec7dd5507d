"""bench.py's host-side pieces on the CPU: the module imports, the peak table
loads, and the CPU baseline (the oracle on a bounded row sample) runs and
reports a positive rate."""
import importlib.util
import os
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_bench_imports_and_peaks():
    b = _bench()
    peaks = b.load_peaks()
    assert peaks["hbm_gbs"] > 0 and peaks["bf16_tflops"] > 0 and peaks["bf16_tflops_sustained"] > 0
    assert peaks["source"] in ("measured", "fallback")
    assert set(b.KERNEL_NAMES) >= {3, 4, 6}


def test_cpu_baseline_sample():
    """All host threads, then one thread: both rates positive, the thread
    counts and the CPU model reported."""
    b = _bench()
    got = b.cpu_sample(budget_s=0.2, min_rows=1, workload="llama32-1b", one_core_s=0.5)
    assert got["value"] > 0 and got["cores"] >= 1 and got["kind"] == "oracle"
    assert "oracle" in got["sample"] and "token rows" in got["sample"]
    assert got["cpu_model"] and got["nproc"] >= 1
    assert got["value_1core"] > 0 and "1 thread" in got["sample_1core"]


def test_peak_choice_and_roofline():
    """Burst peak for a short timed region, sustained only for a long one
    under the power cap; the roofline's achieved rate is the kept-weight work
    of the step over the step time."""
    b = _bench()
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "source": "measured", "hbm_gbs": 1.0}
    hi = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0}
    lo = {"sm_mhz": 1515.0, "sm_max_mhz": 1965.0}
    assert b.choose_peak(peaks, 0.3, dict(hi, reasons=["sw_power_cap"]))[0] == 1600.0
    assert b.choose_peak(peaks, 5.0, dict(lo, reasons=[]))[0] == 1600.0
    assert b.choose_peak(peaks, 5.0, dict(hi, reasons=["sw_power_cap"]))[0] == 1400.0
    assert b.choose_peak(peaks, 0.3, dict(lo, reasons=["sw_power_cap"]))[0] == 1400.0
    assert b.choose_peak(peaks, 0.3, {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]})[0] == 1600.0

    class Info:
        pruned, slabs_total, slabs_pair_sparse, packed_bytes = 64 * 128, 4, 1, 0
        tiles_sparse, tile_rows, tile_cols = 1, 128, 128

    m = b.Member(None, 256, 128, Info(), None, None)
    assert m.kept == 128 * 256 - 64 * 128 and m.executed == 3 * 8192 + 4096
    model = [(None, [m, m])]
    r = b.roofline(model, 10, 2.0, 4, 1600.0, "burst", "k", None, peaks)
    assert abs(r["achieved"] - 2 * 2.0 * 10 * m.kept / 2e-3 / 1e12) < 1e-12
    assert abs(r["frac"] - r["achieved"] / 1600.0) < 1e-15 and r["kernel_ms_per_launch"] == 0.5
    assert abs(r["frac_of_sustained"] - r["achieved"] / 1400.0) < 1e-15


def test_measured_traffic_is_pinned_to_source():
    import hashlib
    b = _bench()
    for name, t in b.MEASURED_TRAFFIC.items():
        with open(os.path.join(ROOT, t["source"]), "rb") as f:
            same = hashlib.sha256(f.read()).hexdigest()[:16] == t["sha256"]
        got = b.measured_traffic(name + " (any label)", t["workload"])
        assert (got == t["bytes_per_launch"]) if same else (got is None)
        assert b.measured_traffic(name, ("llama32-1b", 4096, "128x128")) is None
    assert b.measured_traffic("some_other_kernel") is None


def test_reference_arm_line():
    """--impl reference prints one JSON line on the same metric, unit and
    direction as the GPU arm, from the CPU oracle."""
    import json
    import subprocess
    import sys
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    b = _bench()
    assert line["impl"] == "reference" and line["metric"] == b.METRIC
    assert line["unit"] == "TFLOP/s" and line["higher_is_better"] is True and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_clock_sampler_summary():
    """The clock record: median SM clock under load, the throttle reasons that
    were active, samples below 300 W left out; the temporary file is removed."""
    import sys
    b = _bench()
    script = ("import time\n"
              "rows = ['0, 100, 1965, 80.0, 0x0, Not Active, Not Active, Not Active, Not Active',\n"
              "        '0, 1700, 1965, 650.0, 0x4, Not Active, Not Active, Not Active, Active',\n"
              "        '0, 1800, 1965, 700.0, 0x4, Not Active, Not Active, Not Active, Active']\n"
              "for r in rows * 400:\n"
              "    print(r, flush=True)\n"
              "    time.sleep(0.01)\n")
    with b.ClockSampler(0, cmd=[sys.executable, "-c", script]) as c:
        time.sleep(0.5)
    got = c.summary()
    assert got["sm_mhz"] in (1700.0, 1750.0, 1800.0) and got["sm_max_mhz"] == 1965.0
    assert got["reasons"] == ["sw_power_cap"] and got["power_w_max"] == 700.0
    assert not os.path.exists(c.path)
    with b.ClockSampler(0, cmd=["/nonexistent/nvidia-smi"]) as c:
        pass
    assert c.summary()["sm_mhz"] is None
