"""bench.py's host-side contract, on the CPU: the reference arm (the CPU
oracle on bounded samples) prints one JSON line with the required keys and
only on rank 0, and the figures the native arm reports are derived from the
workload as stated (no GPU involved)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from token_sparse_attention_sm_b200 import synth  # noqa: E402


def _run(args, env_extra=None, timeout=300):
    env = dict(os.environ)
    env.update(env_extra or {})
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                       env=env, capture_output=True, text=True, timeout=timeout)
    return r


def test_reference_arm_prints_one_contract_line():
    r = _run(["--impl", "reference", "--workload", "tiny_f32", "--steps", "2",
              "--warmup", "3"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["unit"] == "steps/s" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] == 3
    assert abs(d["ms_per_step"] - 1e3 / d["value"]) <= 1e-3 * d["ms_per_step"] + 1e-3
    assert d["config"]["workload"] == "tiny_f32"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert cb["unit"] == "steps/s" and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "steps/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    r = _run(["--impl", "reference", "--workload", "tiny_f32", "--steps", "1",
              "--warmup", "3"], {"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_warmup_below_three_is_refused():
    r = _run(["--impl", "reference", "--workload", "tiny_f32", "--steps", "1",
              "--warmup", "2"])
    assert r.returncode != 0


def test_algorithmic_bytes_of_the_headline_step():
    """The K cache once plus the selected K and V rows once: 268,435,456 +
    8,388,608 = 276,824,064 bytes per step at 128K, k = 2048, bf16."""
    scan, gathered = bench.algorithmic_bytes(synth.WORKLOADS["decode_128k"])
    assert scan == 268_435_456 and gathered == 8_388_608


def test_kernels_per_step():
    w = synth.WORKLOADS["decode_128k"]
    assert bench.kernels_per_step(w) == 2                     # scan, select + attention
    assert bench.kernels_per_step(w, reroute=1) == 2 * w.L     # per-layer routing
    assert bench.kernels_per_step(w, reroute=5) == 2 * 4       # ceil(16 / 5) groups
    assert bench.kernels_per_step(synth.WORKLOADS["tiny_f32"]) == 4  # fp32: select, partial, merge
    assert bench.kernels_per_step(synth.WORKLOADS["threshold_128k"]) == 2
    big = w.with_(N=262144)
    assert bench.kernels_per_step(big) == 3                   # select as a kernel of its own


def test_peak_denominator_is_the_measured_copy_bandwidth():
    gbs, src = bench.load_peaks()
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            assert gbs == pytest.approx(float(json.load(f)["hbm_gbs"]))
        assert src.startswith("measured")
    else:
        assert gbs == bench.FALLBACK_HBM_GBS and src.startswith("fallback")


def _smi_row(t, sm, mx=1965, hw="Not Active", thermal="Not Active", cap="Not Active"):
    from datetime import datetime
    stamp = datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    return f"{stamp}, {sm}, {mx}, 700.5, 0x0000000000000000, {hw}, {thermal}, Not Active, {cap}"


def test_clock_summary_of_the_timed_region():
    """Only rows stamped inside the timed region count; the SM clock is their
    median, the max clock the largest seen, and a reason is reported when any
    row shows it Active."""
    t0 = 1_700_000_000.0
    rows = [_smi_row(t0 - 1.0, 345, cap="Active"),          # before the region
            _smi_row(t0 + 0.1, 1965),
            _smi_row(t0 + 0.2, 1900, cap="Active"),
            _smi_row(t0 + 0.3, 1950),
            _smi_row(t0 + 2.0, 210, hw="Active")]           # after it
    c = bench.summarize_clocks("\n".join(rows), t0, t0 + 0.5)
    assert c == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                 "samples": 3}
    c = bench.summarize_clocks("\n".join(rows))              # no region: every row
    assert c["samples"] == 5 and c["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert bench.summarize_clocks("", t0, t0 + 1) is None
    assert bench.summarize_clocks("garbage,row\n", t0, t0 + 1) is None
