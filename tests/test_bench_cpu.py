"""The bench's host-side contract, on CPU: the reference arm's JSON line (the oracle timed on
host cores), rank handling under a multi-rank launch, the warm-up floor, the clock summary
taken during the timed region, the whole-job throughput arithmetic, and the host
bookkeeping timing (allocator and prefix cache through the binding)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _run(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_one_contract_line():
    p = _run(["--impl", "reference", "--workload", "tiny", "--steps", "4", "--warmup", "3"])
    assert p.returncode == 0, p.stderr
    lines = [l for l in p.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    j = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "impl", "cpu_baseline", "e2e"):
        assert key in j, key
    assert j["impl"] == "reference" and j["metric"] == bench.METRIC and j["unit"] == "GB/s"
    assert j["value"] > 0 and j["steps"] == 4 and j["warmup"] == 3 and j["n_gpus"] == 1
    assert j["higher_is_better"] is True and j["dtype"] == "f64"
    assert j["config"]["workload"] == bench.DESCR["tiny"]
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == j["value"] and cb["sample"]
    assert j["e2e"] == {"value": j["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    p = _run(["--impl", "reference", "--workload", "tiny", "--steps", "3", "--warmup", "3"],
             {"WORLD_SIZE": "2", "RANK": "1"})
    assert p.returncode == 0 and p.stdout.strip() == ""


def test_warmup_floor():
    p = _run(["--impl", "reference", "--workload", "tiny", "--steps", "3", "--warmup", "2"])
    assert p.returncode != 0 and "--warmup must be >= 3" in p.stderr


def test_clock_summary():
    cs = bench.ClockSampler(0)
    # timestamp, clocks.sm, clocks.max.sm, power.draw, clocks_event_reasons.active
    cs.samples = [(0.5, "t, 1100, 1965, 300.0, 0x0000000000000001"),
                  (1.0, "t, 1965, 1965, 900.5, 0x0000000000000000"),
                  (1.2, "t, 1900, 1965, 1000.0, 0x0000000000000004"),
                  (1.4, "t, 1950, 1965, 990.0, 0x0000000000000000"),
                  (1.6, "garbled"),
                  (9.0, "t, 300, 1965, 100.0, 0x0000000000000048")]
    s = cs.summary(0.9, 1.5)
    assert s["samples"] == 3 and s["sm_mhz"] == 1950.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["note"] == "inside timed region"
    # a timed region shorter than the sampling period takes the nearest samples
    s = cs.summary(8.9, 8.95)
    assert s["note"].startswith("nearest") and "hw_slowdown" in s["reasons"] \
        and "hw_thermal_slowdown" in s["reasons"]
    # idle is never reported as a reason
    assert "gpu_idle" not in cs.summary(0.0, 0.6)["reasons"]
    empty = bench.ClockSampler(0)
    assert empty.summary(0.0, 1.0)["sm_mhz"] is None


def test_job_throughput_and_slowest_rank():
    # 2 ranks, 1 GB per rank-step, 10 steps, slowest rank 4 s -> 5 GB/s for the job
    assert bench.job_throughput(10 ** 9, 10, 2, 4.0) == pytest.approx(5.0)
    assert bench.slowest_rank_seconds(1.25) == 1.25


def test_host_bookkeeping_timing():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_pa_build", os.path.join(ROOT, "paged_kv_cache_465_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import paged_kv_cache_465_b200 as pa
    h = bench._host_bookkeeping(pa, steps=3)
    assert h["num_seqs"] == 256 and h["unit"] == "us"
    assert h["append_batch_us_per_step"] > 0 and h["append_us_per_step"] > 0
    assert h["add_seq_tokens_us_per_request"] > 0
    assert h["prefix_cached_tokens"] == 99 * 192     # 12 full blocks reused per later request


def test_nvml_clock_summary_inside_timed_region_and_window():
    import numpy as np
    c = bench.NvmlClocks(None, 0)
    c.ok, c.max_mhz = True, 1965.0
    # (time, SM MHz, clock-event reason bits)
    c.samples = [(0.9, 700.0, 0x1), (1.0, 1965.0, 0x0), (1.002, 1950.0, 0x4), (1.5, 1000.0, 0x1),
                 (2.0, 1965.0, 0x0), (2.1, 1965.0, 0x0), (3.0, 500.0, 0x1)]
    s = c.summary((1.0, 1.003), (2.0, 2.2))
    assert s["samples"] == 4 and s["sm_mhz"] == float(np.median([1965, 1950, 1965, 1965]))
    assert s["sm_mhz_timed"] == float(np.median([1965, 1950]))
    assert s["reasons"] == ["sw_power_cap"] and s["sm_max_mhz"] == 1965.0
    assert s["note"].startswith("inside timed region: 2 NVML samples")


def test_parity_stats_pass_and_catch_a_dropped_term():
    import numpy as np
    rng = np.random.default_rng(0)
    ref = rng.standard_normal((5, 4, 8)) * 0.1
    lse = rng.standard_normal((5, 4))
    got = ref + 1e-4
    p = bench.parity_stats(got, lse + 1e-4, ref, lse, "bf16", [1, 3])
    assert p["ok"] and p["seqs"] == [1, 3] and abs(p["max_abs"] - 1e-4) < 1e-12
    bad = got.copy()
    bad[3, 2] = 0.0                       # one head's output lost
    assert not bench.parity_stats(bad, lse, ref, lse, "bf16", [1, 3])["ok"]
    assert not bench.parity_stats(got, lse + 1e-2, ref, lse, "bf16", [1, 3])["ok"]
    lse_inf = lse.copy()
    lse_inf[1, 0] = -np.inf               # an empty row must stay empty
    assert not bench.parity_stats(got, lse, ref, lse_inf, "bf16", [1, 3])["ok"]
