#!/usr/bin/env python
"""Paged decode attention on B200: KV-read GB/s (% of HBM peak) and decode tokens/s.

One step = one decode step of the workload through the library: copy-on-write block copies
(shared-prefix workload only), the slot-mapped write of this step's new K/V, and decode
attention over the paged cache (split into partitions + log-sum-exp reduce where the
workload says so). Inputs are resident in HBM when the timed region starts; L2 is flushed
(a write of twice its size) between timed steps, outside the timed events.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload b256] [--impl ours|reference]

N > 1 runs under torchrun: every rank runs an independent replica of the workload (decode
has no exchange step; there is no collective on the data path), ``value`` counts the KV
bytes of all ranks over the slowest rank's time ("weak" scaling).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "paged decode attention KV GB/s (% of HBM peak) and decode tokens/s at 1 B200"
UNIT = "GB/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
DTYPE = {"f32": "f32", "bf16": "bf16-kv/f32-acc", "fp8": "fp8e4m3-kv/f32-acc",
         "int8": "int8-kv/f32-acc"}
DESCR = {
    "tiny": "tiny paged decode: 4 seqs ctx {5,16,17,40}, 4q/2kv, d64, fp32",
    "b32": "decode batch 32: ctx U[1,4096], 32q/8kv, d128, bf16 KV",
    "shared": "shared prefix: 100 seqs x (200 shared + 50 private), 32q/8kv, d128, bf16, CoW",
    "b256": "decode batch 256: ctx lognormal(1024,1) clip [16,8192], 32q/8kv, d128, fp8-e4m3 KV",
    "long": "long context: 8 seqs x 131072, 64q/8kv, d128, bf16 KV, split-KV 512",
    "b256_int8": "decode batch 256 with an int8 KV cache (scale + zero point per block, kv head)",
}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------------------
_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.proc = None

    def __enter__(self):
        q = "timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active"
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", str(self.index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        rows = []
        for ts, line in self.samples:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 5:
                continue
            try:
                rows.append((ts, float(parts[1]), float(parts[2]), int(parts[4], 16)))
            except ValueError:
                continue
        inside = [r for r in rows if t0 <= r[0] <= t1]
        note = "inside timed region"
        if not inside and rows:
            inside = sorted(rows, key=lambda r: min(abs(r[0] - t0), abs(r[0] - t1)))[:3]
            note = "nearest samples (timed region shorter than the sampling period)"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "nvidia-smi unavailable"}
        mask = 0
        for r in inside:
            mask |= r[3]
        reasons = [n for b, n in _REASONS.items() if mask & b and n != "gpu_idle"]
        return {"sm_mhz": float(np.median([r[1] for r in inside])), "sm_max_mhz": inside[0][2],
                "reasons": reasons, "samples": len(inside), "note": note}


class NvmlClocks:
    """SM clock and clock-event reasons read through NVML (read-only queries) every
    ``period`` seconds on a thread, so that a timed region of a few milliseconds still has
    samples inside it. Falls back to ``ClockSampler`` (nvidia-smi) when NVML is missing."""

    def __init__(self, torch, device_index: int, period: float = 0.001):
        self.torch, self.index, self.period = torch, device_index, period
        self.samples = []
        self.ok = False
        self._stop = threading.Event()

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            uuid = str(self.torch.cuda.get_device_properties(self.index).uuid)
            try:
                self.h = nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-")
                                                      else "GPU-" + uuid)
            except Exception:  # noqa: BLE001
                self.h = nv.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM))
            self.ok = True
        except Exception:  # noqa: BLE001
            self.fallback = ClockSampler(self.index).__enter__()
            return self
        self.thread = threading.Thread(target=self._poll, daemon=True)
        self.thread.start()
        time.sleep(0.05)
        return self

    def _poll(self):
        nv = self.nv
        reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append((time.time(), float(nv.nvmlDeviceGetClockInfo(
                    self.h, nv.NVML_CLOCK_SM)), int(reasons(self.h))))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __exit__(self, *a):
        if not self.ok:
            self.fallback.__exit__(*a)
            return
        self._stop.set()
        self.thread.join(timeout=5)
        try:
            self.nv.nvmlShutdown()
        except Exception:  # noqa: BLE001
            pass

    def summary(self, timed, window=None):
        """Clocks over the timed region (t0, t1) and a loaded window right after it."""
        if not self.ok:
            return self.fallback.summary(*timed)
        inside = [r for r in self.samples if timed[0] <= r[0] <= timed[1]]
        win = [r for r in self.samples if window and window[0] <= r[0] <= window[1]]
        rows = inside + win
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "note": "no NVML samples"}
        mask = 0
        for r in rows:
            mask |= r[2]
        reasons = [n for b, n in _REASONS.items() if mask & b and n != "gpu_idle"]
        note = f"inside timed region: {len(inside)} NVML samples (every {self.period * 1e3:g} ms)"
        if window:
            note += (f"; plus {len(win)} in a {1e3 * (window[1] - window[0]):.0f} ms loaded "
                     f"window of the same steps right after it")
        return {"sm_mhz": float(np.median([r[1] for r in rows])), "sm_max_mhz": self.max_mhz,
                "sm_mhz_timed": float(np.median([r[1] for r in inside])) if inside else None,
                "reasons": reasons, "samples": len(rows), "note": note}


# ---------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------
def _time_steps(torch, sc, steps: int, flush, per_step_events: bool = True):
    """Device time of `steps` steps with an L2 flush between them (outside the events);
    also the device time of the decode call alone inside each step."""
    st = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush()
        a, b, c = ev[i]
        a.record(st)
        if sc.pairs is not None:
            sc.cache.copy(sc.pairs)
        sc.cache.write(sc.step_k, sc.step_v, sc.step_slots)
        b.record(st)
        sc.cache.decode(sc.q, sc.block_tables, sc.context_lens, sc.scale, sc.out,
                        max_context_len=sc.max_context_len, partition_size=sc.partition_size,
                        lse_out=sc.lse, workspace=sc.workspace)
        c.record(st)
    torch.cuda.synchronize()
    total = sum(a.elapsed_time(c) for a, b, c in ev) / 1e3
    dec = [b.elapsed_time(c) / 1e3 for a, b, c in ev]
    return total, float(np.mean(dec))


def _e2e(torch, sc, steps: int, flush, l2_bytes: int):
    """The same steps through the public API from pinned host buffers, pipelined as a
    serving loop would run them: two sets of device inputs, the H2D copies of step i+1's
    inputs on a second stream while step i runs, and the D2H read of every step's output on
    that stream. The timed region is the device time from before the first copy to after
    the last read-back. Returns (seconds, H2D bytes per step, D2H bytes per step, note)."""
    main = torch.cuda.current_stream()
    cs = torch.cuda.Stream()
    names = ("q", "step_k", "step_v", "step_slots", "block_tables", "context_lens")
    host = {n: getattr(sc, n).cpu().pin_memory() for n in names}
    if sc.pairs is not None:
        host["pairs"] = sc.pairs.cpu().pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    sets = []
    for _ in range(2):
        d = {n: torch.empty_like(t, device="cuda") for n, t in host.items()}
        d["out"], d["lse"] = torch.empty_like(sc.out), torch.empty_like(sc.lse)
        d["out_h"] = torch.empty(sc.out.shape, dtype=sc.out.dtype).pin_memory()
        sets.append(d)
    d2h = sets[0]["out_h"].numel() * sets[0]["out_h"].element_size()
    # each step reads more KV than L2 holds: no flush; else flush before each step (timed)
    small = sc.step_bytes()["kv"] < 2 * l2_bytes
    ready = [torch.cuda.Event(), torch.cuda.Event()]

    def copy_in(i):
        b = sets[i % 2]
        with torch.cuda.stream(cs):
            for n, t in host.items():
                b[n].copy_(t, non_blocking=True)
            ready[i % 2].record(cs)

    c = sc.cache
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(main)
    cs.wait_stream(main)
    copy_in(0)
    for i in range(steps):
        if i + 1 < steps:
            copy_in(i + 1)  # into the other set, after its previous read-back on this stream
        b = sets[i % 2]
        main.wait_event(ready[i % 2])
        if small:
            flush()
        if sc.pairs is not None:
            c.copy(b["pairs"])
        c.write(b["step_k"], b["step_v"], b["step_slots"])
        c.decode(b["q"], b["block_tables"], b["context_lens"], sc.scale, b["out"],
                 max_context_len=sc.max_context_len, partition_size=sc.partition_size,
                 lse_out=b["lse"], workspace=sc.workspace)
        done = torch.cuda.Event()
        done.record(main)
        with torch.cuda.stream(cs):
            cs.wait_event(done)
            b["out_h"].copy_(b["out"], non_blocking=True)
    main.wait_stream(cs)
    end.record(main)
    torch.cuda.synchronize()
    assert torch.equal(sets[(steps - 1) % 2]["out"], sc.out)  # the same step's result
    note = ("pipelined: step i+1's H2D copies on a second stream while step i runs, D2H of "
            "every step's out on that stream; L2 " +
            ("flushed before every step (inside the timed region)" if small else
             "not flushed (each step reads more KV than L2 holds)"))
    return start.elapsed_time(end) / 1e3, h2d, d2h, note


def _host_bookkeeping(pa, steps: int = 100):
    """Host side of the step, through the Python binding: the allocator's bookkeeping for
    one new token per sequence of the batch-256 workload (its context lengths, 16-token
    blocks), as one append_batch call per step and, for comparison, one append call per
    sequence; and the prefix cache on the shared-system-prompt example (100 requests of one
    200-token prompt plus 50 private tokens each), one add_seq_tokens call per request."""
    wl = workloads.WORKLOADS["b256"]
    lens = [int(x) - 1 for x in workloads.draw(wl).context_lens]
    ids = np.arange(len(lens), dtype=np.int32)  # the running batch, as a serving loop holds it
    out = {"unit": "us", "threads": 1, "num_seqs": len(lens)}
    for how in ("append_batch", "append"):
        a = pa.BlockAllocator(wl.num_blocks, 16)
        for s, n in zip(ids.tolist(), lens):
            a.add_seq(s, n)
        t0 = time.perf_counter()
        for _ in range(steps):
            if how == "append_batch":
                a.append_batch(ids, 1)
            else:
                for s in ids.tolist():
                    a.append(s, 1)
        dt = (time.perf_counter() - t0) / steps
        out[f"{how}_us_per_step"] = round(dt * 1e6, 2)
    rng = np.random.default_rng(2)
    prompt = rng.integers(0, 32000, 200).tolist()
    reqs = [prompt + rng.integers(0, 32000, 50).tolist() for _ in range(100)]
    a = pa.BlockAllocator(512, 16)
    t0 = time.perf_counter()
    cached = sum(a.add_seq_tokens(r, toks)[1] for r, toks in enumerate(reqs))
    dt = (time.perf_counter() - t0) / len(reqs)
    out["add_seq_tokens_us_per_request"] = round(dt * 1e6, 2)
    out["prefix_cached_tokens"] = int(cached)
    out["steps"] = steps
    out["note"] = ("host time per decode step next to the device step; one call per step "
                   "(append_batch) against one call per sequence (append)")
    return out


# Parity bars on the decode output per KV storage type: (max-abs, relative-L2 per (sequence,
# head), lse), the same as the GPU parity tests use
PARITY_BARS = {"f32": (1e-4, 1e-5, 1e-3), "bf16": (2e-2, 1e-2, 1e-3), "fp8": (3e-2, 3e-2, 1e-3),
               "int8": (3e-2, 3e-2, 1e-3)}


def oracle_sample(wl, n: int = 8):
    """The sequences the CPU-baseline leg recomputes (their K/V come from the seeded draw in
    the GPU run too)."""
    rng = np.random.default_rng(0)
    return sorted(rng.choice(wl.num_seqs, size=min(wl.num_seqs, n), replace=False).tolist())


def parity_stats(got_out, got_lse, ref_out, ref_lse, kv_dtype, seqs):
    """Errors of the GPU's decode output against the oracle's on the sampled sequences."""
    o, ro = got_out[seqs], ref_out[seqs]
    err = np.abs(o - ro)
    rel = np.sqrt((err ** 2).sum(-1)) / np.maximum(np.sqrt((ro ** 2).sum(-1)), 1e-30)
    fin = np.isfinite(ref_lse[seqs])
    lse = np.abs(got_lse[seqs][fin] - ref_lse[seqs][fin])
    bars = PARITY_BARS[kv_dtype]
    res = {"max_abs": float(err.max()), "rel_l2": float(rel.max()),
           "lse": float(lse.max()) if lse.size else 0.0, "seqs": [int(s) for s in seqs],
           "bars": {"max_abs": bars[0], "rel_l2": bars[1], "lse": bars[2]}}
    res["ok"] = bool(res["max_abs"] <= bars[0] and res["rel_l2"] <= bars[1]
                     and res["lse"] <= bars[2]
                     and np.array_equal(np.isfinite(got_lse[seqs]), np.isfinite(ref_lse[seqs])))
    return res


def _cpu_baseline(draw, seconds: float = 12.0, gpu=None):
    """The oracle, as it stands, on the host cores: this step's cache write plus decode for a
    bounded sample of the workload's sequences (cycled until ~`seconds` elapse). ``gpu``:
    (out, lse) of the GPU's last step as float64 arrays; the oracle's outputs for the
    sampled sequences (whose K/V the GPU run took from the same draw) are compared with
    them after the timing."""
    from oracle import flows, paged as opaged, attention
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # noqa: BLE001
        cores = os.cpu_count()
    wl = draw.wl
    sample = oracle_sample(wl)
    st = flows.build_state(draw, write_seqs=sample)
    sc = float(np.float32(1.0 / math.sqrt(wl.head_dim)))
    es = {"f32": 4, "bf16": 2, "fp8": 1, "int8": 1}[wl.kv_dtype]
    done_bytes = 0
    outs = {}
    t0 = time.perf_counter()
    i = 0
    while True:
        s = sample[i % len(sample)]
        k, v = draw.kv(s)
        opaged.ref_reshape_and_cache(k[-1:], v[-1:], st.k_cache, st.v_cache, st.step_slots[s],
                                     wl.in_dtype, wl.kv_dtype, st.k_scales, st.v_scales,
                                     st.k_zeros, st.v_zeros)
        r = attention.ref_decode(draw.q, st.k_cache, st.v_cache, st.block_tables,
                                 st.context_lens, sc, wl.num_kv_heads, wl.in_dtype, wl.kv_dtype,
                                 st.k_scales, st.v_scales, seqs=[s], k_zeros=st.k_zeros,
                                 v_zeros=st.v_zeros)
        outs.setdefault(s, r)
        done_bytes += int(draw.context_lens[s]) * 2 * wl.num_kv_heads * wl.head_dim * es
        i += 1
        el = time.perf_counter() - t0
        if el >= seconds and i >= len(sample):
            break
    res = {"value": done_bytes / el / 1e9, "unit": UNIT, "cores": int(cores), "kind": "oracle",
           "sample": f"{i} (seq, all heads) decode steps cycling over {len(sample)} of "
                     f"{wl.num_seqs} sequences of the same workload, float64 NumPy, "
                     f"{el:.1f} s"}
    if gpu is not None:
        ref_out = np.full(gpu[0].shape, np.nan)
        ref_lse = np.full(gpu[1].shape, np.nan)
        for s, (o, l) in outs.items():
            ref_out[s], ref_lse[s] = o[s], l[s]
        res["parity"] = parity_stats(gpu[0], gpu[1], ref_out, ref_lse, wl.kv_dtype, sample)
    return res


def slowest_rank_seconds(seconds: float, dist=None, device="cpu") -> float:
    """Device time of the slowest rank (max over ranks); identity without a process group.
    Every rank must call it the same number of times."""
    if dist is None:
        return float(seconds)
    import torch
    t = torch.tensor([float(seconds)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_rank_step: int, steps: int, world: int, slowest_s: float) -> float:
    """Whole-job GB/s: every rank's bytes over the slowest rank's time (weak scaling)."""
    return world * bytes_per_rank_step * steps / slowest_s / 1e9


def run_profile(args):
    """Warm-up and timed steps of one workload only (decode or prefill), nothing else: the
    command the ncu summaries under profiles/ capture. Prints one short JSON line."""
    import torch
    import paged_kv_cache_465_b200 as pa
    from paged_kv_cache_465_b200.scenario import DeviceScenario, PrefillScenario
    torch.cuda.set_device(0)
    pa.set_decode_impl(args.decode_impl)
    kw = {"num_seqs": args.seqs} if args.seqs else {}
    if args.workload in workloads.PREFILL_WORKLOADS:
        wl = workloads.PREFILL_WORKLOADS[args.workload].scaled(**kw)
        sc = PrefillScenario(workloads.draw_prefill(wl), draw_seqs=[])
    else:
        wl = workloads.WORKLOADS[args.workload].scaled(**kw)
        sc = DeviceScenario(workloads.draw(wl), draw_seqs=[], partition_size=args.partition)
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    flush_buf = torch.empty(max(2 * l2, 64 << 20) // 4, dtype=torch.float32, device="cuda")
    for i in range(args.warmup + args.steps):
        flush_buf.fill_(1.0)
        if i == args.warmup:
            torch.cuda.synchronize()
            t0 = time.perf_counter()
        sc.step()
    torch.cuda.synchronize()
    err = pa.device_error()
    print(json.dumps({"profile": args.workload, "steps": args.steps, "warmup": args.warmup,
                      "wall_ms_per_step": round((time.perf_counter() - t0) / args.steps * 1e3, 4),
                      "device_error": err}), flush=True)
    if err:
        raise SystemExit(1)


def run_ours(args):
    import torch
    from paged_kv_cache_465_b200.scenario import DeviceScenario
    import paged_kv_cache_465_b200 as pa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    pa.set_decode_impl(args.decode_impl)
    wl = workloads.WORKLOADS[args.workload]
    draw = workloads.draw(wl)
    # the sequences the CPU-baseline leg recomputes take their K/V from the seeded draw (the
    # others get the same distribution drawn on the device)
    parity_seqs = oracle_sample(wl) if (world == 1 and not args.no_cpu_baseline) else []
    sc = DeviceScenario(draw, draw_seqs=parity_seqs, partition_size=args.partition)
    l2 = torch.cuda.get_device_properties(local).L2_cache_size
    flush_buf = torch.empty(max(2 * l2, 64 << 20) // 4, dtype=torch.float32, device="cuda")

    def flush():
        flush_buf.fill_(1.0)

    for _ in range(args.warmup):
        flush()
        sc.step()
    torch.cuda.synchronize()
    assert pa.device_error() == 0
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with NvmlClocks(torch, local) as clk:
        t_wall0 = time.time()
        total, dec_mean = _time_steps(torch, sc, args.steps, flush)
        t_wall1 = time.time()
        # untimed: the same steps for a loaded window of ~0.3 s, for the clock record
        w0 = time.time()
        while time.time() - w0 < 0.3:
            for _ in range(50):
                flush()
                sc.step()
            torch.cuda.synchronize()
        w1 = time.time()
    total = slowest_rank_seconds(total, dist, "cuda")
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    ms = total / args.steps * 1e3
    b = sc.step_bytes()
    peak, peak_kind = _peaks()
    kv_gbs = job_throughput(b["kv"], args.steps, world, total)
    # e2e through the public API from host buffers
    e2e_total, h2d, d2h, e2e_note = _e2e(torch, sc, max(args.steps // 4, 3), flush, l2)
    e2e_total = slowest_rank_seconds(e2e_total, dist, "cuda")
    e2e_steps = max(args.steps // 4, 3)
    e2e_gbs = job_throughput(b["kv"], e2e_steps, world, e2e_total)
    # roofline of the dominant operation: paged_attn_decode (main kernel + LSE reduce)
    dec_achieved = b["decode"] / dec_mean / 1e9
    result = {
        "metric": METRIC, "value": round(kv_gbs, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": DTYPE[wl.kv_dtype], "data": "synthetic (seeded N(0,1) K/V/q, seeded lengths)",
        "config": {"workload": DESCR[args.workload], "name": args.workload,
                   "num_seqs": wl.num_seqs, "q_heads": wl.num_q_heads,
                   "kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim, "block_size": 16,
                   "partition_size": sc.resolved_partition(),
                   "tokens_in_cache": int(draw.context_lens.sum()),
                   "kv_bytes_per_step": b["kv"], "step_bytes": b,
                   "parallelism": f"replicas x{world} (no data-path collective)",
                   "l2": "flushed between timed steps (write of 2x L2), outside the events",
                   "decode_impl": args.decode_impl},
        "pct_hbm_peak": round(100 * kv_gbs / world / peak, 2),
        "pct_hbm_nominal": round(100 * kv_gbs / world / NOMINAL_HBM_GBS, 2),
        "tokens_per_s": round(world * wl.num_seqs / (total / args.steps), 1),
        "tokens_per_s_note": "one attention layer per step; a 32-layer model would decode "
                             "1/32 of this",
        "roofline": {"kernel": "paged_attn_decode (main kernel + LSE reduce)", "bound": "hbm",
                     "achieved": round(dec_achieved, 2), "peak": peak, "unit": "GB/s",
                     "frac": round(dec_achieved / peak, 4), "traffic": None,
                     "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": b["decode"],
                     "launch_ms": round(dec_mean * 1e3, 5)},
        "e2e": {"value": round(e2e_gbs, 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps, "note": e2e_note},
        "gpu_launches": sc.launches_per_step() * args.steps,
        "clocks": clk.summary((t_wall0, t_wall1), (w0, w1)),
    }
    traffic = _traffic_note(args.workload)
    if traffic is not None:
        result["roofline"]["traffic"] = traffic
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gpu = (sc.out.to(torch.float64).cpu().numpy(), sc.lse.to(torch.float64).cpu().numpy())
        cb = _cpu_baseline(draw, args.cpu_seconds, gpu=gpu)
        result["parity"] = cb.pop("parity")
        result["cpu_baseline"] = cb
    if rank == 0:
        result["host"] = _host_bookkeeping(pa)
    if rank == 0 and args.extra and world == 1:
        result["workloads"] = _extra_workloads(torch, pa, args, flush)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


# the sources the decode call's kernels are compiled from
DECODE_SOURCES = ("common.cuh", "decode_simt.cuh", "decode_tc.cuh", "pagedattn.cu")


def decode_sources_hash() -> str:
    """First 16 hex digits of the SHA-256 of the decode kernels' sources, in order."""
    h = hashlib.sha256()
    for f in DECODE_SOURCES:
        with open(os.path.join(ROOT, "paged_kv_cache_465_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def _traffic_note(name):
    """DRAM bytes of one decode call from the committed ncu summary (profiles/traffic.json)
    when it was taken on kernels built from exactly these decode sources; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        j = json.load(f)
    e = j.get(name)
    if not e or j.get("sources") != decode_sources_hash():
        return None
    return e.get("bytes_per_launch")


def _last_block_waste(lens, block_size):
    """Idle slots in the last blocks / allocated slots over the batch."""
    lens = np.asarray(lens, dtype=np.int64)
    alloc = int(((lens + block_size - 1) // block_size).sum()) * block_size
    return (alloc - int(lens.sum())) / alloc if alloc else 0.0


def _bf16_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    return FALLBACK_BF16_TFLOPS, "fallback"


def _prefill_workloads(torch, flush):
    """Prefill steps (write the new tokens' K/V, then causal attention over the paged cache)
    on the prefill workloads: TFLOP/s of the attention call against the bf16 tensor peak."""
    from paged_kv_cache_465_b200.scenario import PrefillScenario
    peak, kind = _bf16_peak()
    out = {}
    for name in ("prefill", "chunked", "chunked_fp8"):
        draw = workloads.draw_prefill(name)
        sc = PrefillScenario(draw, draw_seqs=[])
        for _ in range(3):
            flush()
            sc.step()
        steps = 30
        st = torch.cuda.current_stream()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
               torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            flush()
            e0, e1, e2 = ev[i]
            e0.record(st)
            sc.cache.write(sc.step_k, sc.step_v, sc.step_slots)
            e1.record(st)
            sc.cache.prefill(sc.q, sc.block_tables, sc.context_lens, sc.query_start, sc.scale,
                             sc.out, max_query_len=sc.max_query_len,
                             max_context_len=sc.max_context_len, lse_out=sc.lse)
            e2.record(st)
        torch.cuda.synchronize()
        total = sum(a.elapsed_time(c) for a, b, c in ev) / 1e3 / steps
        attn = sum(b.elapsed_time(c) for a, b, c in ev) / 1e3 / steps
        tflops = sc.flops() / attn / 1e12
        out[name] = {"value": round(tflops, 1), "unit": "TFLOP/s",
                     "pct_bf16_peak": round(100 * tflops / peak, 2), "peak_kind": kind,
                     "ms_per_step": round(total * 1e3, 5), "attention_ms": round(attn * 1e3, 5),
                     "new_tokens_per_s": round(draw.num_tokens / total, 1),
                     "flops_per_step": sc.flops(), "steps": steps,
                     "kernel": "tcgen05 prefill (S and O in tensor memory)"}
        del sc
        torch.cuda.empty_cache()
    return out


def _extra_workloads(torch, pa, args, flush):
    from paged_kv_cache_465_b200.scenario import DeviceScenario
    peak, _ = _peaks()
    out = {}
    # the named workloads, then the batch-256 fp8 workload with 8- and 32-token blocks (the
    # block-size trade-off: last-block waste against table length and tile size)
    runs = [(n, workloads.WORKLOADS[n]) for n in ("tiny", "b32", "shared", "b256", "long",
                                                   "b256_int8") if n != args.workload]
    base = workloads.WORKLOADS["b256"]
    runs += [(f"b256_bs{B}", base.scaled(block_size=B, num_blocks=base.num_blocks * 16 // B))
             for B in (8, 32)]
    # the long-context workload with the library's own split (PA_PARTITION_AUTO) instead of
    # the configured 512 tokens
    runs += [("long_auto", workloads.WORKLOADS["long"].scaled(partition_size=-1))]
    for name, wl in runs:
        draw = workloads.draw(wl)
        sc = DeviceScenario(draw, draw_seqs=[] if name not in ("tiny", "shared") else None)
        for _ in range(3):
            flush()
            sc.step()
        steps = 50 if name.startswith("long") else 200
        total, dec = _time_steps(torch, sc, steps, flush)
        b = sc.step_bytes()
        gbs = b["kv"] * steps / total / 1e9
        out[name] = {"value": round(gbs, 2), "unit": UNIT, "ms_per_step": round(total / steps * 1e3, 5),
                     "pct_hbm_peak": round(100 * gbs / peak, 2),
                     "pct_hbm_nominal": round(100 * gbs / NOMINAL_HBM_GBS, 2),
                     "decode_ms": round(dec * 1e3, 5),
                     "decode_gbs": round(b["decode"] / dec / 1e9, 2),
                     "tokens_per_s": round(draw.wl.num_seqs / (total / steps), 1),
                     "partition_size": sc.resolved_partition(), "block_size": wl.block_size,
                     "last_block_waste": round(_last_block_waste(draw.context_lens,
                                                                 wl.block_size), 6),
                     "steps": steps}
        del sc
        torch.cuda.empty_cache()
    out.update(_prefill_workloads(torch, flush))
    return out


# ---------------------------------------------------------------------------------------
# reference arm: the oracle on the host cores
# ---------------------------------------------------------------------------------------
def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import flows, paged as opaged, attention
    wl = workloads.WORKLOADS[args.workload]
    draw = workloads.draw(wl)
    rng = np.random.default_rng(0)
    sample = sorted(rng.choice(wl.num_seqs, size=min(wl.num_seqs, 8), replace=False).tolist())
    st = flows.build_state(draw, write_seqs=sample)
    sc = float(np.float32(1.0 / math.sqrt(wl.head_dim)))
    es = {"f32": 4, "bf16": 2, "fp8": 1, "int8": 1}[wl.kv_dtype]
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # noqa: BLE001
        cores = os.cpu_count()

    def one(i):
        s = sample[i % len(sample)]
        k, v = draw.kv(s)
        opaged.ref_reshape_and_cache(k[-1:], v[-1:], st.k_cache, st.v_cache, st.step_slots[s],
                                     wl.in_dtype, wl.kv_dtype, st.k_scales, st.v_scales,
                                     st.k_zeros, st.v_zeros)
        attention.ref_decode(draw.q, st.k_cache, st.v_cache, st.block_tables, st.context_lens,
                             sc, wl.num_kv_heads, wl.in_dtype, wl.kv_dtype, st.k_scales,
                             st.v_scales, seqs=[s], k_zeros=st.k_zeros, v_zeros=st.v_zeros)
        return int(draw.context_lens[s]) * 2 * wl.num_kv_heads * wl.head_dim * es

    for i in range(args.warmup):
        one(i)
    t0 = time.perf_counter()
    nbytes = 0
    for i in range(args.steps):
        nbytes += one(args.warmup + i)
    el = time.perf_counter() - t0
    val = nbytes / el / 1e9
    res = {"metric": METRIC, "value": round(val, 4), "unit": UNIT, "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 4),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "f64", "data": "synthetic (seeded N(0,1) K/V/q, seeded lengths)",
           "config": {"workload": DESCR[args.workload], "name": args.workload},
           "impl": "reference",
           "cpu_baseline": {"kind": "oracle", "cores": int(cores), "value": round(val, 4),
                            "unit": UNIT,
                            "sample": f"each step = one sequence (all heads) of {len(sample)} "
                                      f"sampled sequences of the workload, cache write + decode, "
                                      f"float64 NumPy"},
           "e2e": {"value": round(val, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="b256",
                    choices=sorted(workloads.WORKLOADS) + sorted(workloads.PREFILL_WORKLOADS),
                    help="decode workload (prefill workloads with --profile only)")
    ap.add_argument("--profile", action="store_true",
                    help="only the warm-up and timed steps of --workload (for ncu captures)")
    ap.add_argument("--seqs", type=int, default=0,
                    help="with --profile: the workload's first N sequences only")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--decode-impl", default="auto",
                    choices=["auto", "simt", "tc", "tc-grid", "tc-cta", "tc-warps"])
    ap.add_argument("--partition", type=int, default=None,
                    help="split-KV partition in tokens (default: the workload's)")
    ap.add_argument("--no-extra", dest="extra", action="store_false",
                    help="skip the other workloads' lines")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.workload in workloads.PREFILL_WORKLOADS and not args.profile:
        ap.error("prefill workloads run with --profile only")
    if args.profile:
        run_profile(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
