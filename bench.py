"""Benchmark: DSA decode at 128K context (index + top-2048 + sparse MLA) on B200.

One step = one dsa_decode_step over a batch of 16 sequences with 131,072 cached
tokens each (H_I = 64, d_I = 64 FP8 indexer keys, top-2048, 128-head MLA over
bf16 576-value latent rows), inputs resident in HBM.  Prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
  python bench.py --workload prefill [--prefill-len L] [--steps K] [--warmup W]
  python bench.py --workload dense [--steps K] [--warmup W]
  python bench.py --workload paged [--block-size S] [--steps K] [--warmup W]
  python bench.py --workload fp8kv [--steps K] [--warmup W]

N > 1 is launched with torch.distributed.run (one process per GPU); every rank
decodes its own batch (weak scaling, no data-path collective); the time is the
max over ranks.  --impl reference times the CPU oracle (the only reference
implementation there is) on a bounded sample of the same workload.

--workload prefill times dsa_prefill over one causal prompt of L tokens
(default 65,536: every position a query, top-2048, same shapes), then, in a
second pass over the same row chunks, each stage through its own entry point
(dsa_prefill_indexer_scores, dsa_topk, dsa_sparse_mla_attn) for the per-stage
split and the indexer's tensor-core roofline (FP8 peak = 2 x the measured bf16
peak).  It is a secondary line: the default run is the decode headline.

--workload dense times dense MLA over every cached token of the long-decode
batch (dsa_dense_mla_attn) and, in the same run, the DSA decode step on the
same inputs, and reports the measured DSA-vs-dense ratio (the pages quote ~6x
cheaper decode at 128K on H800 and a 13.4x arithmetic saving).

--workload paged times dsa_decode_step_paged on the long-decode batch with its
cache in blocks of a pool (seeded random physical order) and, in the same run,
dsa_decode_step on the contiguous cache, and reports the cost of paging.

--workload fp8kv times the decode step with the latent cache in 656-byte FP8
entries (512 e4m3 values, 4 fp32 scales, 64 bf16 rope values) against the
bf16 cache on the same inputs, same run.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode query-tok/s at 128K (index+top2048+sparse MLA); % HBM roofline"
UNIT = "query-tok/s"
WORKLOAD = "long_decode_b16_128k"
BATCH, CTX = 16, 131072
FALLBACK_HBM_GBS = 6650.0
INDEXER_SRC = os.path.join(ROOT, "sparse_long_context_indexer_b200", "csrc", "indexer_sm100.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "indexer_long_decode_b16_128k.md")
E2E_STEPS = 400          # end-to-end steps timed, whatever --steps is


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=5000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-secondary", action="store_true",
                   help="skip the secondary workloads (decode batch 32, 1M-context decode, prefill) of the default line")
    p.add_argument("--soak-seconds", type=float, default=2.0,
                   help="seconds of back-to-back steps inside the clock-sampled window (0 under a profiler)")
    p.add_argument("--e2e-steps", type=int, default=E2E_STEPS, help="steps of the end-to-end pass")
    p.add_argument("--workload", default="long_decode", choices=["long_decode", "prefill", "dense", "paged", "fp8kv"])
    p.add_argument("--block-size", type=int, default=64)
    p.add_argument("--prefill-len", type=int, default=65536)
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def tensor_peaks():
    """FP8 dense peak (TFLOP/s) = 2 x the measured bf16 cuBLAS figures (the nominal fp8:bf16 ratio)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return 2 * float(d["bf16_tflops"]), 2 * float(d["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 2 * 1590.0, 2 * 1400.0, "fallback"


def indexer_traffic():
    """DRAM bytes per indexer launch from the committed ncu summary, if it was taken on this source."""
    try:
        text = open(TRAFFIC_FILE).read()
        sha = hashlib.sha256(open(INDEXER_SRC, "rb").read()).hexdigest()
        m_sha = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
        m_b = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", text)
        if m_sha and m_b and m_sha.group(1) == sha:
            return int(m_b.group(1))
    except OSError:
        pass
    return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.perf_counter(), line.strip()))

    def wait_first(self, timeout=3.0):
        t0 = time.perf_counter()
        while self.proc is not None and not self.lines and time.perf_counter() - t0 < timeout:
            time.sleep(0.02)

    def stop(self, window=None):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, ln in self.lines:
            if window is not None and not (window[0] <= ts <= window[1] + 0.15):
                continue
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def nvml_reading(gpu_index):
    """One read-only NVML sample of the SM clock and the active clock-event reasons."""
    try:
        import pynvml
        pynvml.nvmlInit()
        try:
            h = pynvml.nvmlDeviceGetHandleByIndex(int(gpu_index))
            sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
            smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
            names = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                     "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                     "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                     "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
            return {"sm_mhz": float(sm), "sm_max_mhz": float(smax),
                    "reasons": sorted(k for k, v in names.items() if r & v)}
        finally:
            pynvml.nvmlShutdown()
    except Exception as e:  # reading only; a missing NVML is reported, not fatal
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [f"nvml unavailable: {type(e).__name__}"]}


def gpu_local_cpus(gpu_index):
    """The host cores NVML lists as local to this GPU (its NUMA node), within the cores this
    process may use; None when NVML cannot tell.  Read-only."""
    try:
        import pynvml
        pynvml.nvmlInit()
        try:
            h = pynvml.nvmlDeviceGetHandleByIndex(int(gpu_index))
            words = pynvml.nvmlDeviceGetCpuAffinity(h, (os.cpu_count() + 63) // 64)
        finally:
            pynvml.nvmlShutdown()
        cpus = {64 * i + b for i, w in enumerate(words) for b in range(64) if (int(w) >> b) & 1}
        cpus &= os.sched_getaffinity(0)
        return cpus or None
    except Exception:
        return None


class near_gpu_memory:
    """Runs its body on the GPU's local cores, so that pinned host buffers allocated inside it
    are placed (first touch) on the GPU's NUMA node; the process's affinity is restored on
    exit.  The DMA engines then read and write memory next to the GPU's PCIe root."""

    def __init__(self, gpu_index):
        self.cpus = gpu_local_cpus(gpu_index)
        self.saved = None

    def __enter__(self):
        if self.cpus:
            self.saved = os.sched_getaffinity(0)
            os.sched_setaffinity(0, self.cpus)
        return self

    def __exit__(self, *exc):
        if self.saved is not None:
            os.sched_setaffinity(0, self.saved)
        return False


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def dist_setup(n):
    import torch
    import torch.distributed as dist
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if n > 1 or world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def max_over_ranks(x: float, world: int) -> float:
    from sparse_long_context_indexer_b200 import dist as ddist
    return ddist.max_over_ranks(x, device="cuda") if world > 1 else x


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------- CPU oracle

_SAMPLES = {}


def oracle_sample(n_rows: int, nthreads: int, seed: int = 3, min_seconds: float = 0.0, max_passes: int = 1):
    """Full oracle pipeline (indexer -> top-k -> sparse attention) on n_rows
    query rows of the long-decode workload (each its own 131,072-token sequence),
    repeated until min_seconds have passed (at most max_passes passes).  Inputs
    are drawn once (untimed) and reused; returns (seconds, passes)."""
    import oracle
    from sparse_long_context_indexer_b200 import inputs
    if (n_rows, seed) not in _SAMPLES:
        _SAMPLES[(n_rows, seed)] = inputs.make_decode_inputs(WORKLOAD, [CTX] * n_rows, T_max=CTX, n_anchors=32,
                                                             recency=True, seed=seed)
    inp = _SAMPLES[(n_rows, seed)]
    passes = 0
    t0 = time.perf_counter()
    while True:
        oracle.decode(inp, nthreads=nthreads)
        passes += 1
        if passes >= max_passes or time.perf_counter() - t0 >= min_seconds:
            break
    return time.perf_counter() - t0, passes


def run_reference(args):
    """The oracle as the reference arm: one 128K-context query row per step (full path)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    cores = oracle.max_threads()
    budget_s = 150.0
    t_cal, _ = oracle_sample(1, cores)        # calibration, counted as the first warm-up step
    for _ in range(max(0, args.warmup - 1)):
        if t_cal * (args.warmup + args.steps) > budget_s:
            break
        oracle_sample(1, cores)
    steps = max(1, min(args.steps, int(budget_s / max(t_cal, 1e-3))))
    times = [oracle_sample(1, cores)[0] for _ in range(steps)]
    tot = sum(times)
    v = steps / tot
    sample = (f"1 query row per step of {WORKLOAD} (a 131072-token sequence; full path: indexer, top-2048, "
              f"128-head sparse MLA), fp64 C oracle, OpenMP on {cores} threads; {steps} of {args.steps} "
              f"requested steps timed to bound the run at ~{budget_s:.0f} s")
    line = {"metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus, "steps": steps,
            "steps_requested": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * tot / steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD, "batch_sampled": 1, "cached_tokens": CTX, "H_I": 64, "d_I": 64,
                       "top_k": 2048, "heads": 128},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm

def run_ours(args):
    import torch
    from sparse_long_context_indexer_b200 import _lib, accounting, api, inputs

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local if world > 1 else 0)
    inp = inputs.make_decode_inputs(WORKLOAD, [CTX] * BATCH, T_max=CTX, n_anchors=32, recency=True,
                                    seed=3 + rank, device=dev)
    dims = api.dims_of(inp)
    ws = api.make_workspace(dims, _lib.DSA_OP_DECODE, dev)
    out, lse = api.alloc_outputs(inp)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    sweep = torch.ones(256 << 20, dtype=torch.uint8, device=dev)

    def flush_l2():
        # write 256 MiB (evicts the step's data), then read another 256 MiB so that the
        # written lines are back in HBM before the timed region: the step starts with
        # clean, unrelated lines in L2 and no write-back of the flush in its timing
        flush.zero_()
        sweep.view(torch.int64).max()
    K, W = args.steps, args.warmup

    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [x for x in vis.split(",") if x.strip()]
    li = local if world > 1 else 0
    gpu_index = ids[li] if li < len(ids) else str(li)
    # clocks are sampled from the warm-up through the end-to-end pass (seconds, not only the
    # few milliseconds of the timed loop), plus one NVML reading on each side of the timed loop
    sampler = ClockSampler(gpu_index)
    sampler.start()
    sampler.wait_first()
    window0 = time.perf_counter()

    for _ in range(W):
        flush_l2()
        api.run_decode(inp, ws=ws, out=out, lse=lse, dims=dims)
    torch.cuda.synchronize()
    status = api.get_device_status(ws)
    if status != 0:
        raise SystemExit(f"device status {status}: {api.status_string(status)}")

    # Headline pass: one start and one end event per step.  Events recorded between the
    # stages cost ~2 us of GPU time each, so the per-stage breakdown (and the indexer
    # duration the roofline uses) comes from a second pass right after this one.
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    barrier(world)
    torch.cuda.synchronize()
    nvml_before = nvml_reading(gpu_index)
    wall0 = time.perf_counter()
    for i in range(K):
        flush_l2()   # outside the timed events
        evs[i][0].record()
        api.run_decode(inp, ws=ws, out=out, lse=lse, dims=dims)
        evs[i][1].record()
    torch.cuda.synchronize()
    wall1 = time.perf_counter()
    nvml_after = nvml_reading(gpu_index)
    wall = wall1 - wall0
    barrier(world)
    step_ms = [evs[i][0].elapsed_time(evs[i][1]) for i in range(K)]
    mean_ms = sum(step_ms) / K
    mean_ms = max_over_ranks(mean_ms, world)

    # Clock soak: the same step back to back for ~2 s of wall time while nvidia-smi samples
    # (the timed loop itself lasts a few milliseconds, too short for 100 ms samples)
    t_soak = time.perf_counter()
    while time.perf_counter() - t_soak < args.soak_seconds:
        for _ in range(200):
            flush_l2()
            api.run_decode(inp, ws=ws, out=out, lse=lse, dims=dims)
        torch.cuda.synchronize()

    # Stage pass: the same steps with an event before the indexer and after every stage.
    KS = min(max(K, 200), 1000)
    sev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(KS)]
    for i in range(KS):
        flush_l2()
        api.run_decode(inp, ws=ws, out=out, lse=lse, dims=dims, events=sev[i])
    torch.cuda.synchronize()
    stage = [[sev[i][j].elapsed_time(sev[i][j + 1]) for j in range(4)] for i in range(KS)]
    stage_us = [1000 * sum(s[j] for s in stage) / KS for j in range(4)]
    status = api.get_device_status(ws)

    # ---- end to end through the C interface with host buffers
    e2e = measure_e2e(inp, dims, dev, steps=args.e2e_steps, warmup=max(W, 10), gpu_index=gpu_index)
    if not e2e["readback_ok"]:
        raise SystemExit("end-to-end loop: the host copy of the last step's output differs from the device's")
    e2e_ms = max_over_ranks(e2e["ms"], world)
    window1 = time.perf_counter()
    clocks = sampler.stop(window=(window0, window1))

    hbm, peak_kind = peaks()
    lens = [CTX] * BATCH
    by = accounting.decode_step_bytes(lens)
    idx_bytes = by["indexer"]
    idx_us = stage_us[0]
    achieved = idx_bytes / (idx_us * 1e-6) / 1e9
    traffic = indexer_traffic()
    value = BATCH * world / (mean_ms * 1e-3)
    step_gbs = by["total"] / (mean_ms * 1e-3) / 1e9

    # ---- secondary workloads (one GPU): decode batch 32 (ragged 16K-32K), 1M-context decode, prefill
    secondary = {}
    if world == 1 and not args.no_secondary:
        del inp, ws, out, lse
        torch.cuda.empty_cache()
        for key, make in (("decode32", inputs.decode32), ("million", inputs.million)):
            secondary[key] = measure_secondary_decode(make, dev, K=max(K, 20), W=max(W, 3), flush_l2=flush_l2,
                                                      hbm=hbm, peak_kind=peak_kind)
            torch.cuda.empty_cache()
        secondary["prefill"] = measure_prefill(65536, dev, K=2, W=1)
        torch.cuda.empty_cache()
        secondary["dense_crossover"] = measure_crossover(dev, K=3, W=1)
        torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        cores = oracle.max_threads()
        rows = BATCH
        t, passes = oracle_sample(rows, cores, min_seconds=10.0, max_passes=40)
        t1, p1 = oracle_sample(1, 1, min_seconds=4.0, max_passes=5)
        cpu = {"value": rows * passes / t, "unit": UNIT, "cores": cores, "kind": "oracle",
               "cpu_model": cpu_model(),
               "sample": f"the {rows} query rows of {WORKLOAD} (each a 131072-token sequence), full path, "
                         f"fp64 C oracle with OpenMP on {cores} threads, {passes} passes in {t:.1f} s",
               "single_thread": {"value": p1 / t1, "unit": UNIT, "cores": 1,
                                 "sample": f"1 query row of {WORKLOAD}, full path, fp64 C oracle on one thread, "
                                           f"{p1} passes in {t1:.1f} s"}}
        if "prefill" in secondary:
            secondary["prefill"]["cpu_baseline"] = prefill_cpu_baseline(65536, cores, dev)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": mean_ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8_e4m3/bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "batch_per_gpu": BATCH, "cached_tokens": CTX, "H_I": 64, "d_I": 64,
                   "top_k": 2048, "heads": 128, "latent": "576 bf16 (512 + 64 rope)",
                   "l2": "flushed between steps outside the timed events: 256 MiB write, then a 256 MiB read "
                         "of another buffer (the written lines reach HBM before the step)",
                   "parallelism": f"replicas x{world} (sequences sharded, no collective)"},
        "roofline": {"bound": "hbm", "kernel": "indexer_fp8_kernel", "achieved": achieved, "peak": hbm,
                     "unit": "GB/s", "frac": achieved / hbm, "traffic": traffic,
                     "peak_source": f"{peak_kind} hbm_gbs", "algorithmic_bytes": idx_bytes},
        "step_roofline": {"achieved": step_gbs, "peak": hbm, "unit": "GB/s", "frac": step_gbs / hbm,
                          "algorithmic_bytes": by["total"]},
        "stages_us": {"indexer": stage_us[0], "topk": stage_us[1], "sparse_mla": stage_us[2],
                      "merge": stage_us[3]},
        "e2e": {"value": BATCH * world / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": e2e["h2d"],
                "d2h_bytes_per_step": e2e["d2h"], "ms_per_step": e2e_ms, "steps": args.e2e_steps,
                "pipeline": "one CUDA-graph replay per step, captured once per buffer slot from the public calls: "
                            "the step's cache append + dsa_decode_step on its slot, the H2D copy of the next "
                            "step's inputs (one packed pinned buffer) and the D2H copy of the previous step's "
                            "out and lse, as three concurrent branches of the graph; the timed region also "
                            "holds the first copy-in and the last copy-out; the last read-back is checked "
                            "against the device copy and against a direct dsa_decode_step call",
                "host_link": e2e["link"]},
        "gpu_launches": launches_per_step() * K,
        "timing": {"step": "one start and one end event per step on the launching stream",
                   "stages_us": f"separate pass of {KS} steps with an event between stages (each adds ~2 us)"},
        "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"], "reasons": clocks["reasons"],
                   "samples": clocks["samples"], "window_s": window1 - window0,
                   "window": "nvidia-smi every 100 ms from the warm-up through the end-to-end pass, which "
                             f"includes ~{args.soak_seconds:g} s of the same step back to back",
                   "nvml_before_timed_loop": nvml_before, "nvml_after_timed_loop": nvml_after},
        "device_status": status,
        "wall_s_timed_loop": wall,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    for key, v in secondary.items():
        line[key] = v
    print(json.dumps(line), flush=True)
    return 0


def measure_secondary_decode(make, dev, K, W, flush_l2, hbm, peak_kind):
    """A secondary decode workload (labelled as such in the line): the same decode step timed
    like the headline (one start/end event per step, L2 flushed outside the timed events)."""
    import torch
    from sparse_long_context_indexer_b200 import _lib, accounting, api
    inp = make(device=dev)
    dims = api.dims_of(inp)
    ws = api.make_workspace(dims, _lib.DSA_OP_DECODE, dev)
    out, lse = api.alloc_outputs(inp)
    for _ in range(W):
        flush_l2()
        api.run_decode(inp, ws=ws, out=out, lse=lse, dims=dims)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    for i in range(K):
        flush_l2()
        evs[i][0].record()
        api.run_decode(inp, ws=ws, out=out, lse=lse, dims=dims)
        evs[i][1].record()
    torch.cuda.synchronize()
    ms = sum(e[0].elapsed_time(e[1]) for e in evs) / K
    status = api.get_device_status(ws)
    lens = list(inp.seq_lens)
    by = accounting.decode_step_bytes(lens)
    gbs = by["total"] / (ms * 1e-3) / 1e9
    return {"label": "secondary workload (the headline is the long decode above)",
            "workload": inp.name, "batch": inp.B, "cached_tokens": {"min": min(lens), "max": max(lens),
                                                                    "sum": sum(lens)},
            "value": inp.B / (ms * 1e-3), "unit": UNIT, "ms_per_step": ms, "steps": K, "warmup": W,
            "step_roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                              "algorithmic_bytes": by["total"], "peak_source": f"{peak_kind} hbm_gbs"},
            "device_status": status}


def run_prefill(args):
    """Secondary line: one causal prompt of L tokens through dsa_prefill, with a per-stage split."""
    import torch
    if args.gpus != 1:
        raise SystemExit("--workload prefill runs on one GPU")
    line = measure_prefill(args.prefill_len, torch.device("cuda", 0), K=max(1, min(args.steps, 10)), W=args.warmup)
    line["metric"] = f"prefill query-tok/s (one causal prompt of {args.prefill_len} tokens; index+top2048+sparse MLA)"
    line.update({"n_gpus": 1, "higher_is_better": True, "scaling": "none", "vs_baseline": None,
                 "dtype": "fp8_e4m3/bf16", "data": "synthetic"})
    if not args.no_cpu_baseline:
        import oracle
        oracle.build()
        line["cpu_baseline"] = prefill_cpu_baseline(args.prefill_len, oracle.max_threads(), torch.device("cuda", 0))
    print(json.dumps(line), flush=True)
    return 0


def measure_prefill(L, dev, K, W):
    """dsa_prefill over one causal prompt of L tokens (median of K timed prompts), then a second
    pass over the same row chunks calling each stage's own entry point for the stage split and
    the indexer's tensor-core roofline."""
    import torch
    from sparse_long_context_indexer_b200 import _lib, api, inputs

    g = inputs.make_prefill_inputs(f"prefill_{L}", L, seed=4, device=dev)
    dims = api.dims_of(g)
    ws = api.make_workspace(dims, _lib.DSA_OP_PREFILL, dev)
    out, lse = api.alloc_outputs(g)
    idx = torch.empty((L, g.k), dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def whole():
        api.prefill(dims, g.q_I, g.q_scale, g.w, g.k_I, g.k_scale, g.q, g.kv, g.q_seq, g.q_len, g.softmax_scale,
                    out, lse, ws, idx_out=idx)

    for _ in range(W):
        whole()
    torch.cuda.synchronize()
    ms = []
    for _ in range(K):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        whole()
        e1.record()
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    status = api.get_device_status(ws)
    total_ms = statistics.median(ms)

    # Stage pass: the same work, chunk by chunk, each stage through its own entry point.
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    chunk = max(1, (64 << 20) // (dims.ld_scores * 4))
    if chunk >= sms // 2:
        chunk = chunk // (sms // 2) * (sms // 2) // 4 * 4   # the library's plan: whole attention waves
    chunk = max(1, min(L, chunk))
    cd = api.Dims(B=1, Nq=chunk, H_I=g.H_I, d_I=g.d_I, H=g.H, k=g.k, T_max=g.T_max, idx_dtype=g.idx_dtype,
                  kv_dtype=g.kv_dtype, ld_scores=dims.ld_scores)
    cws = api.make_workspace(cd, _lib.DSA_OP_SPARSE_MLA, dev)
    scores = torch.empty((chunk, dims.ld_scores), dtype=torch.float32, device=dev)
    cidx = torch.empty((chunk, g.k), dtype=torch.int32, device=dev)
    ev = []
    for r0 in range(0, L, chunk):
        r1 = min(L, r0 + chunk)
        d = cd if r1 - r0 == chunk else dataclasses.replace(cd, Nq=r1 - r0)
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        e[0].record()
        api.prefill_indexer_scores(d, g.q_I[r0:r1], g.q_scale[r0:r1], g.w[r0:r1], g.k_I, g.k_scale, g.q_seq[r0:r1],
                                   g.q_len[r0:r1], scores, cws)
        e[1].record()
        # the chunk's rows hold at most (T_max - L) + r1 positions: the bound dsa_prefill plans its top-k with
        api.topk(dataclasses.replace(d, T_max=g.T_max - L + r1), scores, g.q_len[r0:r1], cidx, cws)
        e[2].record()
        api.sparse_mla_attn(d, g.q[r0:r1], g.kv, cidx, g.q_seq[r0:r1], g.q_len[r0:r1], g.softmax_scale,
                            out[r0:r1], lse[r0:r1], cws)
        e[3].record()
        ev.append(e)
    torch.cuda.synchronize()
    stage_ms = [sum(e[j].elapsed_time(e[j + 1]) for e in ev) for j in range(3)]
    status = status or api.get_device_status(cws)

    pairs = int(g.q_len.sum().item())
    idx_flop = pairs * 2.0 * g.H_I * g.d_I
    sel = torch.clamp(g.q_len, max=g.k).sum().item()
    mla_flop = sel * g.H * 2.0 * (576 + 512)
    burst, sustained, src = tensor_peaks()
    idx_tflops = idx_flop / (stage_ms[0] * 1e-3) / 1e12
    del g, out, lse, idx, scores, cidx
    return {
        "label": "secondary workload (the headline is the long decode above)",
        "value": L / (total_ms * 1e-3), "unit": "query-tok/s", "steps": K, "warmup": W, "ms_per_step": total_ms,
        "config": {"workload": f"prefill_{L}", "H_I": dims.H_I, "d_I": dims.d_I, "top_k": dims.k, "heads": dims.H,
                   "latent": "576 bf16 (512 + 64 rope)", "chunk_rows": chunk,
                   "l2": "256 MiB written between prompts, outside the timed events"},
        "roofline": {"bound": "tensor", "kernel": "indexer_fp8_kernel (four rows per pass)",
                     "achieved": idx_tflops, "peak": burst, "unit": "TFLOP/s", "frac": idx_tflops / burst,
                     "frac_of_sustained": idx_tflops / sustained, "traffic": None,
                     "peak_source": f"2 x {src} bf16_tflops (burst); sustained {sustained:.0f}",
                     "algorithmic_flop": idx_flop},
        "stages_ms": {"indexer": stage_ms[0], "topk": stage_ms[1], "sparse_mla": stage_ms[2]},
        "sparse_mla_tflops": mla_flop / (stage_ms[2] * 1e-3) / 1e12,
        "timing": {"step": "dsa_prefill between two events, median of the timed prompts",
                   "stages_ms": f"second pass of {len(ev)} chunks of {chunk} rows, two events per stage call"},
        "device_status": status,
    }


def prefill_sample_rows(L, k=2048):
    """The fixed 512-row oracle sample of the prefill prompt: rows 0-63 (short rows that take
    every position), 2000-2111 (around the budget), 32 rows spread evenly, and the last 304."""
    spread = [int(round(x)) for x in [(i + 0.5) * L / 32 for i in range(32)]]
    rows = sorted(set(list(range(0, 64)) + list(range(2000, 2112)) + spread + list(range(L - 304, L))))
    return [r for r in rows if 0 <= r < L]


def prefill_cpu_baseline(L, cores, dev=None):
    """The oracle (full path) on the fixed 512-row sample of the prefill prompt, with OpenMP on
    all host cores, timed per group of rows.  The whole prompt is then EXTRAPOLATED with a
    per-row cost a * (t + 1) + b * min(t + 1, k) fitted to the groups (non-negative least
    squares); the line says so."""
    import numpy as np
    import oracle
    from sparse_long_context_indexer_b200 import inputs
    k = 2048
    rows = prefill_sample_rows(L, k)
    # drawn on the device the GPU leg uses (same generator, so the sample rows are the GPU
    # workload's own rows), then handed to the oracle on the host
    sub = inputs.make_prefill_inputs(f"prefill_{L}", L, seed=4, rows=rows, device=dev or "cpu").to("cpu")
    groups = {"0-63": [r for r in rows if r < 64], "2000-2111": [r for r in rows if 2000 <= r < 2112],
              f"last 304": [r for r in rows if r >= L - 304]}
    used = set(sum(groups.values(), []))
    groups["spread"] = [r for r in rows if r not in used]
    pos = {r: i for i, r in enumerate(rows)}
    times, feats = {}, []
    for name, rr in groups.items():
        sel = [pos[r] for r in rr]
        part = subset_rows(sub, sel)
        t0 = time.perf_counter()
        oracle.decode(part, nthreads=cores)
        times[name] = time.perf_counter() - t0
        n = np.array(rr, dtype=np.float64) + 1
        feats.append([n.sum(), np.minimum(n, k).sum()])
    A = np.array(feats)
    y = np.array(list(times.values()))
    from scipy.optimize import nnls
    coef, _ = nnls(A, y)                       # non-negative costs per key and per selected row
    n_all = np.arange(1, L + 1, dtype=np.float64)
    extrap = float(coef[0] * n_all.sum() + coef[1] * np.minimum(n_all, k).sum())
    total = sum(times.values())
    return {"value": len(rows) / total, "unit": "query-tok/s", "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": f"{len(rows)} fixed rows of the {L}-token prompt (0-63, 2000-2111, 32 spread, last 304), "
                      f"full path (indexer over t+1 keys, top-2048, 128-head sparse MLA), fp64 C oracle, "
                      f"OpenMP on {cores} threads, {total:.1f} s",
            "seconds_per_group": times, "rows_per_group": {kk: len(v) for kk, v in groups.items()},
            "extrapolated_prompt_s": extrap,
            "extrapolation": "EXTRAPOLATED, not measured: per-row cost a*(t+1) + b*min(t+1, 2048) fitted to the "
                             f"group times (a = {coef[0]:.3e} s per key, b = {coef[1]:.3e} s per selected row), "
                             f"summed over all {L} rows"}


def subset_rows(inp, sel):
    """The same inputs restricted to the query rows `sel` (the cache is shared)."""
    import torch
    from sparse_long_context_indexer_b200 import inputs
    r = torch.as_tensor(sel, dtype=torch.long)
    out = inputs.DSAInputs(**{f: getattr(inp, f) for f in inp.__dataclass_fields__})
    for f in ("q_I", "q_scale", "w", "q", "q_seq", "q_len"):
        v = getattr(inp, f)
        if v is not None:
            setattr(out, f, v[r].contiguous())
    out.Nq = len(sel)
    return out


def measure_crossover(dev, K=5, W=2, decode_lens=(2048, 4096, 8192, 16384, 32768, 65536, 131072),
                      prefill_lens=(2048, 4096, 8192, 16384, 32768)):
    """Where DSA starts to beat dense attention on this GPU: the DSA decode step (indexer +
    top-2048 + sparse MLA) against dense MLA over every cached token, for a batch of 16 rows
    of each length, and dsa_prefill against dense causal MLA for one prompt of each length.
    Medians of K event-timed runs, L2 flushed between runs (outside the events).  Up to k
    tokens every position is selected and the decode step runs the dense kernel itself, so the
    crossover is the first length above k where DSA wins."""
    import torch
    from sparse_long_context_indexer_b200 import _lib, api, inputs

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def timed(fn):
        for _ in range(W):
            flush.zero_()
            fn()
        torch.cuda.synchronize()
        ms = []
        for _ in range(K):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        return statistics.median(ms)

    k_sel = 2048  # the selection budget of these inputs

    def point(L, dsa_ms, dense_ms):
        # up to k tokens a row selects every position: DSA computes dense attention there
        return {"tokens": L, "dsa_ms": round(dsa_ms, 4), "dense_ms": round(dense_ms, 4),
                "dense_over_dsa": round(dense_ms / dsa_ms, 3), "selects_every_position": L <= k_sel}

    status = 0
    dec = []
    for L in decode_lens:
        g = inputs.make_decode_inputs(f"crossover_decode_{L}", [L] * BATCH, T_max=L, n_anchors=32, recency=True,
                                      seed=3, device=dev)
        dims = api.dims_of(g)
        ws, ws_d = api.make_workspace(dims, _lib.DSA_OP_DECODE, dev), api.make_workspace(dims, _lib.DSA_OP_DENSE_MLA, dev)
        out, lse = api.alloc_outputs(g)
        dsa_ms = timed(lambda: api.run_decode(g, ws=ws, out=out, lse=lse, dims=dims))
        dense_ms = timed(lambda: api.dense_mla_attn(dims, g.q, g.kv, g.q_seq, g.q_len, g.softmax_scale, out, lse, ws_d))
        status = status or api.get_device_status(ws) or api.get_device_status(ws_d)
        dec.append(point(L, dsa_ms, dense_ms))
        del g, ws, ws_d, out, lse
        torch.cuda.empty_cache()
    pre = []
    for L in prefill_lens:
        g = inputs.make_prefill_inputs(f"crossover_prefill_{L}", L, seed=4, device=dev)
        dims = api.dims_of(g)
        ws, ws_d = api.make_workspace(dims, _lib.DSA_OP_PREFILL, dev), api.make_workspace(dims, _lib.DSA_OP_DENSE_MLA, dev)
        out, lse = api.alloc_outputs(g)
        dsa_ms = timed(lambda: api.prefill(dims, g.q_I, g.q_scale, g.w, g.k_I, g.k_scale, g.q, g.kv, g.q_seq, g.q_len,
                                           g.softmax_scale, out, lse, ws))
        dense_ms = timed(lambda: api.dense_mla_attn(dims, g.q, g.kv, g.q_seq, g.q_len, g.softmax_scale, out, lse, ws_d))
        status = status or api.get_device_status(ws) or api.get_device_status(ws_d)
        pre.append(point(L, dsa_ms, dense_ms))
        del g, ws, ws_d, out, lse
        torch.cuda.empty_cache()

    def first_win(pts):
        return next((p["tokens"] for p in pts if p["tokens"] > k_sel and p["dense_over_dsa"] > 1.0), None)

    return {"label": "secondary measurement (the headline is the long decode above)",
            "decode": {"batch": BATCH, "points": dec, "dsa_faster_from_tokens": first_win(dec)},
            "prefill": {"points": pre, "dsa_faster_from_tokens": first_win(pre),
                        "note": "one causal prompt; dense = every row over its whole causal prefix"},
            "k": k_sel, "timing": f"median of {K} event-timed runs per point, L2 flushed between runs",
            "device_status": status}


def run_dense(args):
    """Secondary line: dense MLA over all cached tokens of the long decode, against the DSA step."""
    import torch
    from sparse_long_context_indexer_b200 import _lib, api, inputs

    if args.gpus != 1:
        raise SystemExit("--workload dense runs on one GPU")
    dev = torch.device("cuda", 0)
    inp = inputs.make_decode_inputs(WORKLOAD, [CTX] * BATCH, T_max=CTX, n_anchors=32, recency=True, seed=3,
                                    device=dev)
    dims = api.dims_of(inp)
    ws_d = api.make_workspace(dims, _lib.DSA_OP_DENSE_MLA, dev)
    ws = api.make_workspace(dims, _lib.DSA_OP_DECODE, dev)
    out, lse = api.alloc_outputs(inp)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    K, W = max(1, min(args.steps, 200)), args.warmup

    def dense():
        api.dense_mla_attn(dims, inp.q, inp.kv, inp.q_seq, inp.q_len, inp.softmax_scale, out, lse, ws_d)

    def dsa():
        api.run_decode(inp, ws=ws, out=out, lse=lse, dims=dims)

    def timed(fn):
        for _ in range(W):
            flush.zero_()
            fn()
        torch.cuda.synchronize()
        ms = []
        for _ in range(K):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        return statistics.median(ms)

    dense_ms = timed(dense)
    status = api.get_device_status(ws_d)
    dsa_ms = timed(dsa)
    status = status or api.get_device_status(ws)
    flop = BATCH * dims.H * 2.0 * CTX * (576 + 512)
    by = BATCH * (CTX * 1152 + 147456 + 131072 + 512)
    tflops = flop / (dense_ms * 1e-3) / 1e12
    bf16 = None
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            bf16 = float(json.load(f)["bf16_tflops"])
    except Exception:
        bf16 = 1590.0
    line = {
        "metric": "dense MLA decode query-tok/s at 128K (attention over every cached token)",
        "value": BATCH / (dense_ms * 1e-3), "unit": "query-tok/s", "n_gpus": 1, "steps": K, "warmup": W,
        "ms_per_step": dense_ms, "higher_is_better": True, "scaling": "none", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "batch_per_gpu": BATCH, "cached_tokens": CTX, "heads": dims.H,
                   "latent": "576 bf16 (512 + 64 rope)",
                   "l2": "256 MiB written between steps, outside the timed events"},
        "roofline": {"bound": "tensor", "kernel": "sparse_mla_bf16_kernel (dense mode)", "achieved": tflops,
                     "peak": bf16, "unit": "TFLOP/s", "frac": tflops / bf16,
                     "note": "M = 64 tensor-core tiles run at half the rate of the measured bf16 peak",
                     "algorithmic_flop": flop, "algorithmic_bytes": by,
                     "hbm_gbs": by / (dense_ms * 1e-3) / 1e9},
        "dsa_vs_dense": {"dsa_step_ms": dsa_ms, "dense_attention_ms": dense_ms, "ratio": dense_ms / dsa_ms,
                         "note": "DSA = indexer + top-2048 + sparse MLA on the same batch, same run"},
        "device_status": status,
    }
    del inp, ws, ws_d, out, lse
    torch.cuda.empty_cache()
    line["crossover"] = measure_crossover(dev)
    print(json.dumps(line), flush=True)
    return 0


def run_paged(args):
    """Secondary line: the decode step over a paged cache against the contiguous one."""
    import torch
    from sparse_long_context_indexer_b200 import _lib, api, inputs

    if args.gpus != 1:
        raise SystemExit("--workload paged runs on one GPU")
    dev = torch.device("cuda", 0)
    inp = inputs.make_decode_inputs(WORKLOAD, [CTX] * BATCH, T_max=CTX, n_anchors=32, recency=True, seed=3,
                                    device=dev)
    dims = api.dims_of(inp)
    ws = api.make_workspace(dims, _lib.DSA_OP_DECODE, dev)
    out, lse = api.alloc_outputs(inp)
    out_p, lse_p = api.alloc_outputs(inp)
    k_pool, s_pool, kv_pool, table = inputs.paged_layout(inp, args.block_size, seed=1)
    cache = api.PagedCache(k_pool, s_pool, kv_pool, table, args.block_size)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    sweep = torch.ones(256 << 20, dtype=torch.uint8, device=dev)
    K, W = max(1, min(args.steps, 2000)), args.warmup

    def contiguous():
        api.run_decode(inp, ws=ws, out=out, lse=lse, dims=dims)

    def paged():
        api.decode_step_paged(dims, inp.q_I, inp.q_scale, inp.w, cache, inp.q, inp.q_seq, inp.q_len,
                              inp.softmax_scale, out_p, lse_p, ws)

    def timed(fn):
        for _ in range(W):
            fn()
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        for i in range(K):
            flush.zero_()
            sweep.view(torch.int64).max()
            ev[i][0].record()
            fn()
            ev[i][1].record()
        torch.cuda.synchronize()
        return sum(e[0].elapsed_time(e[1]) for e in ev) / K

    c_ms = timed(contiguous)
    p_ms = timed(paged)
    status = api.get_device_status(ws)
    same = bool(torch.equal(out, out_p) and torch.equal(lse, lse_p))
    line = {
        "metric": f"paged decode query-tok/s at 128K (blocks of {args.block_size} tokens)",
        "value": BATCH / (p_ms * 1e-3), "unit": "query-tok/s", "n_gpus": 1, "steps": K, "warmup": W,
        "ms_per_step": p_ms, "higher_is_better": True, "scaling": "none", "vs_baseline": None,
        "dtype": "fp8_e4m3/bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "batch_per_gpu": BATCH, "cached_tokens": CTX, "block_size": args.block_size,
                   "pool_blocks": int(kv_pool.shape[0]),
                   "l2": "flushed between steps outside the timed events (write, then read of another buffer)"},
        "paged_vs_contiguous": {"paged_ms": p_ms, "contiguous_ms": c_ms, "ratio": p_ms / c_ms,
                                "outputs_identical": same},
        "device_status": status,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_fp8kv(args):
    """Secondary line: the decode step over the FP8 latent cache against the bf16 one."""
    import torch
    from sparse_long_context_indexer_b200 import _lib, accounting, api, inputs

    if args.gpus != 1:
        raise SystemExit("--workload fp8kv runs on one GPU")
    dev = torch.device("cuda", 0)
    inp = inputs.make_decode_inputs(WORKLOAD, [CTX] * BATCH, T_max=CTX, n_anchors=32, recency=True, seed=3,
                                    device=dev)
    inp8 = inputs.with_fp8_latent(inp)
    dims, dims8 = api.dims_of(inp), api.dims_of(inp8)
    ws = api.make_workspace(dims, _lib.DSA_OP_DECODE, dev)
    out, lse = api.alloc_outputs(inp)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    sweep = torch.ones(256 << 20, dtype=torch.uint8, device=dev)
    K, W = max(1, min(args.steps, 2000)), args.warmup

    def timed(g, d):
        for _ in range(W):
            api.run_decode(g, ws=ws, out=out, lse=lse, dims=d)
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        for i in range(K):
            flush.zero_()
            sweep.view(torch.int64).max()
            ev[i][0].record()
            api.run_decode(g, ws=ws, out=out, lse=lse, dims=d)
            ev[i][1].record()
        torch.cuda.synchronize()
        return sum(e[0].elapsed_time(e[1]) for e in ev) / K

    bf16_ms = timed(inp, dims)
    fp8_ms = timed(inp8, dims8)
    status = api.get_device_status(ws)
    by = accounting.decode_step_bytes([CTX] * BATCH)
    gather_bf16 = BATCH * 2048 * 1152
    fp8_bytes = by["total"] - gather_bf16 + BATCH * 2048 * 656
    line = {
        "metric": "decode query-tok/s at 128K with the FP8 latent cache (656-byte entries)",
        "value": BATCH / (fp8_ms * 1e-3), "unit": "query-tok/s", "n_gpus": 1, "steps": K, "warmup": W,
        "ms_per_step": fp8_ms, "higher_is_better": True, "scaling": "none", "vs_baseline": None,
        "dtype": "fp8_e4m3 (indexer and latent)/bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD + "_fp8kv", "batch_per_gpu": BATCH, "cached_tokens": CTX,
                   "latent": "656 B: 512 e4m3 + 4 fp32 scales + 64 bf16 rope",
                   "l2": "flushed between steps outside the timed events (write, then read of another buffer)"},
        "step_roofline": {"achieved": fp8_bytes / (fp8_ms * 1e-3) / 1e9, "peak": peaks()[0], "unit": "GB/s",
                          "algorithmic_bytes": fp8_bytes},
        "fp8_vs_bf16_latent": {"fp8_ms": fp8_ms, "bf16_ms": bf16_ms, "ratio": fp8_ms / bf16_ms,
                               "gather_bytes_per_row": {"fp8": 2048 * 656, "bf16": 2048 * 1152}},
        "device_status": status,
    }
    print(json.dumps(line), flush=True)
    return 0


def launches_per_step():
    """Kernels one decode step launches: indexer, top-k, attention, plus the split
    merge when the attention's split count is above the cluster limit (8)."""
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    s = max(1, min(16, sms // (2 * BATCH)))
    rows = -(-(-(-2048 // s)) // 64) * 64
    splits = -(-2048 // rows)
    return 4 if splits > 8 else 3


def measure_e2e(inp, dims, dev, steps, warmup, gpu_index="0"):
    """End to end through the public API, as a serving loop would run it.  Per step: the H2D
    copy of all of the step's inputs (query-side tensors, the new token's position, bf16
    latent row and fp32 indexer key, packed in one pinned buffer), the cache append
    (dsa_append_tokens, which quantises the key on the device), the decode step, and the D2H
    copy of out and lse.

    Two buffer slots.  Step i runs one CUDA graph, captured once per slot from the public
    calls, with three concurrent branches: the append + decode of step i on its slot, the
    H2D copy of step i+1's inputs into the other slot, and the D2H copy of step i-1's
    outputs from the other slot.  Graph launches on one stream run one after another, which
    orders the slots' reuse; the first copy-in and the last copy-out are inside the timed
    region too.  One host call per step keeps the host's issue cost off the step time."""
    import torch
    from sparse_long_context_indexer_b200 import _lib, api
    B = inp.B
    pos = (inp.q_len - 1).long()
    rows = torch.arange(B, device=dev)
    # the new token of each sequence: its bf16 latent row and its fp32 indexer key (the
    # library quantises it on the device), written at position q_len - 1
    k_new = inp.k_I[rows, pos].view(torch.float8_e4m3fn).float() * inp.k_scale[rows, pos][:, None]
    fields = {
        "q": inp.q, "q_I": inp.q_I, "q_scale": inp.q_scale, "w": inp.w, "q_len": inp.q_len,
        "pos": pos.to(torch.int32), "kv_new": inp.kv[rows, pos], "k_new": k_new,
    }
    offs, off = {}, 0
    for k, v in fields.items():
        offs[k] = off
        off += (v.numel() * v.element_size() + 255) // 256 * 256
    total = off
    h2d = sum(v.numel() * v.element_size() for v in fields.values())
    near = near_gpu_memory(gpu_index)
    with near:                                      # pinned buffers on the GPU's NUMA node
        host_pack = torch.empty(total, dtype=torch.uint8).pin_memory()
        for k, v in fields.items():
            nb = v.numel() * v.element_size()
            host_pack[offs[k]:offs[k] + nb].copy_(v.contiguous().cpu().view(-1).view(torch.uint8))
        ws = api.make_workspace(dims, _lib.DSA_OP_DECODE, dev)
        slots = []
        for _ in range(2):
            dbuf = torch.empty(total, dtype=torch.uint8, device=dev)
            views = {k: dbuf[offs[k]:offs[k] + v.numel() * v.element_size()].view(v.dtype).view(v.shape)
                     for k, v in fields.items()}
            o, l = api.alloc_outputs(inp)
            slots.append({"dbuf": dbuf, "v": views, "out": o, "lse": l,
                          "out_h": torch.empty(o.shape, dtype=o.dtype).pin_memory(),
                          "lse_h": torch.empty(l.shape, dtype=l.dtype).pin_memory()})
    d2h = slots[0]["out_h"].numel() * slots[0]["out_h"].element_size() + \
        slots[0]["lse_h"].numel() * slots[0]["lse_h"].element_size()
    main = torch.cuda.Stream(device=dev)
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    seq = torch.arange(B, dtype=torch.int32, device=dev)

    def copy_in(sl):
        sl["dbuf"].copy_(host_pack, non_blocking=True)

    def compute(sl):
        v = sl["v"]
        api.append_tokens(dims, seq, v["pos"], v["kv_new"], v["k_new"], inp.kv, inp.k_I, inp.k_scale, ws=ws)
        api.decode_step(dims, v["q_I"], v["q_scale"], v["w"], inp.k_I, inp.k_scale, v["q"], inp.kv, inp.q_seq,
                        v["q_len"], inp.softmax_scale, sl["out"], sl["lse"], ws)

    def copy_out(sl):
        sl["out_h"].copy_(sl["out"], non_blocking=True)
        sl["lse_h"].copy_(sl["lse"], non_blocking=True)

    def step_body(s):
        # fork: the other slot's copies run beside this slot's compute; join before the end
        cur, other = slots[s], slots[1 - s]
        fork = torch.cuda.Event()
        fork.record(main)
        s_in.wait_event(fork)
        s_out.wait_event(fork)
        with torch.cuda.stream(s_in):
            copy_in(other)
            in_done = torch.cuda.Event()
            in_done.record(s_in)
        with torch.cuda.stream(s_out):
            copy_out(other)
            out_done = torch.cuda.Event()
            out_done.record(s_out)
        with torch.cuda.stream(main):
            compute(cur)
        main.wait_event(in_done)
        main.wait_event(out_done)

    with torch.cuda.stream(main):                   # eager run first (lazy initialisation)
        copy_in(slots[0])
        copy_in(slots[1])
    main.synchronize()
    for s in (0, 1):
        with torch.cuda.stream(main):
            step_body(s)
    torch.cuda.synchronize(dev)
    graphs = []
    for s in (0, 1):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=main, capture_error_mode="relaxed"):
            step_body(s)
        graphs.append(g)
    torch.cuda.synchronize(dev)

    def run(n):
        with torch.cuda.stream(main):
            copy_in(slots[0])                       # the first step's inputs
            for i in range(n):
                graphs[i % 2].replay()
            copy_out(slots[(n - 1) % 2])            # the last step's outputs

    def link_rate(copy, nbytes, reps=50):
        # the host link alone: the same copies back to back on one stream, GB/s
        with torch.cuda.stream(main):
            for _ in range(5):
                copy()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(main)
            for _ in range(reps):
                copy()
            b.record(main)
        b.synchronize()
        return nbytes * reps / (a.elapsed_time(b) * 1e-3) / 1e9

    h2d_gbs = link_rate(lambda: copy_in(slots[0]), total)
    d2h_gbs = link_rate(lambda: copy_out(slots[0]), d2h)

    run(warmup)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    run(steps)
    e1.record(main)
    torch.cuda.synchronize(dev)
    last = slots[(steps - 1) % 2]
    ok = torch.equal(last["out_h"], last["out"].cpu()) and torch.equal(last["lse_h"], last["lse"].cpu())
    # the replayed step computes what a direct call computes on the same inputs
    ref_out, ref_lse = api.alloc_outputs(inp)
    v = last["v"]
    api.decode_step(dims, v["q_I"], v["q_scale"], v["w"], inp.k_I, inp.k_scale, v["q"], inp.kv, inp.q_seq,
                    v["q_len"], inp.softmax_scale, ref_out, ref_lse, ws)
    torch.cuda.synchronize(dev)
    ok = ok and torch.equal(ref_out.cpu(), last["out_h"]) and torch.equal(ref_lse.cpu(), last["lse_h"])
    status = api.get_device_status(ws)
    return {"ms": e0.elapsed_time(e1) / steps, "h2d": h2d, "d2h": d2h, "readback_ok": ok and status == 0,
            "link": {"h2d_gbs": round(h2d_gbs, 1), "d2h_gbs": round(d2h_gbs, 1),
                     "pinned_on": (f"the GPU's NUMA node ({len(near.cpus)} local cores)" if near.cpus
                                   else "the allocating thread's node (NVML gave no CPU affinity)")}}


def main():
    args = parse_args()
    if os.environ.get("DSA_ORACLE_LIB") or os.environ.get("DSA_ORACLE_MUTANT_RUN"):
        raise SystemExit("bench.py times the committed oracle only: unset DSA_ORACLE_LIB / DSA_ORACLE_MUTANT_RUN")
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "prefill":
        return run_prefill(args)
    if args.workload == "dense":
        return run_dense(args)
    if args.workload == "paged":
        return run_paged(args)
    if args.workload == "fp8kv":
        return run_fp8kv(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
