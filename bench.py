#!/usr/bin/env python
"""Benchmark of one paged GQA decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload long] [--impl ours|reference]

A step is one decode step of the whole path over one batch: the plan (policy
and, for the work-queue mode, the queue) for the batch's lengths, the split
kernel streaming every valid K/V page through the block table, and the merge.
The headline workload is the single long context: B=1, H_q=32, H_kv=8,
D=128, 16-token pages, 32768 tokens scattered over a 4096-page pool.

Metric: KV GB/s = (K+V bytes of the valid tokens + q + out) / step time, and
its fraction of the measured HBM copy bandwidth; also us/step.
  value  steady-state device time: K steps queued back to back on one
         stream between one pair of CUDA events, inputs resident in HBM.
         The K steps are captured once in a CUDA graph and replayed (as a
         serving loop replays its decode step; --no-graph queues them from
         Python instead).  Consecutive steps read different copies of the KV
         pool (enough copies that three L2 sizes of data lie between two
         reads of the same copy), so no step finds its pages in L2.
  latency_us  one isolated step, cold: L2 flushed (a 256 MiB write, then a
         256 MiB read so no dirty lines are left) before each step, CUDA
         events around the step alone.
  e2e    one synchronized pkv_decode_host call per step from pinned host
         buffers (policy + queue on the host, q / block table / lengths and
         the queue copied host->device, kernels, out copied device->host),
         host wall clock; the KV cache stays resident on the device.
Under torchrun (N > 1) every rank decodes its own replica of the workload
(weak scaling, no collective on the data path); the time is the max over
ranks of each rank's summed step times.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_gqa_17_b200.timing import (Flush, n_pool_copies, pool_copies, time_interleaved,  # noqa: E402
                                         time_isolated, time_steady)

METRIC = "paged GQA decode: KV GB/s (% of B200 HBM peak) and µs/step at batch 1/4/8"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="long",
                    choices=["tiny", "long", "crossover", "mixed", "prefix", "bimodal", "uniform", "zipf", "long_g1",
                             "long_g2", "long_g8", "long_g16", "prefix_small"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=None)
    ap.add_argument("--e2e-steps", type=int, default=None, help="steps of the end-to-end timing (default: --steps)")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads' lines in 'all_workloads'")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle cpu_baseline leg")
    ap.add_argument("--cpu-seconds", type=float, default=8.0, help="target CPU time of the cpu_baseline sample")
    ap.add_argument("--no-graph", action="store_true", help="queue the timed steps from Python, not a CUDA graph")
    ap.add_argument("--shared-prefix", action="store_true",
                    help="run the headline workload in the prefix-sharing plan (PKV_FLAG_SHARED_PREFIX)")
    return ap.parse_args(argv)


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def measured_peak():
    """(HBM GB/s, where from) from the machine's measured peaks, else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash():
    """Hash of the CUDA sources (the .cu files and the headers they include)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_gqa_17_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".h")):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the split kernel from the committed ncu summary
    (profiles/traffic.txt: `workload kernel_source_hash bytes` per line), if it
    was taken on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        with open(path) as f:
            for line in f:
                parts = line.split()
                if len(parts) == 3 and not line.startswith("#") and parts[0] == workload:
                    if parts[1] == kernel_source_hash():
                        return int(parts[2])
    except (OSError, ValueError):
        pass
    return None


# ---------------------------------------------------------------------------
# distributed plumbing (also exercised by the gloo tests on CPU)

def init_dist(world: int, backend: str, local_rank: int):
    import torch.distributed as dist

    if world <= 1:
        return None
    kw = {}
    if backend == "nccl":
        import torch

        kw["device_id"] = torch.device("cuda", local_rank)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=180), **kw)
    return dist


def max_over_ranks(value: float, dist, device=None) -> float:
    """Max of a per-rank scalar over all ranks (the timing reduction only)."""
    if dist is None:
        return value
    import torch

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, dist, device=None) -> float:
    if dist is None:
        return value
    import torch

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(dist, device=None):
    if dist is None:
        return
    if device is not None and device.type == "cuda":
        dist.barrier(device_ids=[device.index])
    else:
        dist.barrier()


# ---------------------------------------------------------------------------
# clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML in a thread."""

    REASONS = {
        "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
        "hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
        "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
        "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
        "hw_power_brake_slowdown": "nvmlClocksEventReasonHwPowerBrakeSlowdown",
        "gpu_idle": "nvmlClocksEventReasonGpuIdle",
        "applications_clocks_setting": "nvmlClocksEventReasonApplicationsClocksSetting",
        "sync_boost": "nvmlClocksEventReasonSyncBoost",
    }

    def __init__(self, index: int, period_s: float = 0.005):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml as nv

            nv.nvmlInit()
            self.nv = nv
            self.h = None
            try:  # NVML numbers GPUs physically; match the CUDA device by UUID
                import torch

                uuid = str(torch.cuda.get_device_properties(self.index).uuid)
                self.h = nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                self.h = nv.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.ok = True
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception:  # NVML missing: report no clocks rather than fail the bench
            self.ok = False
        return self

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, attr in self.REASONS.items():
                    if mask & getattr(nv, attr, 0):
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# the GPU arm

def _describe(w, plan):
    names = {0: "NO_SPLIT", 1: "SPLIT_S", 2: "WORK_QUEUE", 3: "BALANCED"}
    lens = w.seq_lens
    return {
        "workload": f"{w.name}: B={w.B} H_q={w.H_q} H_kv={w.H_kv} D={w.D} P={w.P} "
                    f"N={'/'.join(map(str, lens)) if w.B <= 8 else f'{min(lens)}..{max(lens)} (sum {sum(lens)})'}",
        "batch": w.B, "H_q": w.H_q, "H_kv": w.H_kv, "head_dim": w.D, "page_size": w.P,
        "tokens": sum(lens), "pool_pages": w.num_pages, "seed": w.seed,
        "plan": {"mode": names[plan.mode], "num_splits": plan.num_splits, "chunk_pages": plan.chunk_pages,
                 "flags": plan.flags},
    }


def arm_config(w, plan, world: int, graph: bool):
    """The `config` object of the JSON line; both arms print the same one."""
    n_copies = n_pool_copies(w)
    return dict(_describe(w, plan), parallelism=f"replicas x{world} (one workload per GPU)",
                timed_steps="one CUDA graph of the K steps, replayed" if graph else "K steps queued from Python",
                l2=f"inputs larger than L2: back-to-back steps rotate over {n_copies} copies of the KV pool "
                   f"({n_copies * w.kv_bytes() / 2**20:.0f} MiB of step data); latency_us is flushed per step")


def time_e2e(w, K, W, torch, bd, flush):
    """Per-step wall times (ms) of synchronized pkv_decode_host calls from pinned host buffers."""
    q_h = w.q.cpu().pin_memory()
    bt_h = w.block_table.cpu().pin_memory()
    lens_h = torch.tensor(w.seq_lens, dtype=torch.int32).pin_memory()
    out_h = torch.empty_like(q_h).pin_memory()
    shape = bd.shape_of(w.q, w.k_pool, w.block_table)
    dec = bd.HostDecoder(w.q.device)
    dec.ensure(lens_h, shape)
    for i in range(W):
        flush(i)
        dec(q_h, bt_h, lens_h, out_h, w.k_pool, w.v_pool, w.scale, shape)
    times = []
    plan = None
    replays0 = bd.host_replays()
    for i in range(K):
        flush(i)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        plan = dec(q_h, bt_h, lens_h, out_h, w.k_pool, w.v_pool, w.scale, shape)
        times.append((time.perf_counter() - t0) * 1e3)
    replays = bd.host_replays() - replays0
    # where the time goes: the same calls once more through pkv_decode_host_timed
    # (host clock inside the library, CUDA events around the copies and kernels)
    parts = []
    for i in range(min(K, 50)):
        flush(i)
        torch.cuda.synchronize()
        tm = bd.HostTiming()
        t0 = time.perf_counter()
        dec(q_h, bt_h, lens_h, out_h, w.k_pool, w.v_pool, w.scale, shape, timing=tm)
        d = tm.as_dict()
        d["wall_us"] = (time.perf_counter() - t0) * 1e6
        parts.append(d)
    breakdown = {k: round(statistics.median(p[k] for p in parts), 2) for k in parts[0]}
    breakdown["binding_us"] = round(breakdown["wall_us"] - sum(breakdown[k] for k in (
        "host_plan_us", "host_enqueue_us", "host_wait_us", "host_unpack_us", "host_events_us")), 2)
    breakdown["note"] = ("medians over calls of pkv_decode_host_timed: host_* from the library's host clock (plan = "
                         "policy + queue + staging image; enqueue = copy and launches queued; wait = "
                         "cudaStreamSynchronize; unpack = the result read back; events = reading the events), dev_* "
                         "from CUDA events recorded between the copy and the kernels, which cost time of their own "
                         "and keep the kernel from starting early, so these calls run longer than the untimed ones "
                         "of us_per_step; timed calls queue the copy and launches themselves, never the graph the "
                         "untimed ones replay; binding_us = Python and ctypes around the call")
    counters = bd.plan_counters(w.seq_lens, shape, plan)
    h2d = q_h.numel() * 2 + bt_h.numel() * 4 + lens_h.numel() * 4 + counters["queue_bytes"]
    d2h = out_h.numel() * 2 + 16
    return times, h2d, d2h, out_h, breakdown, replays


def fill_budget(w, bd):
    """The fill budget T of the built-in rule that picks a work-queue plan for
    this batch (a rule with chunk_pages = 0), else None."""
    n_max = max(w.seq_lens, default=0)
    for r in bd.default_rules():
        if r.b_lo <= w.B < r.b_hi and r.nmax_lo <= n_max < r.nmax_hi:
            return r.num_splits if r.mode == bd.WORK_QUEUE and r.chunk_pages == 0 else None
    return None


def device_queue_timing(w, dp, K, W, torch, bd, copies):
    """Steady-state and interleaved µs per step of the plan whose blocks derive
    the queue from the device lengths (PKV_FLAG_DEVICE_FILL), beside the
    host-queue plan, for a work-queue batch; None for other plans."""
    T = fill_budget(w, bd)
    if dp.plan.mode != bd.WORK_QUEUE or T is None:
        return None
    shape = bd.shape_of(w.q, w.k_pool, w.block_table)
    dq = bd.plan_decode(w.seq_lens, shape, w.q.device, plan=dp.plan, device_queue=True, fill_blocks=T)
    steady = time_steady(w, dq, K, W, torch, bd, copies) / K
    inter, _ = time_interleaved(w, dq, K, W, torch, bd, copies, lens_jitter=True)
    host_inter, _ = time_interleaved(w, dp, K, W, torch, bd, copies)
    return {"plan": {"mode": "WORK_QUEUE", "fill_blocks": T, "flags": dq.plan.flags},
            "us_per_step": round(steady * 1e3, 2),
            "interleaved_us_per_step": round(inter / K * 1e3, 2),
            "host_queue_interleaved_us_per_step": round(host_inter / K * 1e3, 2),
            "note": "each block derives its item from the device lengths (no host queue, no builder kernel); "
                    "interleaved: after a 64 MiB HBM copy that also moves every length by one token each step "
                    "(host queue: fixed lengths)"}


def shared_prefix_timing(w, dp, K, W, torch, bd, copies):
    """Steady-state µs per step of the prefix-sharing plan beside the built-in
    one, for a workload whose rows share leading pages; None otherwise."""
    if w.shared_rows < 2:
        return None
    shape = bd.shape_of(w.q, w.k_pool, w.block_table)
    dpp = bd.plan_decode(w.seq_lens, shape, w.q.device, plan=dp.plan, shared_prefix_table=w.block_table.cpu())
    steady = time_steady(w, dpp, K, W, torch, bd, copies) / K
    # the same chunk size as a plain work queue: the sharing's own effect
    plain = bd.Plan(bd.WORK_QUEUE, 1, dpp.plan.chunk_pages, dpp.plan.flags & ~bd.FLAG_SHARED_PREFIX)
    dpq = bd.plan_decode(w.seq_lens, shape, w.q.device, plan=plain)
    steady_q = time_steady(w, dpq, K, W, torch, bd, copies) / K
    c = dpp.counters
    return {"plan": {"mode": "WORK_QUEUE", "units": dpp.plan.num_splits, "chunk_pages": dpp.plan.chunk_pages,
                     "flags": dpp.plan.flags}, "items": dpp.n_items, "us_per_step": round(steady * 1e3, 2),
            "same_chunk_work_queue_us_per_step": round(steady_q * 1e3, 2),
            "kv_bytes_streamed": c["kv_bytes_streamed"], "built_in_kv_bytes_streamed": dp.counters["kv_bytes_streamed"],
            "note": "shared chunks staged once per unit of up to 16/G sharing rows (PKV_FLAG_SHARED_PREFIX); "
                    "same_chunk_work_queue: the plain work queue with the same chunk, every row streaming its "
                    "own pages"}


def measure_workload(name, seed, device, K, W, torch, bd, W_mod, flush):
    w = W_mod.make(name, seed=seed, device=device)
    shape = bd.shape_of(w.q, w.k_pool, w.block_table)
    dp = bd.plan_decode(w.seq_lens, shape, device)
    copies = pool_copies(w, torch)
    steady = time_steady(w, dp, K, W, torch, bd, copies) / K
    early_plan = bd.Plan(dp.plan.mode, dp.plan.num_splits, dp.plan.chunk_pages, dp.plan.flags | bd.FLAG_PDL_EARLY)
    early = time_steady(w, bd.plan_decode(w.seq_lens, shape, device, plan=early_plan), K, W, torch, bd, copies) / K
    inter, _ = time_interleaved(w, dp, K, W, torch, bd, copies)
    dq = device_queue_timing(w, dp, K, W, torch, bd, copies)
    sp = shared_prefix_timing(w, dp, K, W, torch, bd, copies)
    del copies
    iso = time_isolated(w, dp, min(K, 50), min(W, 3), torch, bd, flush)
    return {"w": w, "dp": dp, "ms": steady, "early_ms": early, "inter_ms": inter / K, "device_queue": dq,
            "shared_prefix": sp, "iso_ms": statistics.median(iso), "bytes": w.algorithmic_bytes(),
            "bytes_unique": w.algorithmic_bytes(True)}


def cpu_baseline_leg(w, target_s):
    """The oracle as it stands (fp64 C, all host cores) on full decode steps of
    the workload, repeated until about target_s seconds of CPU time."""
    from oracle import oracle as O

    cores = os.cpu_count() or 1
    pr = O.problem(w.q.cpu(), w.k_pool.cpu(), w.v_pool.cpu(), w.block_table.cpu(), w.seq_lens, w.scale)
    t0 = time.perf_counter()
    O.paged_decode(pr, n_threads=cores)
    one = time.perf_counter() - t0
    reps = max(1, int(target_s / max(one, 1e-3)))
    t0 = time.perf_counter()
    for _ in range(reps):
        O.paged_decode(pr, n_threads=cores)
    dt = time.perf_counter() - t0
    return {"value": round(w.algorithmic_bytes() * reps / dt / 1e9, 4), "unit": "GB/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{reps} full decode step(s) of the {w.name} workload ({w.B * w.H_q} (row, head) outputs "
                      f"over {sum(w.seq_lens)} tokens each step), fp64, {dt:.1f} s",
            "us_per_step": round(dt / reps * 1e6, 1)}


def run_ours(args):
    import torch

    from paged_kv_gqa_17_b200 import binding as bd
    from paged_kv_gqa_17_b200 import workloads as W_mod

    rank, local_rank, world = dist_env()
    if world != args.gpus:
        if rank == 0:
            print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist = init_dist(world, "nccl", local_rank)
    bd.lib()
    seed = (args.seed if args.seed is not None else W_mod.SEED_REPORT) + rank
    flush = Flush(torch, device)
    peak, peak_src = measured_peak()

    # the headline workload: warm-up, then EXACTLY K timed steps between barriers
    w = W_mod.make(args.workload, seed=seed, device=device)
    shape = bd.shape_of(w.q, w.k_pool, w.block_table)
    dp = bd.plan_decode(w.seq_lens, shape, device,
                        shared_prefix_table=w.block_table.cpu() if args.shared_prefix else None)
    copies = pool_copies(w, torch)
    barrier(dist, device)
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        steady_ms = time_steady(w, dp, args.steps, args.warmup, torch, bd, copies, graph=not args.no_graph)
    torch.cuda.synchronize()
    barrier(dist, device)
    del copies
    total_ms = max_over_ranks(steady_ms, dist, device)
    total_bytes = sum_over_ranks(float(w.algorithmic_bytes() * args.steps), dist, device)
    ms = time_isolated(w, dp, min(args.steps, 200), min(args.warmup, 5), torch, bd, flush)
    # the same steps with the opt-in early start (PKV_FLAG_PDL_EARLY): valid here
    # because the kernel before each step is the previous step, which writes
    # none of the lengths, table or K/V pages; reported beside the headline only
    copies = pool_copies(w, torch)
    early_ms = None
    if not args.shared_prefix:  # the prefix-sharing grid always waits first
        early_plan = bd.Plan(dp.plan.mode, dp.plan.num_splits, dp.plan.chunk_pages,
                             dp.plan.flags | bd.FLAG_PDL_EARLY)
        dp_early = bd.plan_decode(w.seq_lens, shape, device, plan=early_plan)
        early_ms = time_steady(w, dp_early, args.steps, args.warmup, torch, bd, copies,
                               graph=not args.no_graph) / args.steps
        del dp_early
    inter_k = min(args.steps, 200)
    inter_ms, filler_ms = time_interleaved(w, dp, inter_k, min(args.warmup, 5), torch, bd, copies)
    dq = device_queue_timing(w, dp, min(args.steps, 200), min(args.warmup, 5), torch, bd, copies)
    del copies
    e2e_ms, h2d, d2h, _, e2e_parts, e2e_replays = time_e2e(w, args.e2e_steps or args.steps, min(args.warmup, 3),
                                                           torch, bd, flush)
    e2e_total = max_over_ranks(sum(e2e_ms), dist, device)
    e2e_bytes = sum_over_ranks(float(w.algorithmic_bytes() * len(e2e_ms)), dist, device)

    counters = dp.counters
    step_ms = steady_ms / args.steps
    achieved = w.algorithmic_bytes() / (step_ms * 1e-3) / 1e9
    iso_ms = statistics.median(ms)
    line = {
        "metric": METRIC,
        "value": round(total_bytes / (total_ms * 1e-3) / 1e9, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 6),
        "us_per_step": round(total_ms / args.steps * 1e3, 3),
        "latency_us": round(iso_ms * 1e3, 2),
        "latency_us_p10_p90": [round(x * 1e3, 2) for x in statistics.quantiles(ms, n=10)[::8]]
        if len(ms) >= 10 else None,
        "latency_GB_s": round(w.algorithmic_bytes() / (iso_ms * 1e-3) / 1e9, 1),
        "pdl_early": None if early_ms is None else {
            "us_per_step": round(early_ms * 1e3, 3),
            "GB_s": round(w.algorithmic_bytes() / (early_ms * 1e-3) / 1e9, 2),
            "note": "same steady-state timing with PKV_FLAG_PDL_EARLY (the caller promises the preceding "
                    "kernel writes no length, table or K/V page but a row's last); opt-in, not the headline",
        },
        "interleaved": {
            "us_per_step": round(inter_ms / inter_k * 1e3, 3),
            "GB_s": round(w.algorithmic_bytes() / (inter_ms / inter_k * 1e-3) / 1e9, 2),
            "filler_us_per_step": round(filler_ms / inter_k * 1e3, 3),
            "note": "each step after a 64 MiB HBM copy kernel (a projection's stand-in), the copy's own time "
                    "subtracted: the step without a preceding decode step to overlap with",
        },
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded bf16 N(0,1) q/K/V, random page placement)",
        "config": arm_config(w, dp.plan, world, not args.no_graph),
        "frac_of_nominal_8TBs": round(achieved / NOMINAL_HBM_GBS, 4),
        "roofline": {
            "bound": "hbm",
            "kernel": ("prefix_kernel" if dp.plan.flags & bd.FLAG_SHARED_PREFIX else "split_kernel") +
                      (" (fused merge)" if counters["launches"] == 1 else " + merge_kernel"),
            "achieved": round(achieved, 2),
            "peak": peak,
            "peak_source": f"{peak_src} HBM copy bandwidth",
            "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": recorded_traffic(args.workload),
            "algorithmic_bytes_per_launch": w.algorithmic_bytes(),
        },
        "e2e": {
            "value": round(e2e_bytes / (e2e_total * 1e-3) / 1e9, 2),
            "unit": "GB/s",
            "us_per_step": round(e2e_total / len(e2e_ms) * 1e3, 2),
            "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h,
            "note": "synchronized pkv_decode_host per step: host plan + queue, one H2D copy of "
                    "q/table/lengths/queue from pinned memory, kernels that write out (and any error flags) straight "
                    "into the caller's pinned host buffers over the bus; KV cache resident; from the second call "
                    "with the same buffers and plan the copy and the launches are one replayed CUDA graph",
            "graph_replays": e2e_replays,
            "breakdown": e2e_parts,
        },
        "gpu_launches": int(counters["launches"] * args.steps),
        **({"device_queue": dq} if dq is not None else {}),
        "counters": counters,
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu:
        host_w = dataclasses.replace(w, q=w.q.cpu(), k_pool=w.k_pool.cpu(), v_pool=w.v_pool.cpu(),
                                     block_table=w.block_table.cpu())
        line["cpu_baseline"] = cpu_baseline_leg(host_w, args.cpu_seconds)
        del host_w
    if world == 1 and not args.no_extra:
        extra = {}
        for name in ("crossover", "mixed", "prefix", "tiny"):
            if name == args.workload:
                continue
            r = measure_workload(name, seed, device, min(args.steps, 200), min(args.warmup, 5), torch, bd, W_mod,
                                 flush)
            m = r["ms"]
            gbs = r["bytes"] / (m * 1e-3) / 1e9
            extra[name] = {"config": _describe(r["w"], r["dp"].plan)["workload"],
                           "plan": _describe(r["w"], r["dp"].plan)["plan"],
                           "us_per_step": round(m * 1e3, 2), "GB_s": round(gbs, 1),
                           "latency_us": round(r["iso_ms"] * 1e3, 2),
                           "interleaved_us_per_step": round(r["inter_ms"] * 1e3, 2),
                           "pdl_early_us_per_step": round(r["early_ms"] * 1e3, 2),
                           "frac_of_measured": round(gbs / peak, 4),
                           "frac_of_nominal_8TBs": round(gbs / NOMINAL_HBM_GBS, 4),
                           "launches": r["dp"].counters["launches"]}
            if r["device_queue"] is not None:
                extra[name]["device_queue"] = r["device_queue"]
            if r["shared_prefix"] is not None:
                extra[name]["shared_prefix"] = r["shared_prefix"]
            if r["bytes_unique"] != r["bytes"]:
                gbu = r["bytes_unique"] / (m * 1e-3) / 1e9
                extra[name]["GB_s_unique"] = round(gbu, 1)
                extra[name]["frac_of_measured_unique"] = round(gbu / peak, 4)
            del r
            torch.cuda.empty_cache()
        line["all_workloads"] = extra
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def run_reference(args):
    """The reference arm: the CPU oracle as it stands, on the host cores."""
    rank, _, world = dist_env()
    if rank != 0:
        return
    import torch  # noqa: F401

    from paged_kv_gqa_17_b200 import workloads as W_mod
    from oracle import oracle as O

    seed = args.seed if args.seed is not None else W_mod.SEED_REPORT
    w = W_mod.make(args.workload, seed=seed)
    pr = O.problem(w.q, w.k_pool, w.v_pool, w.block_table, w.seq_lens, w.scale)
    # the plan our arm runs, from the oracle's own policy lookup over the built-in
    # table (bit-identical to the library's), so that both lines carry one config
    rules = O.load_rules(os.path.join(ROOT, "paged_kv_gqa_17_b200", "policy_b200.json"))
    plan = type("Plan", (), dict(zip(("mode", "num_splits", "chunk_pages", "flags"),
                                     O.select_policy(w.seq_lens, w.P, rules, w.H_kv))))
    cores = os.cpu_count() or 1
    for _ in range(args.warmup):
        O.paged_decode(pr, n_threads=cores)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        O.paged_decode(pr, n_threads=cores)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = round(w.algorithmic_bytes() * args.steps / total / 1e9, 4)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": arm_config(w, plan, world, not args.no_graph),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"full decode steps of the {w.name} workload, fp64 C oracle, {cores} threads"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    line["reference_method"] = "fp64 two-pass softmax per (row, head), no split (the CPU oracle)"
    print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
