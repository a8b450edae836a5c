"""Scheduler study on B=8 traces: launch fan-out, merge-state traffic, time.

    python -m paged_kv_gqa_17_b200.trace_study [--out REPORT.md]

The PersistentKV explainer (Technical summary > Results, scheduling overhead)
reports on a bimodal B=8 trace that the compact work queue cut launch fan-out
from 16.00 launches per step (exact-length buckets) to 2.00 and merge-state
traffic by about 37 %; its Bimodal / Uniform / Zipf trace parameters are not
published.  This script runs the same comparison on the generated B=8 traces
of workloads.py (bimodal, uniform, zipf, plus the mixed workload):

  - launches per step: exact-length bucketing (one split and one merge launch
    per distinct length), the compact queue with a separate merge kernel (the
    pages' two launches), the queue with the merge fused (one launch);
  - merge-state bytes of the rectangular split grid against the compact queue
    at the same chunk size (the library's closed-form counters);
  - steady-state µs per step of no-split, split-S, the queue (fused and
    separate merge), the balanced grid and the built-in policy's plan.
"""
from __future__ import annotations

import argparse
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

TRACES = ("bimodal", "uniform", "zipf", "mixed")
CHUNK = 16  # pages per chunk for the rectangular-vs-queue comparison


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--out", default=None, help="also write the markdown report to this file")
    ap.add_argument("--steps", type=int, default=200)
    args = ap.parse_args(argv)

    import torch

    from paged_kv_gqa_17_b200 import binding as bd
    from paged_kv_gqa_17_b200 import timing as T
    from paged_kv_gqa_17_b200 import workloads as W

    dev = torch.device("cuda")
    lines = ["# Scheduler study on B=8 traces (B200)", "",
             "Command: `python -m paged_kv_gqa_17_b200.trace_study" + (f" --out {args.out}" if args.out else "") + "`. Traces from workloads.py (seed 20260623; "
             "generated parameters, the pages publish none). H_q=32, H_kv=8, D=128, 16-token pages. Times are "
             "steady-state µs per step (back-to-back steps over rotating pool copies).", "",
             f"Counters (closed form, library `pkv_plan_counters`), chunk C = {CHUNK} pages:", "",
             "| trace | lengths | bucket launches | queue launches (separate / fused) | rect. merge bytes | "
             "queue merge bytes | saved |",
             "|---|---|---|---|---|---|---|"]
    timing_rows = []
    for name in TRACES:
        w = W.make(name, device=dev)
        shape = bd.shape_of(w.q, w.k_pool, w.block_table)
        pm = -(-max(w.seq_lens) // 16)
        S = -(-pm // CHUNK)
        rect = bd.plan_counters(w.seq_lens, shape, bd.Plan(1, S, CHUNK, 1))
        wq_sep = bd.plan_counters(w.seq_lens, shape, bd.Plan(2, S, CHUNK, 1))
        wq_fused = bd.plan_counters(w.seq_lens, shape, bd.Plan(2, S, CHUNK, 0))
        saved = 1 - wq_sep["merge_state_bytes"] / rect["merge_state_bytes"] if rect["merge_state_bytes"] else 0.0
        lines.append(f"| {name} | {w.seq_lens} | {wq_sep['bucket_launches']} | {wq_sep['launches']} / "
                     f"{wq_fused['launches']} | {rect['merge_state_bytes']} | {wq_sep['merge_state_bytes']} | "
                     f"{100 * saved:.1f}% |")
        copies = T.pool_copies(w, torch)
        plans = {"no-split": bd.Plan(0, 1, 0, 0), f"split-S C={CHUNK}": bd.Plan(1, S, CHUNK, 0),
                 f"queue C={CHUNK} fused": bd.Plan(2, S, CHUNK, 0),
                 f"queue C={CHUNK} separate": bd.Plan(2, S, CHUNK, 1),
                 "balanced 296": bd.Plan(3, 296, 0, 0)}
        default = bd.select_policy(w.seq_lens, shape)
        plans[f"policy {default.tuple()}"] = default
        row = [name]
        for label, plan in plans.items():
            dp = bd.plan_decode(w.seq_lens, shape, dev, plan=plan)
            us = T.time_steady(w, dp, args.steps, 5, torch, bd, copies) / args.steps * 1e3
            row.append((label, us, w.algorithmic_bytes() / us / 1e3))
            print(name, label, f"{us:.2f} us", flush=True)
        timing_rows.append(row)
        del copies, w
        torch.cuda.empty_cache()
    lines += ["", "Steady-state µs per step (GB/s of K/V + q + out in parentheses):", ""]
    header = [lab for lab, _, _ in timing_rows[0][1:-1]] + ["built-in policy"]
    lines.append("| trace | " + " | ".join(header) + " |")
    lines.append("|---|" + "---|" * len(header))
    for row in timing_rows:
        cells = [f"{us:.2f} ({gbs:.0f})" for _, us, gbs in row[1:]]
        cells[-1] = f"{row[-1][0][7:]}: {cells[-1]}"
        lines.append(f"| {row[0]} | " + " | ".join(cells) + " |")
    if args.out:
        os.makedirs(os.path.dirname(os.path.abspath(args.out)), exist_ok=True)
        with open(args.out, "w") as f:
            f.write("\n".join(lines) + "\n")
    print("\n".join(lines))


if __name__ == "__main__":
    main()
