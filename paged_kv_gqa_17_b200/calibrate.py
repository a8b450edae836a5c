"""Calibrate the built-in policy table on the GPU from measured timings.

    python -m paged_kv_gqa_17_b200.calibrate [--out paged_kv_gqa_17_b200/policy_b200.json] [--report REPORT.md]
        [--steps 60] [--draws 3]

The policy maps (batch size B, longest row N_max) to an execution plan
[PersistentKV explainer, Technical summary > Methodology > 2 "Calibrated
adaptive policy": thresholds calibrated by hand on one seed, results reported
on a holdout seed].  This script does the same by measurement:

  1. For every cell of a (B, N_max) grid it draws three batches with the
     calibration seed 20260622: one row of the cell's representative length,
     the others log-uniform between 1/8, 1/64 and 1/512 of it (one batch
     each) and it (H_kv=8, D=128, 16-token pages; G = 4 for the first two
     batches, G = 8 for the third).
  2. It times every candidate plan (no-split; split-S over several S with
     and without the deep ring, and with the cluster merge at S = 8 and 16;
     the work queue over ten chunk sizes from 8 to 512 pages, with and
     without the deep ring,
     and with the chunk size that fills one wave of 222 to 444 blocks; the
     balanced grid at one and two blocks per SM) as the steady-state device
     time of back-to-back steps over rotating pool copies.
  3. The plan with the smallest geometric-mean time over the cell's batches
     becomes a rule (within 1 % of it, the simplest plan: no-split, split-S,
     queue, balanced, then fewest flags); neighbouring cells of one B with the
     same plan are merged.
  4. Every cell is re-measured with the holdout seed 20260623; the report
     lists the chosen plan's time against the best candidate (the regret).

It writes the table as JSON (the library's build turns it into its built-in
table) and prints a markdown report (also written to --report when given).
With --only-b B it re-measures only the cells of B's row and replaces that
row's rules in the existing table, keeping every other rule.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

B_EDGES = [1, 2, 4, 8, 16, 32, 2**31 - 1]          # rules cover [B_EDGES[i], B_EDGES[i+1])
N_EDGES = [0, 1024, 4096, 16384, 65536, 2**31 - 1]  # and [N_EDGES[j], N_EDGES[j+1])
N_REP = [512, 2048, 8192, 32768, 131072]            # representative N_max of each N range
B_REP = [1, 2, 4, 8, 16, 64]                        # representative B of each B range
MODE_NAMES = {0: "NO_SPLIT", 1: "SPLIT_S", 2: "WORK_QUEUE", 3: "BALANCED"}


def candidates():
    """(mode, num_splits, chunk_pages, flags) rules to try in every cell."""
    out = [(0, 1, 0, 0)]
    for S in (8, 16, 32, 37, 64):
        out += [(1, S, 0, 0), (1, S, 0, 4)]
    for S in (8, 16):
        out.append((1, S, 0, 12))  # cluster merge, deep ring
    for C in (8, 16, 24, 32, 48, 64, 96, 128, 256, 512):
        out += [(2, 1, C, 0), (2, 1, C, 4)]
    # C chosen to fill one wave of T blocks: about 1.5, 1.8 and 2 blocks per SM with
    # the deep ring (two fit per SM), 2 and 3 per SM with the 8-page ring
    out += [(2, 222, 0, 4), (2, 264, 0, 4), (2, 296, 0, 4), (2, 296, 0, 0), (2, 444, 0, 0)]
    out += [(3, 296, 0, 0), (3, 148, 0, 4)]
    return out


def cell_lengths(B: int, n_rep: int, seed: int, draw: int = 0):
    import torch

    g = torch.Generator().manual_seed(seed * 1000 + B * 7 + n_rep + 100003 * draw)
    lo = max(16, n_rep // (8, 64, 512)[draw % 3])  # mild, strong and extreme length skew
    rest = torch.rand(max(0, B - 1), generator=g, dtype=torch.float64)
    lens = [n_rep] + [int(math.exp(math.log(lo) + float(u) * (math.log(n_rep) - math.log(lo)))) for u in rest]
    return lens


def measure_cell(B, n_rep, seed, steps, cands, torch, bd, W, bench, draws=1):
    """Geometric mean over `draws` batches of the cell of each candidate's
    steady-state µs per step."""
    dev = torch.device("cuda")
    logs = {c: 0.0 for c in cands}
    for d in range(draws):
        H_q = 64 if d % 3 == 2 else 32  # G = 4, and G = 8 for the third batch
        w = W.make_custom(cell_lengths(B, n_rep, seed, d), H_q, 8, 128, seed=seed + d, device=dev)
        shape = bd.shape_of(w.q, w.k_pool, w.block_table)
        copies = bench.pool_copies(w, torch)
        for c in cands:
            rule = bd.Rule(0, 2**31 - 1, 0, 2**31 - 1, *c)
            dp = bd.plan_decode(w.seq_lens, shape, dev, rules=[rule])
            us = bench.time_steady(w, dp, steps, 3, torch, bd, copies) / steps * 1e3
            logs[c] += math.log(us) / draws
        del copies, w
        torch.cuda.empty_cache()
    return {c: math.exp(v) for c, v in logs.items()}


TIE = 0.01  # timings closer than this cannot tell two plans apart


def pick(times):
    """The fastest candidate; among those within TIE of it, the simplest plan
    (fewest device-side steps: no-split, split-S, queue, balanced; then the
    fewest flags), since their measured difference is below the noise."""
    fastest = min(times.values())
    near = [c for c, t in times.items() if t <= fastest * (1 + TIE)]
    return min(near, key=lambda c: (c[0], bin(c[3]).count("1"), times[c]))


def build_rules(best, rows):
    """best[(bi, nj)] -> candidate; merge equal neighbours along N for each B range in rows."""
    rules = []
    for bi in rows:
        nj = 0
        while nj < len(N_REP):
            c = best[(bi, nj)]
            nk = nj
            while nk + 1 < len(N_REP) and best[(bi, nk + 1)] == c:
                nk += 1
            mode, S, C, flags = c
            r = {"b_lo": B_EDGES[bi], "b_hi": B_EDGES[bi + 1], "nmax_lo": N_EDGES[nj], "nmax_hi": N_EDGES[nk + 1],
                 "mode": MODE_NAMES[mode]}
            if mode in (1, 3):
                r["num_splits"] = S
            if mode == 2:
                if C > 0:
                    r["chunk_pages"] = C
                else:
                    r["num_splits"] = S  # the item budget of the fill rule
                    r["chunk_pages"] = 0
            if flags:
                r["flags"] = flags
            rules.append(r)
            nj = nk + 1
    return rules


def replace_row(old_rules, row_rules, b_lo):
    """The table with the rules of the B range starting at b_lo replaced by
    row_rules, ordered by (b_lo, nmax_lo)."""
    rules = [r for r in old_rules if r["b_lo"] != b_lo] + list(row_rules)
    return sorted(rules, key=lambda r: (r["b_lo"], r["nmax_lo"]))


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--out", default=os.path.join(HERE, "policy_b200.json"))
    ap.add_argument("--report", default=None, help="also write the markdown report to this file")
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--draws", type=int, default=3, help="batches per cell (geometric mean)")
    ap.add_argument("--only-b", type=int, default=None, choices=B_REP,
                    help="re-measure only this representative B's row; keep the table's other rules")
    args = ap.parse_args(argv)
    rows = [B_REP.index(args.only_b)] if args.only_b is not None else list(range(len(B_REP)))

    import torch

    from paged_kv_gqa_17_b200 import binding as bd
    from paged_kv_gqa_17_b200 import timing as bench
    from paged_kv_gqa_17_b200 import workloads as W

    bd.lib()
    cands = candidates()
    best, calib = {}, {}
    for bi in rows:
        B = B_REP[bi]
        for nj, n in enumerate(N_REP):
            t = measure_cell(B, n, W.SEED_CALIBRATE, args.steps, cands, torch, bd, W, bench, args.draws)
            calib[(bi, nj)] = t
            best[(bi, nj)] = pick(t)
            print(f"B={B:3d} N_max={n:6d} best {best[(bi, nj)]} {t[best[(bi, nj)]]:.2f} us", flush=True)
    rules = build_rules(best, rows)
    if args.only_b is not None:
        with open(args.out) as f:
            rules = replace_row(json.load(f)["rules"], rules, B_EDGES[rows[0]])
    doc = {
        "name": "b200_calibrated",
        "about": "Built-in policy table of libpkv.so (pkv_default_policy), written by "
                 "paged_kv_gqa_17_b200/calibrate.py from steady-state timings on B200 with seed 20260622 "
                 "(H_kv=8, G=4 and 8, D=128, 16-token pages). Rules are checked in order; the first whose "
                 "half-open ranges hold (B, N_max) decides.",
        "rules": rules,
    }
    with open(args.out, "w") as f:
        json.dump(doc, f, indent=1)
        f.write("\n")
    # holdout check
    lines = ["# Policy calibration on B200", "",
             "Command: `python -m paged_kv_gqa_17_b200.calibrate" + (f" --report {args.report}" if args.report else "")
             + (f" --only-b {args.only_b}" if args.only_b is not None else "")
             + "` (writes paged_kv_gqa_17_b200/policy_b200.json).", "",
             "Steady-state µs per decode step (CUDA-graph replay of back-to-back steps over rotating pool copies), "
             f"H_kv=8, D=128; each cell is the geometric mean over {args.draws} batches (G = 4, 4, 8). "
             "Calibration seed 20260622 picks the plan; holdout seed 20260623 (other batches) re-measures it.", "",
             "| B | N_max | chosen plan (mode, S/T, C, flags) | calib µs | holdout µs | holdout best | best µs | regret |",
             "|---|---|---|---|---|---|---|---|"]
    for bi in rows:
        B = B_REP[bi]
        for nj, n in enumerate(N_REP):
            c = best[(bi, nj)]
            hold = measure_cell(B, n, W.SEED_REPORT, args.steps, cands, torch, bd, W, bench, args.draws)
            hb = min(hold, key=hold.get)
            lines.append(f"| {B} | {n} | {MODE_NAMES[c[0]]} {c[1:]} | {calib[(bi, nj)][c]:.2f} | {hold[c]:.2f} | "
                         f"{MODE_NAMES[hb[0]]} {hb[1:]} | {hold[hb]:.2f} | {100 * (hold[c] / hold[hb] - 1):.1f}% |")
            print(lines[-1], flush=True)
    if args.report:
        os.makedirs(os.path.dirname(os.path.abspath(args.report)), exist_ok=True)
        with open(args.report, "w") as f:
            f.write("\n".join(lines) + "\n")
    print("\n".join(lines))
    print(f"wrote {args.out}" + (f" and {args.report}" if args.report else ""))


if __name__ == "__main__":
    main()
