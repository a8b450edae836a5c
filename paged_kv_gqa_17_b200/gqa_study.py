"""What the group size G = H_q / H_kv costs the tensor-core decode path.

    python -m paged_kv_gqa_17_b200.gqa_study [--out REPORT.md] [--steps 200]

The split kernel computes S^T = K Q^T and O^T += V^T P^T for the G query
heads of one KV head with warp-level tensor-core MMAs whose n = 8 (16 for G
> 8) carries the heads, so G < 8 pads the MMA's columns with zeros.  Decode
reads every K/V byte once whatever G is [PersistentKV explainer, Technical
summary > Methodology > 1: GQA, G heads share a KV head], so if the MMAs
cost nothing the step time must not depend on G.  This script times the long
context (B=1, 8 KV heads, D=128, 32768 tokens, the same 134 MB of K/V) at
G = 1, 2, 4, 8, 16 in the built-in policy's plan, steady state (CUDA-graph
replay of back-to-back steps over rotating pool copies), after a 64 MiB
streaming kernel (interleaved), and cold (L2 flushed).
"""
from __future__ import annotations

import argparse
import os
import statistics
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

VARIANTS = (("long_g1", 1), ("long_g2", 2), ("long", 4), ("long_g8", 8), ("long_g16", 16))


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
    flush = T.Flush(torch, dev)
    lines = ["# Group size G against step time (B200)", "",
             "Command: `python -m paged_kv_gqa_17_b200.gqa_study" + (f" --out {args.out}" if args.out else "") +
             "`. Long context, B=1, 8 KV heads, D=128, N=32768 (134 MB of K/V at every G), built-in policy's "
             "plan; µs per step and GB/s of K/V + q + out.", "",
             "| G | H_q | plan | steady µs | GB/s | interleaved µs | cold µs |", "|---|---|---|---|---|---|---|"]
    for name, G in VARIANTS:
        w = W.make(name, device=dev)
        shape = bd.shape_of(w.q, w.k_pool, w.block_table)
        dp = bd.plan_decode(w.seq_lens, shape, dev)
        copies = T.pool_copies(w, torch)
        steady = min(T.time_steady(w, dp, args.steps, 10, torch, bd, copies) / args.steps for _ in range(3))
        inter, _ = T.time_interleaved(w, dp, min(args.steps, 100), 5, torch, bd, copies)
        cold = statistics.median(T.time_isolated(w, dp, 30, 3, torch, bd, flush))
        del copies
        gbs = w.algorithmic_bytes() / (steady * 1e-3) / 1e9
        lines.append(f"| {G} | {w.H_q} | {dp.plan.tuple()} | {steady * 1e3:.2f} | {gbs:.0f} | "
                     f"{inter / min(args.steps, 100) * 1e3:.2f} | {cold * 1e3:.2f} |")
        print(lines[-1], flush=True)
        del w
        torch.cuda.empty_cache()
    if args.out:
        os.makedirs(os.path.dirname(os.path.abspath(args.out)), exist_ok=True)
        with open(args.out, "w") as f:
            f.write("\n".join(lines) + "\n")
    print("\n".join(lines))


if __name__ == "__main__":
    main()
