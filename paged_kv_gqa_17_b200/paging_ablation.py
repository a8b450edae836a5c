"""Paging-overhead ablation on B200: how much the block-table indirection and
the pool layout cost.

    python -m paged_kv_gqa_17_b200.paging_ablation [--out REPORT.md]

"Chapter 8 - Next-generation KV cache management" (actionbridge.io), section
8.1, states that a paged kernel runs within a few percent of a kernel over a
contiguous ("slab") cache.  This script measures it for this library:

  - permuted: the workload as generated, each row's pages scattered at random
    over the pool;
  - identity: the same K/V values gathered so that each row's pages are
    consecutive physical pages in block-table order (a contiguous cache seen
    through an identity table);
  - NHD: the permuted workload with the pool laid out [pages][16][H_kv][D]
    instead of [pages][H_kv][16][D].

Same plan (the built-in policy's) for all three; steady-state µs per step
(back-to-back steps replayed from a CUDA graph, rotating pool copies).
"""
from __future__ import annotations

import argparse
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def identity_copy(w, torch):
    """The workload with each row's pages moved to consecutive physical ids."""
    import dataclasses

    order = []
    tables = []
    for i, n in enumerate(w.seq_lens):
        pages = w.block_table[i, :-(-n // w.P)].tolist() if n else []
        tables.append(list(range(len(order), len(order) + len(pages))))
        order += pages
    idx = torch.tensor(order if order else [0], dtype=torch.long, device=w.k_pool.device)
    k = w.k_pool.index_select(0, idx).contiguous()
    v = w.v_pool.index_select(0, idx).contiguous()
    bt = torch.zeros_like(w.block_table)
    for i, t in enumerate(tables):
        if t:
            bt[i, :len(t)] = torch.tensor(t, dtype=torch.int32)
    return dataclasses.replace(w, k_pool=k, v_pool=v, block_table=bt, num_pages=int(idx.numel()))


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--out", default=None, help="also write the markdown report to this file")
    ap.add_argument("--steps", type=int, default=300)
    args = ap.parse_args(argv)

    import torch

    from paged_kv_gqa_17_b200 import binding as bd
    from paged_kv_gqa_17_b200 import timing as T
    from paged_kv_gqa_17_b200 import workloads as W

    dev = torch.device("cuda")
    lines = ["# Paging-overhead ablation (B200)", "",
             "Command: `python -m paged_kv_gqa_17_b200.paging_ablation" + (f" --out {args.out}" if args.out else "") + "`. Same values, same plan (built-in policy); "
             "steady-state µs per step (CUDA-graph replay of back-to-back steps over rotating pool copies).", "",
             "| workload | plan | permuted HND | identity HND | permuted NHD | identity / permuted |",
             "|---|---|---|---|---|---|"]
    for name in ("long", "crossover", "mixed"):
        res = {}
        w = W.make(name, device=dev)
        shape = bd.shape_of(w.q, w.k_pool, w.block_table)
        plan = bd.select_policy(w.seq_lens, shape)
        variants = (("permuted HND", w), ("identity HND", identity_copy(w, torch)),
                    ("permuted NHD", W.make(name, device=dev, layout="NHD")))
        for label, v in variants:
            vshape = bd.shape_of(v.q, v.k_pool, v.block_table, v.layout)
            dp = bd.plan_decode(v.seq_lens, vshape, dev, plan=plan)
            copies = T.pool_copies(v, torch)
            res[label] = T.time_steady(v, dp, args.steps, 5, torch, bd, copies) / args.steps * 1e3
            del copies
            print(name, label, f"{res[label]:.2f} us", flush=True)
        lines.append(f"| {name} | {plan.tuple()} | {res['permuted HND']:.2f} | {res['identity HND']:.2f} | "
                     f"{res['permuted NHD']:.2f} | {res['identity HND'] / res['permuted HND']:.3f} |")
        torch.cuda.empty_cache()
    if args.out:
        os.makedirs(os.path.dirname(os.path.abspath(args.out)), exist_ok=True)
        with open(args.out, "w") as f:
            f.write("\n".join(lines) + "\n")
    print("\n".join(lines))


if __name__ == "__main__":
    main()
