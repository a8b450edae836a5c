"""Helpers shared by the GPU tests: run the CUDA path, run the oracle on the
same inputs, and compare within the stated tolerance."""
from __future__ import annotations

import numpy as np
import torch

from oracle import oracle as O
from paged_kv_gqa_17_b200 import binding as bd
from paged_kv_gqa_17_b200 import workloads as W

# bf16 inputs, fp32 accumulation, bf16 output:
#   |gpu - ref| <= ATOL + RTOL * |ref|   element-wise
ATOL = 4e-3
RTOL = 1e-2


def to_device(w: W.Workload, device="cuda") -> W.Workload:
    w.q, w.k_pool, w.v_pool = w.q.to(device), w.k_pool.to(device), w.v_pool.to(device)
    w.block_table = w.block_table.to(device)
    return w


def run(w: W.Workload, plan=None, rules=None, mode_rule=None):
    """Decode one step of w on the GPU; returns (out as float64 numpy, DecodePlan)."""
    shape = bd.shape_of(w.q, w.k_pool, w.block_table, w.layout)
    if mode_rule is not None:
        rules = [mode_rule]
    dp = bd.plan_decode(w.seq_lens, shape, w.q.device, rules=rules, plan=plan)
    lens_dev = torch.tensor(w.seq_lens, dtype=torch.int32, device=w.q.device)
    out = bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table, lens_dev, w.P, w.scale, plan=dp,
                          layout=w.layout)
    torch.cuda.synchronize()
    err = bd.workspace_status(dp)
    assert err == 0, f"device error mask {err}"
    return out.float().cpu().double().numpy(), dp


def oracle_full(w: W.Workload, threads=8) -> np.ndarray:
    pr = O.problem(w.q.cpu(), w.k_pool.cpu(), w.v_pool.cpu(), w.block_table.cpu(), w.seq_lens, w.scale,
                   layout=w.layout)
    return O.paged_decode(pr, n_threads=threads)


def oracle_sampled(w: W.Workload, pairs, threads=8) -> np.ndarray:
    """Oracle outputs for the listed (row, query head) pairs only.  Only the
    pages those rows use are copied to the host (a pure gather: pages are
    renumbered in a compact pool, the block table rewritten to match)."""
    rows = sorted({r for r, _ in pairs})
    bt = w.block_table.cpu()
    used = []
    for r in rows:
        used += bt[r, :-(-w.seq_lens[r] // w.P)].tolist() if w.seq_lens[r] else []
    uniq = sorted(set(used))
    remap = {p: i for i, p in enumerate(uniq)}
    idx = torch.tensor(uniq if uniq else [0], dtype=torch.long, device=w.k_pool.device)
    k = w.k_pool.index_select(0, idx).cpu()
    v = w.v_pool.index_select(0, idx).cpu()
    sub_bt = torch.zeros((len(rows), bt.shape[1]), dtype=torch.int32)
    for j, r in enumerate(rows):
        n = -(-w.seq_lens[r] // w.P)
        sub_bt[j, :n] = torch.tensor([remap[p] for p in bt[r, :n].tolist()], dtype=torch.int32)
    q = w.q[rows].cpu()
    pr = O.problem(q, k, v, sub_bt, [w.seq_lens[r] for r in rows], w.scale, layout=w.layout)
    row_of = {r: j for j, r in enumerate(rows)}
    return O.paged_decode_pairs(pr, [(row_of[r], hq) for r, hq in pairs], n_threads=threads)


def assert_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} elements out of tolerance; worst at {i}: "
                             f"gpu {got[i]!r} ref {ref[i]!r}")


def rel_l2(got: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
