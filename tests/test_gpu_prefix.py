"""Prefix-aware scheduling on the GPU (PKV_FLAG_SHARED_PREFIX): rows whose
block tables share leading physical pages get their shared chunks staged
once per unit of up to 16 / G rows.  Every output against the oracle, on
NaN-poisoned pools, for every G the fast path supports; the full prefix
workload (B = 64, G = 8, a 2048-token prefix shared by 16 rows)."""
import os

import numpy as np
import pytest
import torch

from paged_kv_gqa_17_b200 import binding as bd
from paged_kv_gqa_17_b200 import workloads as W

from .gpu_util import assert_close, oracle_full, rel_l2, to_device

pytestmark = pytest.mark.gpu

ANY = (0, 2**31 - 1, 0, 2**31 - 1)
CORES = os.cpu_count() or 8


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_gqa_17_b200 import build

    build.build()
    bd.lib()


def run_prefix(w, C, flags=0):
    shape = bd.shape_of(w.q, w.k_pool, w.block_table)
    plan = bd.Plan(2, 1, C, flags)
    dp = bd.plan_decode(w.seq_lens, shape, "cuda", plan=plan, shared_prefix_table=w.block_table.cpu())
    assert dp.plan.flags & bd.FLAG_SHARED_PREFIX and dp.plan.chunk_pages == C
    lens = torch.tensor(w.seq_lens, dtype=torch.int32, device="cuda")
    out = bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table, lens, w.P, w.scale, plan=dp)
    torch.cuda.synchronize()
    assert bd.workspace_status(dp) == 0, f"device error, plan {dp.plan}"
    return out.float().cpu().double().numpy(), dp


# lens, shared rows, shared pages, H_q, H_kv: sharers of every length class (shorter than
# the prefix, exactly the prefix, a partial page past it, far past it) and unrelated rows
CASES = {
    "g8": ([700, 320, 321, 5000, 333, 1000, 17, 0, 2500, 64], 6, 20, 16, 2),
    "g4": ([330, 330, 331, 900, 47, 2000, 600, 1], 5, 20, 8, 2),
    "g2": ([400, 401, 402, 403, 404, 405, 406, 407, 408, 2000], 9, 25, 8, 4),
    "g1": ([256] * 18 + [1000], 18, 16, 2, 2),
    "g16": ([1200, 1200, 99], 2, 40, 32, 2),
}


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("C", [1, 3, 7, 64])
def test_prefix_plan_every_output(case, C):
    lens, rows, pages, H_q, H_kv = CASES[case]
    w = to_device(W.make_custom(lens, H_q, H_kv, 128 if case != "g2" else 64, seed=160, poison=True, q_scale=3.0,
                                shared_rows=rows, shared_pages=pages))
    got, dp = run_prefix(w, C)
    ref = oracle_full(w, threads=CORES)
    assert_close(got, ref, f"{case} C={C} plan {dp.plan}")
    assert rel_l2(got, ref) < 1e-2
    if case != "g16":  # 16 heads per row: every unit has one member
        assert dp.plan.num_splits < dp.n_items  # some units stage pages for several rows


@pytest.mark.parametrize("flags", [1, 4, 2])
def test_prefix_plan_merge_paths_and_rings(flags):
    """Separate merge kernel, the deep ring, no programmatic dependent launch."""
    lens, rows, pages, H_q, H_kv = CASES["g8"]
    w = to_device(W.make_custom(lens, H_q, H_kv, 128, seed=161, poison=True, shared_rows=rows, shared_pages=pages))
    got, dp = run_prefix(w, 5, flags)
    assert_close(got, oracle_full(w, threads=CORES), f"flags {flags} plan {dp.plan}")


def test_prefix_plan_is_deterministic_and_reads_less():
    lens, rows, pages, H_q, H_kv = CASES["g4"]
    w = to_device(W.make_custom(lens, H_q, H_kv, 128, seed=162, poison=True, shared_rows=rows, shared_pages=pages))
    a, dp = run_prefix(w, 4)
    b, _ = run_prefix(w, 4)
    assert np.array_equal(a, b)
    plain = bd.plan_counters(w.seq_lens, dp.shape, bd.select_policy(w.seq_lens, dp.shape,
                                                                     [bd.Rule(*ANY, 2, 1, 4, 0)]))
    assert dp.counters["kv_bytes_streamed"] < plain["kv_bytes_streamed"]
    assert dp.counters["work_items"] < plain["work_items"]


def test_full_prefix_workload_with_shared_prefix_plan_every_output():
    """B=64, G=8, rows 0-15 share 128 pages: units of two sharers stream the
    prefix once for both; all 64 x 64 x 128 outputs, poisoned pools."""
    w = W.make("prefix", device="cuda", poison=True)
    shape = bd.shape_of(w.q, w.k_pool, w.block_table)
    base = bd.select_policy(w.seq_lens, shape)
    dp = bd.plan_decode(w.seq_lens, shape, "cuda", plan=base, shared_prefix_table=w.block_table.cpu())
    lens = torch.tensor(w.seq_lens, dtype=torch.int32, device="cuda")
    out = bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table, lens, w.P, w.scale, plan=dp)
    torch.cuda.synchronize()
    assert bd.workspace_status(dp) == 0
    got = out.float().cpu().double().numpy()
    ref = oracle_full(w, threads=CORES)
    assert_close(got, ref, f"prefix plan {dp.plan}")
    assert rel_l2(got, ref) < 1e-2
    # 16 sharers x 8 heads of shared chunks ride in units of 2
    assert dp.n_items - dp.plan.num_splits == 8 * 8 * -(-128 // dp.plan.chunk_pages)
