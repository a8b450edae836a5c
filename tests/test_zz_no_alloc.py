"""pkv_paged_decode_noalloc against pkv_paged_decode, through the C ABI.

The no-alloc entry point serves callers that cannot allocate device memory
where they decode (a plugin in a framework that owns all allocations, a
fixed memory budget, a loop that cannot take an allocation's device
synchronization): it takes no workspace and uses a fixed scratch array inside
the library instead.  Its results must match the workspace entry point's
within the tests' tolerance, call after call, even when consecutive calls use
different plans and so leave different contents in the shared scratch.

This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from paged_kv_gqa_17_b200 import binding as bd
from paged_kv_gqa_17_b200 import workloads as W

from .gpu_util import ATOL, RTOL, to_device

pytestmark = pytest.mark.gpu

ANY = (0, 2**31 - 1, 0, 2**31 - 1)
RULES = [
    bd.Rule(*ANY, 1, 37, 0, 4),   # split-S, fused merge, deep ring
    bd.Rule(*ANY, 2, 1, 3, 0),    # work queue, fused merge
    bd.Rule(*ANY, 2, 1, 5, 1),    # work queue, separate merge kernel
    bd.Rule(*ANY, 0, 1, 0, 0),    # no split
    bd.Rule(*ANY, 1, 9, 0, 0),    # split-S again, other slot layout
    bd.Rule(*ANY, 3, 24, 0, 0),   # balanced grid: several items per block, deferred merges
    bd.Rule(*ANY, 1, 8, 0, 8),    # split-S as clusters merging over distributed shared memory
    bd.Rule(*ANY, 3, 37, 0, 4),   # balanced grid, deep ring
    bd.Rule(*ANY, 2, 37, 0, 36),  # self-planned queue: the blocks derive their items from the lengths
    bd.Rule(*ANY, 1, 16, 0, 20),  # split-S with the early start (the kernel before writes only outputs)
]


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_gqa_17_b200 import build

    build.build()
    return bd.lib()


def _noalloc(L, w, dp, lens_dev):
    out = torch.full_like(w.q, float("nan"))
    rc = L.pkv_paged_decode_noalloc(
        w.q.data_ptr(), w.k_pool.data_ptr(), w.v_pool.data_ptr(), w.block_table.data_ptr(), lens_dev.data_ptr(),
        w.P, ctypes.c_float(w.scale), out.data_ptr(), ctypes.byref(dp.shape), ctypes.byref(dp.plan),
        dp.items.data_ptr() if dp.items is not None else None,
        dp.indptr.data_ptr() if dp.indptr is not None else None, dp.n_items,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, rc
    return out


def _close(a: torch.Tensor, b: torch.Tensor, what: str):
    x = a.float().cpu().double().numpy()
    y = b.float().cpu().double().numpy()
    assert np.isfinite(x).all(), what
    assert (np.abs(x - y) <= ATOL + RTOL * np.abs(y)).all(), f"{what}: max diff {np.abs(x - y).max():.3e}"


@pytest.mark.parametrize("lens,H_q,H_kv,D", [([3000, 17, 1024, 0, 513], 32, 8, 128), ([700, 64], 8, 2, 64)])
def test_noalloc_matches_workspace_entry_point(L, lens, H_q, H_kv, D):
    w = to_device(W.make_custom(lens, H_q, H_kv, D, seed=301, poison=True))
    lens_dev = torch.tensor(w.seq_lens, dtype=torch.int32, device="cuda")
    shape = bd.shape_of(w.q, w.k_pool, w.block_table)
    for rule in RULES:
        dp = bd.plan_decode(w.seq_lens, shape, "cuda", rules=[rule])
        ref = bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table, lens_dev, w.P, w.scale, plan=dp)
        torch.cuda.synchronize()
        assert bd.workspace_status(dp) == 0
        first = _noalloc(L, w, dp, lens_dev)
        second = _noalloc(L, w, dp, lens_dev)  # the scratch now holds the first call's states
        torch.cuda.synchronize()
        assert bd.noalloc_status() == 0, f"device error after the no-alloc calls, plan {dp.plan}"
        _close(first, ref, f"first call, plan {dp.plan}")
        _close(second, ref, f"second call, plan {dp.plan}")


def test_noalloc_prefix_sharing_plan(L):
    """The prefix-sharing grid through the no-alloc entry point: rows that
    share leading pages, the same outputs as the workspace entry point."""
    w = to_device(W.make_custom([1200, 1100, 900, 40, 2000], 32, 8, 128, seed=303, poison=True, shared_rows=3,
                                shared_pages=32))
    lens_dev = torch.tensor(w.seq_lens, dtype=torch.int32, device="cuda")
    shape = bd.shape_of(w.q, w.k_pool, w.block_table)
    dp = bd.plan_decode(w.seq_lens, shape, "cuda", rules=[bd.Rule(*ANY, 2, 1, 16, 4)],
                        shared_prefix_table=w.block_table.cpu())
    assert dp.plan.flags & bd.FLAG_SHARED_PREFIX and dp.n_items > dp.plan.num_splits  # some units share
    ref = bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table, lens_dev, w.P, w.scale, plan=dp)
    torch.cuda.synchronize()
    assert bd.workspace_status(dp) == 0
    for call in ("first", "second"):
        got = _noalloc(L, w, dp, lens_dev)
        torch.cuda.synchronize()
        assert bd.noalloc_status() == 0
        _close(got, ref, f"{call} call, prefix-sharing plan")


def test_noalloc_rejects_plans_larger_than_its_scratch(L):
    # B=64 rows, G=8, D=128 and 5000 work items need 5000*8*(128+2)*4 bytes of
    # partial states, more than the 16 MiB array: rejected before any launch.
    shape = bd.make_shape(64, 64, 8, 128, 16, 8192, 100000)
    plan = bd.Plan(2, 600, 8, 0)
    assert bd.workspace_bytes(shape, plan, 5000) > (16 << 20)
    rc = L.pkv_paged_decode_noalloc(None, None, None, None, None, 16, ctypes.c_float(1.0), None,
                                    ctypes.byref(shape), ctypes.byref(plan), None, None, 5000, None)
    assert rc == -3


def test_noalloc_rejected_call_queues_nothing(L):
    """A call the argument checks reject leaves the scratch as it was: the
    error word a flagged call left stays readable."""
    w = to_device(W.make_custom([100, 200], 8, 2, 64, seed=302))
    shape = bd.shape_of(w.q, w.k_pool, w.block_table)
    dp = bd.plan_decode(w.seq_lens, shape, "cuda", rules=[bd.Rule(*ANY, 0, 1, 0, 0)])
    lens_bad = torch.tensor([100, shape.max_pages_per_seq * 16 + 5], dtype=torch.int32, device="cuda")
    _noalloc(L, w, dp, lens_bad)  # the kernel clamps the length and flags it
    assert bd.noalloc_status() & 2
    bad_plan = bd.Plan(1, 0, 0, 0)  # SPLIT_S with no splits: rejected before anything is queued
    rc = L.pkv_paged_decode_noalloc(
        w.q.data_ptr(), w.k_pool.data_ptr(), w.v_pool.data_ptr(), w.block_table.data_ptr(), lens_bad.data_ptr(),
        w.P, ctypes.c_float(w.scale), w.q.data_ptr(), ctypes.byref(dp.shape), ctypes.byref(bad_plan), None, None, 0,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == -1
    assert bd.noalloc_status() & 2, "a rejected call cleared the scratch"
    lens = torch.tensor(w.seq_lens, dtype=torch.int32, device="cuda")
    _noalloc(L, w, dp, lens)
    assert bd.noalloc_status() == 0
