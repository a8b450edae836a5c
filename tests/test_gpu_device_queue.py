"""The queues built on the GPU (pkv_build_balanced_queue_device,
pkv_build_fill_queue_device): bit-identical to the host builders, decodes
that match the oracle, and decode steps captured once in a CUDA graph that
stay correct while the lengths change on the device between replays."""
import numpy as np
import pytest
import torch

from paged_kv_gqa_17_b200 import binding as bd
from paged_kv_gqa_17_b200 import workloads as W

from .gpu_util import assert_close, oracle_full, to_device

pytestmark = pytest.mark.gpu

ANY = (0, 2**31 - 1, 0, 2**31 - 1)


def rule(mode, S=1, C=0, flags=0):
    return bd.Rule(*ANY, mode, S, C, flags)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_gqa_17_b200 import build

    build.build()
    bd.lib()


def _device_queue(lens, shape, T):
    cap = bd.balanced_queue_capacity(shape, T)
    items = torch.full((cap, 4), -7, dtype=torch.int32, device="cuda")
    indptr = torch.full((shape.B * shape.H_kv + 1 + T + 1,), -7, dtype=torch.int32, device="cuda")
    ws = torch.zeros(bd.workspace_bytes(shape, bd.Plan(3, T, 0, 0), cap), dtype=torch.uint8, device="cuda")
    lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
    bd.build_balanced_queue_device(lens_d, shape, T, items, indptr, ws)
    torch.cuda.synchronize()
    return items.cpu(), indptr.cpu(), ws


def test_device_builder_matches_host_builder_bit_exactly():
    rng = np.random.default_rng(21)
    cases = [([0, 0, 0], 2, 5), ([1], 1, 296), ([17, 0, 5], 4, 296), ([16] * 5, 8, 7), ([32768], 8, 296),
             ([12129, 621, 1118, 1452, 2891, 1419, 518, 3174], 8, 296), ([5000, 0, 1, 16, 17], 2, 1)]
    for _ in range(40):
        B = int(rng.integers(1, 70))
        lens = [int(x) for x in rng.choice([0, 1, 15, 16, 17, 300, 5000, 40000], B)]
        cases.append((lens, int(rng.choice([1, 2, 4, 8])), int(rng.choice([1, 3, 37, 148, 296, 1000]))))
    for lens, H_kv, T in cases:
        max_pages = max([-(-n // 16) for n in lens] + [1])
        shape = bd.make_shape(len(lens), 4 * H_kv, H_kv, 128, 16, max_pages, 10)
        h_items, h_indptr = bd.build_balanced_queue(lens, shape, T)
        d_items, d_indptr, ws = _device_queue(lens, shape, T)
        n = h_items.shape[0]
        assert n <= d_items.shape[0]
        assert torch.equal(d_items[:n], h_items), (lens, H_kv, T)
        assert torch.equal(d_indptr, h_indptr), (lens, H_kv, T)
        assert (d_items[n:] == -7).all()  # entries past the real count untouched
        assert int(ws[:4].view(torch.int32)[0]) == 0


@pytest.mark.parametrize("T", [1, 7, 37, 296])
def test_decode_with_device_queue_matches_oracle(T):
    w = to_device(W.make_custom([3000, 77, 1999, 16, 0, 1], 32, 8, 128, seed=140, poison=True))
    shape = bd.shape_of(w.q, w.k_pool, w.block_table)
    dp = bd.plan_decode(w.seq_lens, shape, "cuda", plan=bd.Plan(3, T, 0, 0), device_queue=True)
    lens = torch.tensor(w.seq_lens, dtype=torch.int32, device="cuda")
    out = bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table, lens, 16, w.scale, plan=dp)
    torch.cuda.synchronize()
    assert bd.workspace_status(dp) == 0
    got = out.float().cpu().double().numpy()
    assert_close(got, oracle_full(w), f"device queue T={T}")
    host = bd.plan_decode(w.seq_lens, shape, "cuda", plan=bd.Plan(3, T, 0, 0))
    ref = bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table, lens, 16, w.scale, plan=host)
    assert torch.equal(out, ref)  # same queue, same kernels: the same bits


def test_graph_replay_follows_lengths_changed_on_the_device():
    """One decode step captured in a CUDA graph (queue build + balanced
    kernel); between replays only the device lengths change (rows grow,
    shrink, empty), and every replay matches the oracle for its lengths."""
    full = [2500, 900, 40, 1300]
    w = to_device(W.make_custom(full, 16, 4, 128, seed=141, poison=False))
    shape = bd.shape_of(w.q, w.k_pool, w.block_table)
    dp = bd.plan_decode(full, shape, "cuda", plan=bd.Plan(3, 37, 0, 0), device_queue=True)
    lens = torch.tensor(full, dtype=torch.int32, device="cuda")
    out = torch.empty_like(w.q)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table, lens, 16, w.scale, plan=dp, out=out)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table, lens, 16, w.scale, plan=dp, out=out)
    cap = shape.max_pages_per_seq * 16  # 157 pages: lengths up to 2512 fit the tables
    for step_lens in ([2500, 900, 40, 1300], [2501, 901, 41, 1301], [17, 0, 40, cap], [0, 0, 0, 0], [1, 2, 3, 4],
                      [2000, 2000, 2000, 2000]):
        lens.copy_(torch.tensor(step_lens, dtype=torch.int32))
        g.replay()
        torch.cuda.synchronize()
        assert bd.workspace_status(dp) == 0
        w.seq_lens = list(step_lens)
        assert_close(out.float().cpu().double().numpy(), oracle_full(w), f"replay {step_lens}")
    del g


def test_device_builder_flags_bad_lengths():
    shape = bd.make_shape(3, 8, 2, 128, 16, 4, 10)
    lens = torch.tensor([10, 4 * 16 + 1, -3], dtype=torch.int32, device="cuda")
    cap = bd.balanced_queue_capacity(shape, 5)
    items = torch.zeros((cap, 4), dtype=torch.int32, device="cuda")
    indptr = torch.zeros(3 * 2 + 1 + 5 + 1, dtype=torch.int32, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    bd.build_balanced_queue_device(lens, shape, 5, items, indptr, ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32)[0]) & 2
    # the clamped lengths (10, 64, 0) give the host builder's queue
    h_items, h_indptr = bd.build_balanced_queue([10, 64, 0], shape, 5)
    assert torch.equal(items.cpu()[:h_items.shape[0]], h_items) and torch.equal(indptr.cpu(), h_indptr)


def _fill_queue(lens, shape, T):
    cap = bd.fill_queue_capacity(shape, T)
    items = torch.full((cap, 4), -7, dtype=torch.int32, device="cuda")
    indptr = torch.full((shape.B * shape.H_kv + 1,), -7, dtype=torch.int32, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
    bd.build_fill_queue_device(lens_d, shape, T, items, indptr, ws)
    torch.cuda.synchronize()
    return items.cpu(), indptr.cpu(), ws


def test_fill_builder_matches_policy_and_host_queue_bit_exactly():
    """The device's chunk is the host policy's fill chunk, and its queue is
    pkv_build_work_queue's at that chunk."""
    rng = np.random.default_rng(22)
    cases = [([1], 1, 296), ([17, 0, 5], 4, 296), ([32768], 8, 296), ([16] * 5, 8, 7), ([5000, 0, 1, 16, 17], 2, 1),
             ([12129, 621, 1118, 1452, 2891, 1419, 518, 3174], 8, 296), ([40000] * 64, 8, 296)]
    for _ in range(40):
        B = int(rng.integers(1, 70))
        lens = [int(x) for x in rng.choice([0, 1, 15, 16, 17, 300, 5000, 40000], B)]
        if max(lens) == 0:
            lens[0] = 1
        cases.append((lens, int(rng.choice([1, 2, 4, 8])), int(rng.choice([1, 3, 37, 148, 296, 444]))))
    for lens, H_kv, T in cases:
        max_pages = max(-(-n // 16) for n in lens)
        shape = bd.make_shape(len(lens), 4 * H_kv, H_kv, 128, 16, max_pages, 10)
        plan = bd.select_policy(lens, shape, [rule(2, T, 0, 0)])
        h_items, h_indptr = bd.build_work_queue(lens, shape, plan.chunk_pages)
        d_items, d_indptr, ws = _fill_queue(lens, shape, T)
        n = h_items.shape[0]
        assert torch.equal(d_items[:n], h_items), (lens, H_kv, T, plan.tuple())
        assert torch.equal(d_indptr, h_indptr), (lens, H_kv, T)
        assert (d_items[n:] == -7).all()
        assert int(ws[:4].view(torch.int32)[0]) == 0


@pytest.mark.parametrize("T,flags,fused", [(37, 0, False), (296, 4, False), (5, 1, False), (37, 0, True),
                                           (296, 4, True), (5, 0, True)])
def test_decode_with_device_fill_queue_matches_oracle(T, flags, fused):
    """The fill queue from the builder kernel, or derived by every decode
    block itself (PKV_FLAG_DEVICE_FILL): the oracle's answer, and the same
    bits as the host-built queue at the policy's chunk."""
    w = to_device(W.make_custom([3000, 77, 1999, 16, 0, 1], 32, 8, 128, seed=142, poison=True))
    shape = bd.shape_of(w.q, w.k_pool, w.block_table)
    plan = bd.select_policy(w.seq_lens, shape, [rule(2, T, 0, flags)])
    dp = bd.plan_decode(w.seq_lens, shape, "cuda", plan=plan, device_queue=True, fill_blocks=T, device_fill=fused)
    assert bool(dp.plan.flags & bd.FLAG_DEVICE_FILL) == fused and (dp.items is None) == fused
    lens = torch.tensor(w.seq_lens, dtype=torch.int32, device="cuda")
    out = bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table, lens, 16, w.scale, plan=dp)
    torch.cuda.synchronize()
    assert bd.workspace_status(dp) == 0
    assert_close(out.float().cpu().double().numpy(), oracle_full(w), f"device fill queue T={T}")
    host = bd.plan_decode(w.seq_lens, shape, "cuda", plan=plan)
    ref = bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table, lens, 16, w.scale, plan=host)
    assert torch.equal(out, ref)  # same queue, same kernels: the same bits


@pytest.mark.parametrize("fused", [False, True])
def test_graph_replay_of_the_fill_queue_follows_device_lengths(fused):
    full = [2500, 900, 40, 1300]
    w = to_device(W.make_custom(full, 16, 4, 128, seed=143, poison=False))
    shape = bd.shape_of(w.q, w.k_pool, w.block_table)
    plan = bd.select_policy(full, shape, [rule(2, 148, 0, 4)])
    dp = bd.plan_decode(full, shape, "cuda", plan=plan, device_queue=True, fill_blocks=148, device_fill=fused)
    lens = torch.tensor(full, dtype=torch.int32, device="cuda")
    out = torch.empty_like(w.q)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table, lens, 16, w.scale, plan=dp, out=out)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table, lens, 16, w.scale, plan=dp, out=out)
    cap = shape.max_pages_per_seq * 16
    for step_lens in ([2500, 900, 40, 1300], [17, 0, 40, cap], [0, 0, 0, 0], [1, 2, 3, 4], [cap] * 4):
        lens.copy_(torch.tensor(step_lens, dtype=torch.int32))
        g.replay()
        torch.cuda.synchronize()
        assert bd.workspace_status(dp) == 0
        w.seq_lens = list(step_lens)
        assert_close(out.float().cpu().double().numpy(), oracle_full(w), f"fill replay {step_lens}")
    del g


def test_device_queue_request_passes_queue_free_plans_through():
    """device_queue=True with a split-S plan needs no queue: the plan reads the
    lengths on the device, so a captured step serves any lengths up to those
    it was planned for."""
    full = [2000, 700, 1500]
    w = to_device(W.make_custom(full, 16, 4, 128, seed=144, poison=False))
    shape = bd.shape_of(w.q, w.k_pool, w.block_table)
    dp = bd.plan_decode(full, shape, "cuda", rules=[rule(1, 8, 0, 4)], device_queue=True)
    assert dp.plan.mode == bd.SPLIT_S and not dp.device_queue and dp.items is None
    lens = torch.tensor(full, dtype=torch.int32, device="cuda")
    out = torch.empty_like(w.q)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table, lens, 16, w.scale, plan=dp, out=out)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table, lens, 16, w.scale, plan=dp, out=out)
    for step_lens in ([2000, 700, 1500], [1999, 0, 2000], [5, 6, 7]):
        lens.copy_(torch.tensor(step_lens, dtype=torch.int32))
        g.replay()
        torch.cuda.synchronize()
        assert bd.workspace_status(dp) == 0
        w.seq_lens = list(step_lens)
        assert_close(out.float().cpu().double().numpy(), oracle_full(w), f"split-S replay {step_lens}")
    del g


def test_device_fill_derives_the_host_queue_bit_for_bit():
    """Random batches (B up to 70, all-empty rows, single-token rows, rows at
    the table's capacity), H_kv 1..8, budgets from 1 to past the item count:
    every block's self-derived item gives the same bits as the host-built
    fill queue, and the error word stays clean."""
    rng = np.random.default_rng(23)
    cases = [([12129, 621, 1118, 1452, 2891, 1419, 518, 3174], 8, 296), ([32768], 8, 296), ([1], 1, 296),
             ([0, 0, 5], 2, 7), ([16] * 5, 8, 7), ([40000] * 33, 2, 296), ([5000, 0, 1, 16, 17], 2, 1)]
    for _ in range(14):
        B = int(rng.integers(1, 71))
        lens = [int(x) for x in rng.choice([0, 1, 15, 16, 17, 300, 5000, 20000], B)]
        cases.append((lens, int(rng.choice([1, 2, 4, 8])), int(rng.choice([1, 3, 37, 148, 296, 444, 5000]))))
    for lens, H_kv, T in cases:
        w = to_device(W.make_custom(lens, 4 * H_kv, H_kv, 64, seed=145 + len(lens), poison=True))
        shape = bd.shape_of(w.q, w.k_pool, w.block_table)
        lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
        fused = bd.plan_decode(lens, shape, "cuda", plan=bd.Plan(2, T, 0, bd.FLAG_DEVICE_FILL))
        host_plan = bd.select_policy(lens, shape, [rule(2, T, 0, 0)])
        host = bd.plan_decode(lens, shape, "cuda", plan=host_plan)
        a = bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table, lens_d, 16, w.scale, plan=fused)
        b = bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table, lens_d, 16, w.scale, plan=host)
        torch.cuda.synchronize()
        assert bd.workspace_status(fused) == 0 and bd.workspace_status(host) == 0, (lens, H_kv, T)
        assert torch.equal(a, b), (lens, H_kv, T, host_plan.tuple())
        if host_plan.mode == bd.WORK_QUEUE:
            assert fused.counters["work_items"] == host.counters["work_items"] and fused.counters["queue_bytes"] == 0


def test_device_fill_flags_bad_lengths_and_clamps():
    """A length past the table's capacity is clamped and reported, like the
    other paths; the output equals the host queue's for the clamped lengths."""
    w = to_device(W.make_custom([100, 64, 40], 8, 2, 64, seed=146))
    shape = bd.shape_of(w.q, w.k_pool, w.block_table)
    cap = shape.max_pages_per_seq * 16
    dp = bd.plan_decode(w.seq_lens, shape, "cuda", plan=bd.Plan(2, 37, 0, bd.FLAG_DEVICE_FILL))
    bad = torch.tensor([100, cap + 9, -4], dtype=torch.int32, device="cuda")
    out = bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table, bad, 16, w.scale, plan=dp)
    assert bd.workspace_status(dp) & 2
    clamped = [100, cap, 0]
    host = bd.plan_decode(clamped, shape, "cuda", plan=bd.select_policy(clamped, shape, [rule(2, 37, 0, 0)]))
    ref = bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table,
                          torch.tensor(clamped, dtype=torch.int32, device="cuda"), 16, w.scale, plan=host)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


def test_stale_guess_is_drained_and_skipped():
    """Decode blocks start while the builder kernel before them still writes
    the queue (programmatic dependent launch), so a block's guess of its item
    comes from the previous step's queue.  The lengths alternate between two
    sets with different queues: most guesses are wrong, and the pages copied
    ahead from them must be drained and skipped.  Every step against the
    oracle for its own lengths."""
    sets = ([2500, 900, 40, 1300], [700, 2300, 1500, 33])
    w = to_device(W.make_custom([max(a, b) for a, b in zip(*sets)], 16, 4, 128, seed=147, poison=False))
    shape = bd.shape_of(w.q, w.k_pool, w.block_table)
    plan = bd.select_policy(sets[0], shape, [rule(2, 148, 0, 4)])
    dp = bd.plan_decode(sets[0], shape, "cuda", plan=plan, device_queue=True, fill_blocks=148, device_fill=False)
    lens = torch.tensor(sets[0], dtype=torch.int32, device="cuda")
    dev_sets = [torch.tensor(x, dtype=torch.int32, device="cuda") for x in sets]
    outs = []
    for i in range(8):
        lens.copy_(dev_sets[i % 2])
        outs.append(bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table, lens, 16, w.scale, plan=dp))
    torch.cuda.synchronize()
    assert bd.workspace_status(dp) == 0
    refs = []
    for x in sets:
        w.seq_lens = list(x)
        refs.append(oracle_full(w))
    for i, out in enumerate(outs):
        assert_close(out.float().cpu().double().numpy(), refs[i % 2], f"step {i}")
