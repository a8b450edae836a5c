"""pkv_decode_host (host buffers in, host buffer out, one packed copy each
way) against the oracle and against pkv_paged_decode with the same plan.

Both paths run the same kernels on the same plan, so their outputs must be
bit-identical; the oracle comparison uses the tolerance of the other parity
tests.  Covers every plan family the policy can pick (the balanced one
included), inputs that travel inside the packed copies and inputs too large
for them (q, block table, out above 64 KiB), and buffer reuse after a call
that the kernels reported a device-input error on."""
import dataclasses

import numpy as np
import pytest
import torch

from paged_kv_gqa_17_b200 import binding as bd
from paged_kv_gqa_17_b200 import workloads as W

from .gpu_util import assert_close, oracle_full, oracle_sampled, run, to_device

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


def host_inputs(w):
    q_h = w.q.cpu().pin_memory()
    bt_h = w.block_table.cpu().pin_memory()
    lens_h = torch.tensor(w.seq_lens, dtype=torch.int32).pin_memory()
    out_h = torch.full_like(q_h, float("nan")).pin_memory()
    return q_h, bt_h, lens_h, out_h


def host_decode(w, rules=None, dec=None):
    q_h, bt_h, lens_h, out_h = host_inputs(w)
    shape = bd.shape_of(w.q, w.k_pool, w.block_table, w.layout)
    dec = dec or bd.HostDecoder(w.q.device)
    dec.ensure(lens_h, shape, rules)
    plan = dec(q_h, bt_h, lens_h, out_h, w.k_pool, w.v_pool, w.scale, shape, rules=rules)
    return out_h.float().double().numpy(), plan


PLANS = {
    "nosplit": rule(0),
    "split7": rule(1, 7),
    "split32_deep_sep": rule(1, 32, 0, 5),
    "wq3": rule(2, 1, 3),
    "wq16_sep": rule(2, 1, 16, 1),
    "bal37": rule(3, 37),
    "bal296": rule(3, 296),
    "split16_cl": rule(1, 16, 0, 8),
    "wqfill37_dev": rule(2, 37, 0, 4 | 32),  # blocks derive their items from the uploaded lengths
}


@pytest.mark.parametrize("name", sorted(PLANS))
def test_host_path_matches_oracle_and_device_path(name):
    w = to_device(W.make_custom([1000, 4097, 2500, 17, 0], 32, 8, 128, seed=130, poison=True))
    got, plan = host_decode(w, rules=[PLANS[name]])
    assert plan.tuple()[0] == PLANS[name].mode
    assert_close(got, oracle_full(w), f"host/{name}")
    dev, dp = run(w, mode_rule=PLANS[name])
    assert dp.plan.tuple() == plan.tuple()
    assert np.array_equal(got, dev), name


@pytest.mark.parametrize("rules", [[rule(3, 296)], [rule(2, 296, 0, 4)], None])
def test_host_path_builds_the_queues_itself(rules):
    """B=8, N_max = 20000: the balanced grid, the queue whose chunk fills one
    wave (chunk_pages = 0) and the built-in table's plan, each built and
    uploaded by the host path itself."""
    lens = [20000, 300, 9000, 17000, 64, 5000, 12345, 1]
    w = to_device(W.make_custom(lens, 32, 8, 128, seed=131, poison=True))
    got, plan = host_decode(w, rules=rules)
    if rules is not None:
        assert plan.mode == rules[0].mode, plan.tuple()
    dev, dp = run(w, rules=rules)
    assert dp.plan.tuple() == plan.tuple()
    assert np.array_equal(got, dev)
    pairs = [(0, 0), (0, 31), (3, 17), (7, 5), (4, 9), (6, 30)]
    assert_close(np.stack([got[r, h] for r, h in pairs]), oracle_sampled(w, pairs), f"host/{plan.tuple()}")


@pytest.mark.parametrize("rules", [None, [rule(2, 1, 8)]])
def test_host_path_large_inputs_use_their_own_copies(rules):
    """B=64, H_q=64: q and out are 1 MiB and the block table 64 x 350 x 4 B,
    all above the 64 KiB that travel inside the packed copies."""
    rng = np.random.default_rng(11)
    lens = [int(x) for x in rng.integers(1, 5600, 64)]
    lens[5] = 350 * 16
    w = W.make_custom(lens, 64, 8, 128, seed=132, poison=True, device="cuda")
    assert w.q.numel() * 2 > 64 * 1024 and w.block_table.numel() * 4 > 64 * 1024
    got, plan = host_decode(w, rules=rules)
    dev, dp = run(w, rules=rules)
    assert dp.plan.tuple() == plan.tuple()
    assert np.array_equal(got, dev)
    pairs = [(0, 0), (5, 63), (63, 1), (31, 40)]
    assert_close(np.stack([got[r, h] for r, h in pairs]), oracle_sampled(w, pairs), "host/large")


def test_host_path_reuses_buffers_after_a_device_input_error():
    """The upload zeroes the error word and counters every call: a call that
    the kernels flagged (page id out of range) leaves nothing behind for the
    next call on the same buffers."""
    w = to_device(W.make_custom([700, 1500, 33], 16, 4, 128, seed=133, poison=True))
    ref = oracle_full(w)
    dec = bd.HostDecoder("cuda")
    for r in ([rule(1, 7)], [rule(2, 1, 3)], [rule(3, 11)]):
        got, _ = host_decode(w, rules=r, dec=dec)
        assert_close(got, ref, f"host/{r[0].mode} first")
        q_h, bt_h, lens_h, out_h = host_inputs(w)
        bt_h[1, 2] = w.num_pages + 9
        shape = bd.shape_of(w.q, w.k_pool, w.block_table)
        with pytest.raises(bd.PkvError) as e:
            dec(q_h, bt_h, lens_h, out_h, w.k_pool, w.v_pool, w.scale, shape, rules=r)
        assert e.value.status == -6  # PKV_ERR_DEVICE_INPUT
        got, _ = host_decode(w, rules=r, dec=dec)
        assert_close(got, ref, f"host/{r[0].mode} after error")


def test_host_path_empty_rows():
    w = to_device(W.make_custom([0, 0], 8, 2, 64, seed=134, poison=True))
    got, _ = host_decode(w)
    assert (got == 0).all()


@pytest.mark.parametrize("name", ["split7", "wq16_sep", "bal37"])
def test_pageable_out_takes_the_copy_and_matches_the_direct_path(name):
    """Page-locked out: the kernels write the result straight into it; a
    pageable out takes the packed device->host copy.  Same kernels, same
    bits; a device-input error is reported on both paths."""
    w = to_device(W.make_custom([1000, 4097, 2500, 17, 0], 32, 8, 128, seed=135, poison=True))
    shape = bd.shape_of(w.q, w.k_pool, w.block_table)
    q_h, bt_h, lens_h, out_pinned = host_inputs(w)
    out_pageable = torch.full_like(out_pinned, float("nan"))
    assert not out_pageable.is_pinned()
    dec = bd.HostDecoder("cuda")
    dec.ensure(lens_h, shape, [PLANS[name]])
    dec(q_h, bt_h, lens_h, out_pinned, w.k_pool, w.v_pool, w.scale, shape, rules=[PLANS[name]])
    dec(q_h, bt_h, lens_h, out_pageable, w.k_pool, w.v_pool, w.scale, shape, rules=[PLANS[name]])
    assert torch.equal(out_pinned, out_pageable)
    assert_close(out_pageable.float().double().numpy(), oracle_full(w), f"pageable/{name}")
    bad = bt_h.clone()
    bad[1, 3] = w.num_pages + 2
    for out in (out_pinned, out_pageable):
        with pytest.raises(bd.PkvError) as e:
            dec(q_h, bad, lens_h, out, w.k_pool, w.v_pool, w.scale, shape, rules=[PLANS[name]])
        assert e.value.status == -6


def test_repeated_call_takes_the_parameter_block_and_sees_new_contents():
    """A HostDecoder call with the same (checked) tensors as the last one goes
    through pkv_decode_host_call with the stored parameter block; new
    contents of those tensors (q, lengths, table) are what it decodes."""
    w = to_device(W.make_custom([3000, 517, 0, 1200], 32, 8, 128, seed=131, poison=False))
    q_h, bt_h, lens_h, out_h = host_inputs(w)
    shape = bd.shape_of(w.q, w.k_pool, w.block_table, w.layout)
    dec = bd.HostDecoder(w.q.device)
    dec.ensure(lens_h, shape)
    dec(q_h, bt_h, lens_h, out_h, w.k_pool, w.v_pool, w.scale, shape)
    assert_close(out_h.float().double().numpy(), oracle_full(w), "first call")
    assert dec._args is not None
    calls = []
    real = dec._fn_call
    dec._fn_call = lambda ref: calls.append(1) or real(ref)
    g = torch.Generator().manual_seed(7)
    # lengths within each row's pages; step 1 swaps the tables of rows 0 and 3
    for step, lens in enumerate(([2999, 528, 0, 1], [1200, 1, 0, 3008], [3000, 517, 0, 1200])):
        new_q = torch.randn(w.q.shape, generator=g).to(torch.bfloat16)
        q_h.copy_(new_q)
        lens_h.copy_(torch.tensor(lens, dtype=torch.int32))
        if step in (1, 2):
            bt_h[[0, 3]] = bt_h[[3, 0]].clone()
        dec.ensure(lens_h, shape)  # a serving loop's per-step sizing keeps the stored block
        dec(q_h, bt_h, lens_h, out_h, w.k_pool, w.v_pool, w.scale, shape)
        w2 = dataclasses.replace(w, q=new_q.to(w.q.device), seq_lens=list(lens),
                                 block_table=bt_h.to(w.q.device))
        assert_close(out_h.float().double().numpy(), oracle_full(w2), f"step {step}")
    assert len(calls) == 3
    tm = bd.HostTiming()  # the timed step goes through the same block
    dec(q_h, bt_h, lens_h, out_h, w.k_pool, w.v_pool, w.scale, shape, timing=tm)
    assert len(calls) == 4 and tm.dev_kernel_us > 0 and tm.host_wait_us > 0
    assert_close(out_h.float().double().numpy(), oracle_full(w2), "timed step")


@pytest.mark.parametrize("name", sorted(PLANS))
def test_repeated_steps_replay_a_captured_graph(name):
    """The second call in a row with the same buffers and plan captures the
    step as a CUDA graph and later calls replay it: every replayed step
    decodes its own new q and matches the oracle, a call with other lengths
    (another queue) runs without the graph, and a device-input error found
    during a replay is reported like any other."""
    w = to_device(W.make_custom([1000, 4097, 2500, 17, 0], 32, 8, 128, seed=132, poison=True))
    q_h, bt_h, lens_h, out_h = host_inputs(w)
    shape = bd.shape_of(w.q, w.k_pool, w.block_table, w.layout)
    rules = [PLANS[name]]
    dec = bd.HostDecoder(w.q.device)
    dec.ensure(lens_h, shape, rules)
    g = torch.Generator().manual_seed(11)
    before = bd.host_replays()
    for step in range(4):
        new_q = torch.randn(w.q.shape, generator=g).to(torch.bfloat16)
        q_h.copy_(new_q)
        out_h.fill_(float("nan"))
        dec(q_h, bt_h, lens_h, out_h, w.k_pool, w.v_pool, w.scale, shape, rules=rules)
        w2 = dataclasses.replace(w, q=new_q.to(w.q.device))
        assert_close(out_h.float().double().numpy(), oracle_full(w2), f"{name} step {step}")
    assert bd.host_replays() - before == 3  # the first call runs directly, the next three replay
    lens2 = [999, 4097, 2496, 16, 0]  # shorter only: the slots past each length are poisoned
    lens_h.copy_(torch.tensor(lens2, dtype=torch.int32))
    dec.ensure(lens_h, shape, rules)
    dec(q_h, bt_h, lens_h, out_h, w.k_pool, w.v_pool, w.scale, shape, rules=rules)
    w3 = dataclasses.replace(w2, seq_lens=lens2)
    assert_close(out_h.float().double().numpy(), oracle_full(w3), f"{name} other lengths")
    lens_h.copy_(torch.tensor(w.seq_lens, dtype=torch.int32))
    for _ in range(2):
        dec(q_h, bt_h, lens_h, out_h, w.k_pool, w.v_pool, w.scale, shape, rules=rules)
    assert_close(out_h.float().double().numpy(), oracle_full(w2), f"{name} back")
    bad = bt_h.clone()
    bad[1, 3] = w.num_pages + 2
    n = bd.host_replays()
    with pytest.raises(bd.PkvError) as e:
        dec(q_h, bad, lens_h, out_h, w.k_pool, w.v_pool, w.scale, shape, rules=rules)
    assert e.value.status == -6 and bd.host_replays() == n + 1  # reported from a replayed step
    dec(q_h, bt_h, lens_h, out_h, w.k_pool, w.v_pool, w.scale, shape, rules=rules)
    assert_close(out_h.float().double().numpy(), oracle_full(w2), f"{name} after the error")


def test_two_threads_each_replay_their_own_step():
    """Two host threads, each with its own HostDecoder and stream, call the
    host path concurrently (the binding releases the interpreter lock during
    the call): each thread keeps its own captured graph and every output
    matches the oracle for that thread's q."""
    import threading

    w = to_device(W.make_custom([2500, 700, 33], 32, 8, 128, seed=133, poison=True))
    shape = bd.shape_of(w.q, w.k_pool, w.block_table, w.layout)
    results, errors = {}, []

    def worker(tag, seed):
        try:
            st = torch.cuda.Stream()
            q_h, bt_h, lens_h, out_h = host_inputs(w)
            dec = bd.HostDecoder(w.q.device, stream=st)
            dec.ensure(lens_h, shape)
            g = torch.Generator().manual_seed(seed)
            before = bd.host_replays()
            outs = []
            for _ in range(6):
                q = torch.randn(w.q.shape, generator=g).to(torch.bfloat16)
                q_h.copy_(q)
                dec(q_h, bt_h, lens_h, out_h, w.k_pool, w.v_pool, w.scale, shape)
                outs.append((q, out_h.clone()))
            results[tag] = (outs, bd.host_replays() - before)
        except Exception as e:  # reported below
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(t, 50 + t)) for t in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    for tag, (outs, replays) in results.items():
        assert replays == 5, (tag, replays)  # per thread: one direct call, then replays
        for q, out in outs[::2]:
            w2 = dataclasses.replace(w, q=q.to(w.q.device))
            assert_close(out.float().double().numpy(), oracle_full(w2), f"thread {tag}")
