"""Pins for the oracle's host scheduling pieces (work queue, policy, counters).

Each check takes the oracle module `O`, so the same checks run against the
real oracle and against copies with a planted mistake.

  queue_closed_form   n_items = H_kv * sum_i max(1, ceil(ceil(N_i / P) / C))
  queue_cover         per (row, head), items tile [0, N_i) in order, without
                      gaps or overlap, every item non-empty and page aligned
  queue_bruteforce    enumerate-and-filter over a rectangular (i, h, c) grid
  policy_paper        the page's decisions at B = 1 / 4 / 8 (tests/golden/paper_policy.txt)
  policy_semantics    first match wins, ranges are half-open, S' and C closed forms
  policy_fill         a queue rule with chunk_pages = 0 takes the smallest C whose
                      queue (counted by building it) has at most T items
  launch_fanout       16 bucket launches vs 2 queue launches at B = 8
                      (tests/golden/launch_fanout_b8.txt)
  merge_state_closed  queue merge traffic = 2*G*(D+2)*4 * H_kv * (slots of
                      multi-chunk pairs); rectangular = the same over B*H_kv*S slots
  prefix_queue        the queue that stages shared prefix pages once: items tile
                      every row, units partition the items, a unit's members cover
                      the same tokens on the same physical pages, the shared
                      ranges are maximal, and without sharing it is the plain queue
  counters_recount    every counter of every mode, recounted from what the step
                      really moves: the bytes of the queue as built, the pages
                      the row's tokens touch (token by token), the blocks a
                      grid launches; plus two worked examples by hand
"""
from __future__ import annotations

import itertools
import os
import random

HERE = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.join(os.path.dirname(HERE), "paged_kv_gqa_17_b200")


def _cdiv(a, b):
    return -(-a // b)


CASES = [
    ([512], 1, 16, 4),
    ([32768], 8, 16, 64),
    ([0, 1, 15, 16, 17, 255, 256, 257], 2, 16, 1),
    ([0, 1, 15, 16, 17, 255, 256, 257], 3, 16, 5),
    ([4097, 16384, 9000, 5001], 8, 16, 16),
    ([0, 0], 4, 16, 2),
    ([], 8, 16, 8),
]


def _random_cases(seed=7, n=40):
    rng = random.Random(seed)
    for _ in range(n):
        B = rng.randint(1, 9)
        lens = [rng.choice([0, rng.randint(1, 40), rng.randint(1, 5000)]) for _ in range(B)]
        yield lens, rng.randint(1, 8), rng.choice([8, 16, 32]), rng.randint(1, 70)


def queue_closed_form(O):
    for lens, H_kv, P, C in itertools.chain(CASES, _random_cases()):
        items, indptr = O.build_work_queue(lens, H_kv, P, C)
        want = H_kv * sum(max(1, _cdiv(_cdiv(n, P), C)) for n in lens)
        assert len(items) == want, ("queue_closed_form", lens, H_kv, P, C)
        assert len(indptr) == len(lens) * H_kv + 1 and indptr[-1] == len(items)


def queue_cover(O):
    for lens, H_kv, P, C in itertools.chain(CASES, _random_cases(8)):
        items, indptr = O.build_work_queue(lens, H_kv, P, C)
        for i, n in enumerate(lens):
            for h in range(H_kv):
                pair = items[indptr[i * H_kv + h]:indptr[i * H_kv + h + 1]]
                assert all(it[0] == i and it[1] == h for it in pair), "queue_cover: wrong pair"
                if n == 0:
                    assert pair == [(i, h, 0, 0)], "queue_cover: empty row"
                    continue
                pos = 0
                for (_, _, b, e) in pair:
                    assert b == pos and e > b and b % (C * P) == 0, ("queue_cover", lens, i, h, pair)
                    assert e - b <= C * P
                    pos = e
                assert pos == n, ("queue_cover: gap at end", lens, i, h)


def queue_bruteforce(O):
    for lens, H_kv, P, C in itertools.chain(CASES, _random_cases(9)):
        items, indptr = O.build_work_queue(lens, H_kv, P, C)
        n_max = max(lens, default=0)
        grid = []
        for i, h, c in itertools.product(range(len(lens)), range(H_kv), range(max(1, _cdiv(n_max, C * P)))):
            n = lens[i]
            if n == 0 and c == 0:
                grid.append((i, h, 0, 0))
            elif c * C * P < n:
                grid.append((i, h, c * C * P, min(n, (c + 1) * C * P)))
        assert items == grid, ("queue_bruteforce", lens, H_kv, P, C)
        ptr = [0]
        for i, h in itertools.product(range(len(lens)), range(H_kv)):
            ptr.append(ptr[-1] + sum(1 for it in grid if it[0] == i and it[1] == h))
        assert indptr == ptr


def read_golden(name):
    rows = []
    with open(os.path.join(HERE, "golden", name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def policy_paper(O):
    rules = O.load_rules(os.path.join(PKG, "policy_paper_rule.json"))
    names = {"NO_SPLIT": O.NO_SPLIT, "SPLIT_S": O.SPLIT_S, "WORK_QUEUE": O.WORK_QUEUE}
    for B, n_max, mode in read_golden("paper_policy.txt"):
        B, n_max = int(B), int(n_max)
        lens = [n_max] + [max(1, n_max // 3)] * (B - 1)
        plan = O.select_policy(lens, 16, rules)
        assert plan[0] == names[mode], ("policy_paper", B, n_max, plan)


def policy_semantics(O):
    R = O.Rule
    rules = [R(1, 2, 4096, O.INT32_MAX, O.SPLIT_S, num_splits=37),
             R(1, 2, 0, 4096, O.NO_SPLIT, flags=1),
             R(2, 8, 0, O.INT32_MAX, O.WORK_QUEUE, chunk_pages=24, flags=1),
             R(0, O.INT32_MAX, 0, O.INT32_MAX, O.WORK_QUEUE, chunk_pages=8)]
    P = 16
    # B = 1, N_max = 32768: S = 37 -> C = ceil(2048 / 37) = 56, S' = ceil(2048 / 56) = 37
    assert O.select_policy([32768], P, rules) == (O.SPLIT_S, 37, 56, 0)
    # boundary of a half-open range: 4096 belongs to the first rule, 4095 to the second;
    # 256 pages, S = 37 -> C = ceil(256 / 37) = 7, S' = ceil(256 / 7) = 37
    assert O.select_policy([4096], P, rules) == (O.SPLIT_S, 37, 7, 0)
    # 100 pages, S = 37 -> C = 3, S' = ceil(100 / 3) = 34: the tight split count
    assert O.select_policy([1600], P, [R(1, 2, 0, O.INT32_MAX, O.SPLIT_S, num_splits=37)]) == (O.SPLIT_S, 34, 3, 0)
    assert O.select_policy([4095], P, rules) == (O.NO_SPLIT, 1, 0, 1)
    # B = 8 misses [2, 8) and falls to the catch-all
    assert O.select_policy([100] * 8, P, rules) == (O.WORK_QUEUE, 1, 8, 0)
    assert O.select_policy([1000, 5] * 2, P, rules) == (O.WORK_QUEUE, 3, 24, 1)
    # a balanced rule takes its block count as given
    assert O.select_policy([5000, 7], P, [R(0, 9, 0, O.INT32_MAX, 3, num_splits=296, flags=4)]) == (3, 296, 0, 4)
    # a device-fill queue rule leaves the chunk to the device and carries its budget T
    dev_fill = [R(0, 9, 0, O.INT32_MAX, O.WORK_QUEUE, num_splits=296, flags=O.FLAG_DEVICE_FILL | 4)]
    assert O.select_policy([5000, 7], P, dev_fill) == (O.WORK_QUEUE, 296, 0, O.FLAG_DEVICE_FILL | 4)
    # no rule matches -> single kernel; empty batch and all-empty rows -> single kernel
    assert O.select_policy([10], P, rules[:1]) == (O.NO_SPLIT, 1, 0, 0)
    assert O.select_policy([], P, rules) == (O.NO_SPLIT, 1, 0, 0)
    assert O.select_policy([0, 0], P, rules) == (O.NO_SPLIT, 1, 0, 0)
    for bad in ([R(0, 9, 0, 9, 7)], [R(0, 9, 0, 9, O.SPLIT_S, num_splits=0)],
                [R(0, 9, 0, 9, O.WORK_QUEUE, chunk_pages=-1)],
                [R(0, 9, 0, 9, O.WORK_QUEUE, num_splits=0, chunk_pages=0)], [R(0, 9, 0, 9, 3, num_splits=0)],
                [R(0, 9, 0, 9, O.WORK_QUEUE, num_splits=8, chunk_pages=3, flags=O.FLAG_DEVICE_FILL)],
                [R(0, 9, 0, 9, O.SPLIT_S, num_splits=8, flags=O.FLAG_DEVICE_FILL)]):
        try:
            O.select_policy([5], P, bad)
        except ValueError:
            continue
        raise AssertionError("policy_semantics: invalid table accepted")
    try:
        O.select_policy([-1], P, rules)
    except ValueError:
        pass
    else:
        raise AssertionError("policy_semantics: negative length accepted")


def launch_fanout(O):
    g = {k: int(v) for k, v in read_golden("launch_fanout_b8.txt")}
    rng = random.Random(5)
    lens = sorted(rng.sample(range(600, 40000), g["distinct_lengths"]))
    assert len(lens) == g["batch"]
    plan = (O.WORK_QUEUE, 0, 32, O.FLAG_SEPARATE_MERGE)
    plan = (plan[0], _cdiv(_cdiv(max(lens), 16), 32), 32, plan[3])
    c = O.counters(lens, 32, 8, 128, 16, plan)
    assert c.bucket_launches == g["bucket_launches_per_step"], ("launch_fanout", c)
    assert c.launches == g["queue_launches_per_step"], ("launch_fanout", c)
    # exact-length bucketing launches one (split, merge) pair per distinct
    # non-empty length, however many rows share it
    rep = [700, 700, 5000, 700, 5000, 0, 123, 123]
    c = O.counters(rep, 32, 8, 128, 16, plan)
    assert c.bucket_launches == 2 * 3, ("launch_fanout", c)


def merge_state_closed(O):
    for lens, H_kv, P, C in itertools.chain(CASES, _random_cases(10)):
        if not lens:
            continue
        H_q, D = H_kv * 4, 64
        state = 4 * (D + 2) * 4
        S = max(1, _cdiv(_cdiv(max(lens), P), C))
        wq = O.counters(lens, H_q, H_kv, D, P, (O.WORK_QUEUE, S, C, 0))
        rect = O.counters(lens, H_q, H_kv, D, P, (O.SPLIT_S, S, C, 0))
        slots = sum(k for k in (max(1, _cdiv(_cdiv(n, P), C)) for n in lens) if k > 1)
        assert wq.merge_state_bytes == 2 * state * H_kv * slots, ("merge_state_closed", lens)
        assert rect.merge_state_bytes == (2 * state * len(lens) * H_kv * S if S > 1 else 0)
        assert wq.work_items + rect.empty_items == rect.work_items + H_kv * sum(1 for n in lens if n == 0)
        assert wq.kv_bytes == rect.kv_bytes == sum(lens) * H_kv * 4 * D


def _balanced_cases(seed=11, n=25):
    rng = random.Random(seed)
    fixed = [([32768], 8, 16, 296), ([32768], 8, 16, 37), ([0, 0], 2, 16, 5), ([5], 1, 16, 8), ([], 4, 16, 3),
             ([100, 0, 3000, 17], 8, 16, 296), ([1, 1, 1], 3, 16, 1)]
    yield from fixed
    for _ in range(n):
        B = rng.randint(1, 9)
        lens = [rng.choice([0, rng.randint(1, 40), rng.randint(1, 5000)]) for _ in range(B)]
        yield lens, rng.randint(1, 8), rng.choice([8, 16]), rng.randint(1, 300)


def balanced_shares(O):
    """Closed form: block b streams exactly floor((b+1)U/T) - floor(bU/T) pages,
    which is floor(U/T) or ceil(U/T)."""
    for lens, H_kv, P, T in _balanced_cases():
        items, indptr, bptr = O.build_balanced_queue(lens, H_kv, P, T)
        U = H_kv * sum(_cdiv(n, P) for n in lens)
        assert len(bptr) == T + 1 and bptr[0] == 0 and bptr[-1] == len(items), ("balanced_shares", lens, T)
        for b in range(T):
            got = sum(_cdiv(e, P) - bg // P for (_, _, bg, e) in items[bptr[b]:bptr[b + 1]] if e > bg)
            want = ((b + 1) * U) // T - (b * U) // T
            assert got == want and U // T <= got <= _cdiv(U, T), ("balanced_shares", lens, T, b, got, want)


def balanced_cover(O):
    for lens, H_kv, P, T in _balanced_cases(12):
        items, indptr, bptr = O.build_balanced_queue(lens, H_kv, P, T)
        assert len(indptr) == len(lens) * H_kv + 1
        for i, n in enumerate(lens):
            for h in range(H_kv):
                pair = items[indptr[i * H_kv + h]:indptr[i * H_kv + h + 1]]
                assert all(it[0] == i and it[1] == h for it in pair), "balanced_cover: wrong pair"
                if n == 0:
                    assert pair == [(i, h, 0, 0)], "balanced_cover: empty row"
                    continue
                pos = 0
                for (_, _, b, e) in pair:
                    assert b == pos and e > b and b % P == 0, ("balanced_cover", lens, T, pair)
                    pos = e
                assert pos == n, ("balanced_cover: gap", lens, T)


def _small_balanced_cases(seed=13, n=25):
    rng = random.Random(seed)
    yield from [([0, 0], 2, 16, 5), ([5], 1, 16, 8), ([], 4, 16, 3), ([100, 0, 300, 17], 4, 16, 40), ([1, 1, 1], 3, 16, 1)]
    for _ in range(n):
        B = rng.randint(1, 5)
        lens = [rng.choice([0, rng.randint(1, 40), rng.randint(1, 600)]) for _ in range(B)]
        yield lens, rng.randint(1, 4), rng.choice([8, 16]), rng.randint(1, 64)


def balanced_bruteforce(O):
    """Assign every page on its own to the block whose share holds it (found by
    scanning all blocks), then group runs of one pair inside one block."""
    for lens, H_kv, P, T in _small_balanced_cases():
        items, indptr, bptr = O.build_balanced_queue(lens, H_kv, P, T)
        U = H_kv * sum(_cdiv(n, P) for n in lens)
        owner_of_page = []
        for u in range(U):
            owner_of_page.append([b for b in range(T) if (b * U) // T <= u < ((b + 1) * U) // T][0])
        want, want_owner, u = [], [], 0
        for i, n in enumerate(lens):
            for h in range(H_kv):
                pg = _cdiv(n, P)
                if n == 0:
                    want.append((i, h, 0, 0))
                    want_owner.append(max(b for b in range(T) if (b * U) // T <= u))
                for j in range(pg):
                    b = owner_of_page[u + j]
                    if j > 0 and want_owner[-1] == b and want[-1][:2] == (i, h):
                        r = want[-1]
                        want[-1] = (i, h, r[2], min((j + 1) * P, n))
                    else:
                        want.append((i, h, j * P, min((j + 1) * P, n)))
                        want_owner.append(b)
                u += pg
        assert items == want, ("balanced_bruteforce", lens, H_kv, P, T)
        got_owner = [b for b in range(T) for _ in range(bptr[b + 1] - bptr[b])]
        assert got_owner == want_owner, ("balanced_bruteforce owners", lens, T)


def policy_fill(O):
    """The fill rule by its definition: the queue at the chosen C (built, not
    counted by formula) has at most T items, and at C - 1 it has more; when
    even whole rows exceed T, C is the longest row's page count."""
    R = O.Rule
    rng = random.Random(17)
    P = 16
    for _ in range(60):
        B = rng.randint(1, 9)
        lens = [rng.choice([0, rng.randint(1, 50), rng.randint(1, 900), rng.randint(1, 6000)]) for _ in range(B)]
        H_kv = rng.choice([1, 2, 4, 8])
        T = rng.choice([1, 7, 37, 148, 296])
        pages_max = max(_cdiv(n, P) for n in lens)
        mode, S, C, flags = O.select_policy(lens, P, [R(0, O.INT32_MAX, 0, O.INT32_MAX, O.WORK_QUEUE,
                                                       num_splits=T, chunk_pages=0, flags=4)], H_kv)
        if pages_max == 0:
            assert mode == O.NO_SPLIT, ("policy_fill empty", lens)
            continue
        assert mode == O.WORK_QUEUE and flags == 4 and 1 <= C <= pages_max, ("policy_fill", lens, T, C)
        assert S == _cdiv(pages_max, C), ("policy_fill S'", lens, T, C, S)
        n_at = len(O.build_work_queue(lens, H_kv, P, C)[0])
        if n_at > T:
            assert C == pages_max, ("policy_fill: queue too long", lens, H_kv, T, C, n_at)
            assert len(O.build_work_queue(lens, H_kv, P, pages_max)[0]) == B * H_kv
        elif C > 1:
            assert len(O.build_work_queue(lens, H_kv, P, C - 1)[0]) > T, ("policy_fill: not smallest", lens, T, C)
    # worked case: B=8 mixed-like rows, 8 heads, one wave of 296 blocks
    lens = [12129, 621, 1118, 1452, 2891, 1419, 518, 3174]
    plan = O.select_policy(lens, P, [R(0, O.INT32_MAX, 0, O.INT32_MAX, O.WORK_QUEUE, num_splits=296)], 8)
    # pages per row 759, 39, 70, 91, 181, 89, 33, 199.  C = 45: chunks 17+1+2+3+5+2+1+5 = 36 per head,
    # 8 * 36 = 288 <= 296.  C = 44: 18+1+2+3+5+3+1+5 = 38, 8 * 38 = 304 > 296.  So C = 45, S' = 17.
    assert plan == (O.WORK_QUEUE, 17, 45, 0), ("policy_fill worked case", plan)


def counters_recount(O):
    """Counters recounted by another route than the oracle's closed forms.

    queue_bytes: 16 bytes per item of the queue as built plus 4 per entry of
    its offset arrays (pair offsets; for BALANCED also the block offsets);
    kv_bytes_streamed: the distinct pages that the rows' tokens fall on,
    enumerated token by token, times a whole page of K and V per KV head;
    work_items / empty_items: the blocks of the grid and those with no token;
    merge_state_bytes: a state written and read back for every slot of a pair
    with more than one slot.  A state is G * (D + 2) fp32 values."""
    R = O.Rule
    for lens, H_kv, P, C in itertools.chain(CASES, _random_cases(21, 25)):
        G, D = 2, 64
        H_q = G * H_kv
        state = G * (D + 2) * 4
        B = len(lens)
        pages_touched = sum(len({t // P for t in range(n)}) for n in lens)
        streamed = pages_touched * P * H_kv * 2 * D * 2
        S = max(1, _cdiv(_cdiv(max(lens, default=0), P), C))
        T = (C * 7) % 41 + 1
        plans = [(O.NO_SPLIT, 1, 0, 0), (O.NO_SPLIT, 1, 0, O.FLAG_SEPARATE_MERGE), (O.SPLIT_S, S, C, 0),
                 (O.WORK_QUEUE, S, C, 0), (O.WORK_QUEUE, S, C, O.FLAG_SEPARATE_MERGE), (O.BALANCED, T, 0, 0)]
        for plan in plans:
            mode, S_, C_, flags = plan
            c = O.counters(lens, H_q, H_kv, D, P, plan)
            what = ("counters_recount", lens, H_kv, P, plan)
            assert c.kv_bytes_streamed == streamed, what
            assert c.kv_bytes == sum(lens) * H_kv * 2 * D * 2, what
            assert c.q_bytes == c.out_bytes == B * H_q * D * 2, what
            if mode == O.NO_SPLIT:
                assert (c.work_items, c.merge_state_bytes, c.queue_bytes, c.launches) == (B * H_kv, 0, 0, 1), what
                assert c.empty_items == sum(1 for i in range(B) for h in range(H_kv) if lens[i] == 0), what
                continue
            if mode == O.SPLIT_S:
                grid = [(i, h, s) for i in range(B) for h in range(H_kv) for s in range(S_)]
                assert c.work_items == len(grid) and c.queue_bytes == 0, what
                assert c.empty_items == sum(1 for (i, h, s) in grid if s * C_ * P >= lens[i]), what
                assert c.merge_state_bytes == (2 * state * len(grid) if S_ > 1 else 0), what
                continue
            if mode == O.WORK_QUEUE:
                items, indptr = O.build_work_queue(lens, H_kv, P, C_)
                offsets = len(indptr)
            else:
                items, indptr, bptr = O.build_balanced_queue(lens, H_kv, P, S_)
                offsets = len(indptr) + len(bptr)
            assert c.queue_bytes == 16 * len(items) + 4 * offsets, what
            assert c.work_items == (len(items) if mode == O.WORK_QUEUE else S_), what
            assert c.empty_items == sum(1 for it in items if it[2] == it[3]), what
            multi = sum(indptr[k + 1] - indptr[k] for k in range(B * H_kv) if indptr[k + 1] - indptr[k] > 1)
            assert c.merge_state_bytes == 2 * state * multi, what
            assert c.launches == 1 + (1 if flags & O.FLAG_SEPARATE_MERGE else 0), what
    # A device-fill plan (2, T, 0, flags) does the work of the queue the fill rule
    # picks on the host for the same budget, and sends no queue.
    for lens, H_kv, P, C in itertools.chain(CASES, _random_cases(22, 20)):
        for T in (1, 7, 37, 296):
            host = O.select_policy(lens, P, [R(0, O.INT32_MAX, 0, O.INT32_MAX, O.WORK_QUEUE, num_splits=T)], H_kv)
            dev = O.counters(lens, 8 * H_kv, H_kv, 64, P, (O.WORK_QUEUE, T, 0, O.FLAG_DEVICE_FILL))
            what = ("counters_recount device fill", lens, H_kv, P, T)
            if host[0] != O.WORK_QUEUE:  # no tokens at all: every pair has one empty item
                assert dev.work_items == len(lens) * H_kv and dev.merge_state_bytes == 0, what
                continue
            ref = O.counters(lens, 8 * H_kv, H_kv, 64, P, host)
            items, _ = O.build_work_queue(lens, H_kv, P, host[2])
            assert dev.work_items == ref.work_items == len(items) and dev.queue_bytes == 0, what
            assert (dev.merge_state_bytes, dev.empty_items) == (ref.merge_state_bytes, ref.empty_items), what
            assert dev.work_items <= max(T, len(lens) * H_kv), what
    # Worked example, by hand: lens [40, 0], H_q = 4, H_kv = 2, D = 64, P = 16, T = 3.
    # Pages per pair: 3 and 0, so U = 6 and the shares are [0,2) [2,4) [4,6).
    # Pair (0,0) = pages 0..2 -> items (0,0,0,32) in block 0 and (0,0,32,40) in block 1;
    # pair (0,1) = pages 3..5 -> (0,1,0,16) in block 1 and (0,1,16,40) in block 2;
    # row 1 is empty -> (1,0,0,0), (1,1,0,0) in block 2.  Six items, 5 pair offsets,
    # 4 block offsets: 16*6 + 4*5 + 4*4 = 132 queue bytes.  Two pairs of two slots with
    # states of 2*(64+2)*4 = 528 bytes: 2 * 4 * 528 = 4224 merge bytes.  K+V of 40 tokens:
    # 40 * 2 * 2 * 64 * 2 = 20480; of 3 whole pages: 48 * 512 = 24576.
    c = O.counters([40, 0], 4, 2, 64, 16, (O.BALANCED, 3, 0, 0))
    assert (c.launches, c.work_items, c.empty_items, c.merge_state_bytes, c.kv_bytes, c.kv_bytes_streamed,
            c.queue_bytes) == (1, 3, 2, 4224, 20480, 24576, 132), ("counters worked balanced", c)
    # The same batch without a split: 4 blocks, 2 of them for the empty row, nothing to merge.
    c = O.counters([40, 0], 4, 2, 64, 16, (O.NO_SPLIT, 1, 0, 0))
    assert (c.launches, c.work_items, c.empty_items, c.merge_state_bytes, c.queue_bytes) == (1, 4, 2, 0, 0), \
        ("counters worked no-split", c)
    # The work queue at C = 2 pages: pair (0,h) has items [0,32) and [32,40), row 1 one empty
    # item per head -> 6 items and 5 offsets: 16*6 + 4*5 = 116 bytes; merge 2 * 4 * 528.
    c = O.counters([40, 0], 4, 2, 64, 16, (O.WORK_QUEUE, 2, 2, 0))
    assert (c.work_items, c.empty_items, c.merge_state_bytes, c.queue_bytes) == (6, 2, 4224, 116), \
        ("counters worked queue", c)


def _prefix_cases(seed=31, n=40):
    """(lens, block_table, H_kv, P, C, M): rows drawn into a few sharing groups
    over a small pool, with shared runs of random length, short rows, empty
    rows and rows whose last page is partial."""
    rng = random.Random(seed)
    fixed_bt = [[5, 6, 7, 8], [5, 6, 7, 9], [5, 6, 1, 2], [3, 4, 0, 0], [5, 6, 7, 8]]
    yield [64, 60, 40, 20, 50], fixed_bt, 1, 16, 2, 2
    yield [64, 64, 64], [[1, 2, 3, 4], [1, 2, 3, 4], [1, 2, 3, 4]], 2, 16, 1, 3
    yield [15, 15, 33], [[1, 0, 0], [1, 0, 0], [1, 7, 2]], 1, 16, 1, 4
    for _ in range(n):
        B = rng.randint(1, 8)
        P = rng.choice([8, 16])
        maxp = rng.randint(1, 9)
        prefixes = [[rng.randint(0, 40) for _ in range(maxp)] for _ in range(rng.randint(1, 3))]
        lens, bt = [], []
        for _ in range(B):
            n = rng.choice([0, rng.randint(1, P * maxp), P * rng.randint(1, maxp)])
            base = rng.choice(prefixes)
            k = rng.randint(0, maxp)
            row = base[:k] + [rng.randint(41, 80) for _ in range(maxp - k)]
            lens.append(n)
            bt.append(row)
        yield lens, bt, rng.randint(1, 4), P, rng.randint(1, 4), rng.randint(1, 5)


def prefix_queue(O):
    for lens, bt, H_kv, P, C, M in _prefix_cases():
        items, indptr, uptr, uitems = O.build_prefix_queue(lens, bt, H_kv, P, C, M)
        what = ("prefix_queue", lens, bt, H_kv, P, C, M)
        groups = O.shared_prefixes(lens, bt, P)
        L_of = {r: L for rows, L in groups for r in rows}
        # items tile every (row, head) in order, page aligned, and a shared row's
        # chunks restart at its shared length
        assert len(indptr) == len(lens) * H_kv + 1 and indptr[-1] == len(items), what
        for i, n in enumerate(lens):
            for h in range(H_kv):
                pair = items[indptr[i * H_kv + h]:indptr[i * H_kv + h + 1]]
                assert all(it[:2] == (i, h) for it in pair), what
                if n == 0:
                    assert pair == [(i, h, 0, 0)], what
                    continue
                pos, L = 0, L_of.get(i, 0)
                for (_, _, b, e) in pair:
                    assert b == pos and e > b and b % P == 0 and e - b <= C * P, what
                    origin = 0 if b < L * P else L * P
                    assert (b - origin) % (C * P) == 0 and (b >= L * P or e <= L * P), what
                    pos = e
                assert pos == n, what
        # units partition the items; sizes; members share KV head, tokens and pages
        assert uptr[0] == 0 and uptr[-1] == len(uitems) == len(items), what
        assert sorted(uitems) == list(range(len(items))), what
        firsts = [uitems[uptr[u]] for u in range(len(uptr) - 1)]
        assert firsts == sorted(firsts), what
        for u in range(len(uptr) - 1):
            mem = [items[x] for x in uitems[uptr[u]:uptr[u + 1]]]
            assert 1 <= len(mem) <= M, what
            if len(mem) == 1:
                continue
            i0, h0, b0, e0 = mem[0]
            assert [m[0] for m in mem] == sorted(m[0] for m in mem), what
            for (i, h, b, e) in mem:
                assert (h, b, e) == (h0, b0, e0) and e <= (lens[i] // P) * P, what
                for pg in range(b // P, e // P):
                    assert int(bt[i][pg]) == int(bt[i0][pg]), what
        # groups: rows with a full page and a common first page; L maximal
        for rows, L in groups:
            assert len(rows) >= 2 and L >= 1, what
            first = int(bt[rows[0]][0])
            assert all(lens[r] >= P and int(bt[r][0]) == first for r in rows), what
            assert all(int(bt[r][k]) == int(bt[rows[0]][k]) for r in rows for k in range(L)), what
            assert any(lens[r] // P == L or (L < len(bt[r]) and int(bt[r][L]) != int(bt[rows[0]][L]))
                       for r in rows), what
        # completeness: two rows with a full page each and one first page share it
        group_id = {r: g for g, (rows, _) in enumerate(groups) for r in rows}
        for i in range(len(lens)):
            for j in range(i + 1, len(lens)):
                if lens[i] >= P and lens[j] >= P and int(bt[i][0]) == int(bt[j][0]):
                    assert i in group_id and group_id.get(j) == group_id[i], what
        # no sharing: the plain queue, one item per unit
        distinct = [[100 + 10 * r + k for k in range(len(bt[r]))] for r in range(len(lens))]
        items2, indptr2, uptr2, uitems2 = O.build_prefix_queue(lens, distinct, H_kv, P, C, M)
        assert (items2, indptr2) == tuple(O.build_work_queue(lens, H_kv, P, C)), what
        assert uitems2 == list(range(len(items2))) and uptr2 == list(range(len(items2) + 1)), what
    # worked example: rows 0, 1, 2, 4 share first page 5; rows 2 and 4 hold 2 full
    # pages in common with row 0, so L = 2 pages = 32 tokens
    lens, bt = [64, 60, 40, 20, 50], [[5, 6, 7, 8], [5, 6, 7, 9], [5, 6, 1, 2], [3, 4, 0, 0], [5, 6, 7, 8]]
    assert O.shared_prefixes(lens, bt, 16) == [([0, 1, 2, 4], 2)]
    items, indptr, uptr, uitems = O.build_prefix_queue(lens, bt, 1, 16, 2, 2)
    assert items == [(0, 0, 0, 32), (0, 0, 32, 64), (1, 0, 0, 32), (1, 0, 32, 60), (2, 0, 0, 32), (2, 0, 32, 40),
                     (3, 0, 0, 20), (4, 0, 0, 32), (4, 0, 32, 50)]
    assert uptr == [0, 2, 3, 4, 6, 7, 8, 9] and uitems == [0, 2, 1, 3, 4, 7, 5, 6, 8]


HOST_PINS = (queue_closed_form, queue_cover, queue_bruteforce, policy_paper, policy_semantics, policy_fill,
             launch_fanout, merge_state_closed, counters_recount, balanced_shares, balanced_cover,
             balanced_bruteforce, prefix_queue)


def run_all(O):
    failed = []
    for pin in HOST_PINS:
        try:
            pin(O)
        except (AssertionError, ValueError, IndexError, TypeError) as e:
            failed.append(f"{pin.__name__}: {e}")
    return failed
