"""Property-based search (hypothesis) for the C host planner against the
oracle's plain-Python planner, aimed at the edges the seeded random cases
reach only by chance: lengths one token either side of a page or chunk
boundary, empty rows, and fill budgets equal to the item count of some
chunk size.  Bounded example counts keep the suite to seconds."""
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from oracle import oracle as O
from paged_kv_gqa_17_b200 import binding as bd

P = 16
ANY = (0, 2**31 - 1, 0, 2**31 - 1)
SETTINGS = settings(max_examples=250, deadline=None, derandomize=True, suppress_health_check=[HealthCheck.too_slow])

boundary = st.builds(lambda k, d: max(0, k * P + d), st.integers(0, 300), st.integers(-1, 1))
length = st.one_of(st.just(0), st.integers(1, 40), boundary, st.integers(1, 70000))
lengths = st.lists(length, min_size=0, max_size=14)
heads = st.sampled_from([1, 2, 4, 8])


@pytest.fixture(scope="module")
def L():
    from paged_kv_gqa_17_b200 import build

    build.build()
    return bd.lib()


def shape_for(lens, H_kv, G=4, D=128):
    return bd.make_shape(len(lens), H_kv * G, H_kv, D, P, 1 + max([-(-n // P) for n in lens] + [0]), 1)


def items_at(lens, H_kv, C):
    return H_kv * sum(max(1, -(-(-(-n // P)) // C)) for n in lens)


@SETTINGS
@given(lens=lengths, H_kv=heads, T=st.integers(1, 700), deep=st.booleans())
def test_fill_rule_matches_the_oracle_and_is_minimal(L, lens, H_kv, T, deep):
    shape = shape_for(lens, H_kv)
    rules = [bd.Rule(*ANY, bd.WORK_QUEUE, T, 0, 4 if deep else 0)]
    got = bd.select_policy(lens, shape, rules).tuple()
    assert got == O.select_policy(lens, P, [O.Rule(*r.tuple()) for r in rules], H_kv)
    pages_max = max([-(-n // P) for n in lens] + [0])
    if not lens or pages_max == 0:
        assert got[0] == bd.NO_SPLIT
        return
    C = got[2]
    assert 1 <= C <= pages_max and got[1] == -(-pages_max // C)
    if items_at(lens, H_kv, pages_max) > T:
        assert C == pages_max          # even whole rows overflow the wave
    else:
        assert items_at(lens, H_kv, C) <= T
        assert C == 1 or items_at(lens, H_kv, C - 1) > T


@SETTINGS
@given(lens=lengths, H_kv=heads, C=st.integers(1, 80))
def test_work_queue_matches_the_oracle(L, lens, H_kv, C):
    items, indptr = bd.build_work_queue(lens, shape_for(lens, H_kv), C)
    w_items, w_indptr = O.build_work_queue(lens, H_kv, P, C)
    assert [tuple(x) for x in items.tolist()] == w_items
    assert indptr.tolist() == w_indptr


@SETTINGS
@given(lens=lengths, H_kv=heads, T=st.integers(1, 400))
def test_balanced_queue_matches_the_oracle_and_its_capacity_bound(L, lens, H_kv, T):
    shape = shape_for(lens, H_kv)
    items, indptr = bd.build_balanced_queue(lens, shape, T)
    w_items, w_indptr, w_bptr = O.build_balanced_queue(lens, H_kv, P, T)
    assert [tuple(x) for x in items.tolist()] == w_items
    assert indptr.tolist() == w_indptr + w_bptr
    assert len(w_items) <= bd.balanced_queue_capacity(shape, T)


@SETTINGS
@given(lens=lengths, H_kv=heads, G=st.sampled_from([1, 4, 8, 16]), mode=st.sampled_from([0, 1, 2, 3]),
       S=st.integers(1, 64), C=st.integers(0, 40), flags=st.sampled_from([0, 1, 4, 5]))
def test_counters_match_the_oracle(L, lens, H_kv, G, mode, S, C, flags):
    shape = shape_for(lens, H_kv, G)
    plan = bd.select_policy(lens, shape, [bd.Rule(*ANY, mode, S, C, flags)])
    got = bd.plan_counters(lens, shape, plan)
    assert got == O.counters(lens, H_kv * G, H_kv, 128, P, plan.tuple()).__dict__


@SETTINGS
@given(lens=lengths, H_kv=heads, T=st.integers(1, 700))
def test_fill_queue_capacity_bounds_every_fill_queue(L, lens, H_kv, T):
    shape = shape_for(lens, H_kv)
    plan = bd.select_policy(lens, shape, [bd.Rule(*ANY, bd.WORK_QUEUE, T, 0, 0)])
    if plan.mode != bd.WORK_QUEUE:
        return
    items, _ = bd.build_work_queue(lens, shape, plan.chunk_pages)
    assert items.shape[0] <= bd.fill_queue_capacity(shape, T)
