"""Randomised forms of the oracle's invariant pins (hypothesis), on small
problems drawn at random instead of the fixed cases of tests/oracle_pins.py:

  split_merge       cutting a row's tokens at ANY points (page-aligned or not,
                    empty pieces included) and merging the partial states
                    gives the unsplit result (the page's exact merge)
  page_permutation  renumbering physical pages changes nothing, bit for bit
  nan_poison        NaN in every unused page and tail slot changes nothing
  gqa_replication   G-way sharing equals MHA on a pool with each KV head
                    copied G times, bit for bit
  sdpa_dense        torch's scaled_dot_product_attention in float64 on the
                    gathered rows (library routine) agrees to 1e-12
"""
import numpy as np
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from oracle import oracle as O
from paged_kv_gqa_17_b200 import workloads as W

SETTINGS = settings(max_examples=30, deadline=None, derandomize=True,
                    suppress_health_check=[HealthCheck.too_slow, HealthCheck.function_scoped_fixture])

lens_st = st.lists(st.one_of(st.integers(0, 40), st.integers(1, 300)), min_size=1, max_size=4)
group_st = st.sampled_from([(4, 1), (8, 2), (8, 4), (16, 2), (4, 4)])   # (H_q, H_kv)
seed_st = st.integers(0, 2**31 - 1)


def _pr(w, layout=None):
    return O.problem(w.q, w.k_pool, w.v_pool, w.block_table, w.seq_lens, w.scale, layout=layout or w.layout)


@SETTINGS
@given(lens=lens_st, heads=group_st, seed=seed_st, cuts=st.lists(st.floats(0, 1), max_size=6),
       q_scale=st.sampled_from([1.0, 8.0]))
def test_split_at_any_points_merges_to_the_unsplit_result(olib, lens, heads, seed, cuts, q_scale):
    H_q, H_kv = heads
    w = W.make_custom(lens, H_q, H_kv, 64, seed=seed % 100000, poison=True, q_scale=q_scale)
    pr = _pr(w)
    full = O.paged_decode(pr, lib=olib)
    for i, n in enumerate(w.seq_lens):
        bounds = sorted({0, n, *(int(c * n) for c in cuts)})
        pieces = list(zip(bounds[:-1], bounds[1:])) + [(n, n)]   # plus one empty piece
        for hq in {0, H_q - 1}:
            ms, ls, accs = zip(*[O.partial_state(pr, i, hq, b, e, lib=olib) for b, e in pieces])
            merged = O.merge_states(ms, ls, accs, lib=olib)
            assert np.allclose(merged, full[i, hq], rtol=0, atol=1e-12), (lens, i, hq, pieces)


@SETTINGS
@given(lens=lens_st, heads=group_st, seed=seed_st, perm_seed=seed_st)
def test_renumbering_pages_changes_nothing(olib, lens, heads, seed, perm_seed):
    H_q, H_kv = heads
    w = W.make_custom(lens, H_q, H_kv, 64, seed=seed % 100000, poison=True)
    got = O.paged_decode(_pr(w), lib=olib)
    perm = torch.randperm(w.num_pages, generator=torch.Generator().manual_seed(perm_seed))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(w.num_pages)
    pr2 = O.problem(w.q, w.k_pool[perm].clone(), w.v_pool[perm].clone(), inv[w.block_table.long()].to(torch.int32),
                    w.seq_lens, w.scale)
    assert np.array_equal(got, O.paged_decode(pr2, lib=olib))


@SETTINGS
@given(lens=lens_st, heads=group_st, seed=seed_st)
def test_nan_outside_the_rows_changes_nothing(olib, lens, heads, seed):
    H_q, H_kv = heads
    clean = W.make_custom(lens, H_q, H_kv, 64, seed=seed % 100000, poison=False)
    dirty = W.make_custom(lens, H_q, H_kv, 64, seed=seed % 100000, poison=True)
    a = O.paged_decode(_pr(clean), lib=olib)
    b = O.paged_decode(_pr(dirty), lib=olib)
    assert np.isfinite(b).all() and np.array_equal(a, b)


@SETTINGS
@given(lens=lens_st, heads=group_st, seed=seed_st)
def test_grouped_heads_equal_replicated_heads(olib, lens, heads, seed):
    H_q, H_kv = heads
    G = H_q // H_kv
    w = W.make_custom(lens, H_q, H_kv, 64, seed=seed % 100000, poison=False)
    got = O.paged_decode(_pr(w), lib=olib)
    pr1 = O.problem(w.q, w.k_pool.repeat_interleave(G, dim=1), w.v_pool.repeat_interleave(G, dim=1),
                    w.block_table, w.seq_lens, w.scale)
    assert np.array_equal(got, O.paged_decode(pr1, lib=olib))


@SETTINGS
@given(lens=st.lists(st.integers(1, 64), min_size=1, max_size=3), heads=group_st, seed=seed_st,
       q_scale=st.sampled_from([1.0, 4.0]))
def test_library_attention_agrees_on_gathered_rows(olib, lens, heads, seed, q_scale):
    H_q, H_kv = heads
    G = H_q // H_kv
    w = W.make_custom(lens, H_q, H_kv, 64, seed=seed % 100000, poison=True, q_scale=q_scale)
    got = O.paged_decode(_pr(w), lib=olib)
    for i, n in enumerate(w.seq_lens):
        pages = w.block_table[i, :-(-n // w.P)].long()
        k = w.k_pool[pages].permute(1, 0, 2, 3).reshape(H_kv, -1, w.D)[:, :n].double()   # [H_kv][N][D]
        v = w.v_pool[pages].permute(1, 0, 2, 3).reshape(H_kv, -1, w.D)[:, :n].double()
        q = w.q[i].double().unsqueeze(1)                                                     # [H_q][1][D]
        ref = torch.nn.functional.scaled_dot_product_attention(
            q, k.repeat_interleave(G, dim=0), v.repeat_interleave(G, dim=0), scale=w.scale)
        assert np.allclose(got[i], ref.squeeze(1).numpy(), rtol=0, atol=1e-12), (lens, i)
