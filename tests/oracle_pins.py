"""Pins that tie the CPU oracle to facts other than itself.

Each check takes a loaded C oracle (`lib`), so the same checks run against the
real oracle (tests/test_oracle_pins.py) and against copies with a planted
mistake (tests/test_oracle_mutations.py), which must fail at least one of them.

What pins what (the method's definition is the plain softmax-weighted sum of
the cached values, read through the block table; see the oracle's header):
  single_token      N = 1 returns that token's V exactly (closed form)
  identical_keys    equal keys give the plain mean of V (closed form)
  scale_zero        scale = 0 gives the plain mean of V (closed form)
  ones_values       V = 1 everywhere gives exactly 1 (normalisation)
  dominant_key      one key with a logit gap > 50 returns its V (limit case)
  sdpa_dense        identity block table == dense tensor; torch's
                    scaled_dot_product_attention in float64 with K/V heads
                    repeated G times (library routine) agrees to 1e-12
  gqa_replication   G = 4 equals G = 1 (MHA) on a pool with each KV head copied G times
  page_permutation  renumbering physical pages (pool + table) changes nothing
  nan_poison        NaN in every unused page / tail slot / table entry changes nothing
  empty_row         N = 0 gives zeros
  split_merge       partial states over any chunking, merged, equal the unsplit result
"""
from __future__ import annotations

import math

import numpy as np
import torch

from oracle import oracle as O
from paged_kv_gqa_17_b200 import workloads as W


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float64).numpy()


def _pr(w: W.Workload, scale=None):
    return O.problem(w.q, w.k_pool, w.v_pool, w.block_table, w.seq_lens,
                     w.scale if scale is None else scale, layout=w.layout)


def _row_values(w: W.Workload, pool: torch.Tensor, row: int, h: int) -> np.ndarray:
    """[N][D] values of (row, kv head h) in token order, read page by page."""
    n = w.seq_lens[row]
    out = []
    for p in range(-(-n // w.P)):
        page = int(w.block_table[row, p])
        take = min(w.P, n - p * w.P)
        out.append(_f64(pool[page, h, :take, :]))
    return np.concatenate(out, axis=0) if out else np.zeros((0, w.D))


def single_token(lib):
    w = W.make_custom([1, 1, 1, 1], H_q=8, H_kv=2, D=64, seed=11, poison=True)
    got = O.paged_decode(_pr(w), lib=lib)
    for i in range(w.B):
        page = int(w.block_table[i, 0])
        for hq in range(w.H_q):
            want = _f64(w.v_pool[page, hq // w.G, 0, :])
            assert np.array_equal(got[i, hq], want), ("single_token", i, hq)


def identical_keys(lib):
    w = W.make_custom([37, 100, 16, 129], H_q=8, H_kv=2, D=64, seed=12, poison=True)
    key = torch.randn(w.D, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    for i, n in enumerate(w.seq_lens):
        for p in range(-(-n // w.P)):
            page = int(w.block_table[i, p])
            take = min(w.P, n - p * w.P)
            w.k_pool[page, :, :take, :] = key
    got = O.paged_decode(_pr(w), lib=lib)
    for i in range(w.B):
        for hq in range(w.H_q):
            want = _row_values(w, w.v_pool, i, hq // w.G).mean(axis=0)
            assert np.allclose(got[i, hq], want, rtol=0, atol=1e-12), ("identical_keys", i, hq)


def scale_zero(lib):
    w = W.make_custom([50, 300], H_q=4, H_kv=2, D=128, seed=13, poison=True)
    got = O.paged_decode(_pr(w, scale=0.0), lib=lib)
    for i in range(w.B):
        for hq in range(w.H_q):
            want = _row_values(w, w.v_pool, i, hq // w.G).mean(axis=0)
            assert np.allclose(got[i, hq], want, rtol=0, atol=1e-12), ("scale_zero", i, hq)


def ones_values(lib):
    w = W.make_custom([77, 513, 5], H_q=8, H_kv=2, D=64, seed=14, poison=True, q_scale=4.0)
    for i, n in enumerate(w.seq_lens):
        for p in range(-(-n // w.P)):
            page = int(w.block_table[i, p])
            take = min(w.P, n - p * w.P)
            w.v_pool[page, :, :take, :] = 1.0
    got = O.paged_decode(_pr(w), lib=lib)
    assert np.allclose(got, 1.0, rtol=0, atol=1e-14), "ones_values"


def dominant_key(lib):
    """Token t* gets a key along q of its head group, so its logit exceeds every
    other by more than 50: the output is its V to within exp(-50)."""
    w = W.make_custom([200, 61], H_q=4, H_kv=4, D=64, seed=15, poison=True)
    rng = np.random.default_rng(3)
    for i, n in enumerate(w.seq_lens):
        t_star = int(rng.integers(0, n))
        page = int(w.block_table[i, t_star // w.P])
        slot = t_star % w.P
        for h in range(w.H_kv):
            qv = w.q[i, h].to(torch.float32)
            w.k_pool[page, h, slot, :] = (qv * (600.0 / float(qv.norm() ** 2) * math.sqrt(w.D))).to(torch.bfloat16)
    got = O.paged_decode(_pr(w), lib=lib)
    rng = np.random.default_rng(3)
    for i, n in enumerate(w.seq_lens):
        t_star = int(rng.integers(0, n))
        page = int(w.block_table[i, t_star // w.P])
        for hq in range(w.H_q):
            want = _f64(w.v_pool[page, hq, t_star % w.P, :])
            assert np.allclose(got[i, hq], want, rtol=0, atol=1e-12), ("dominant_key", i, hq)


def sdpa_dense(lib):
    """Pages laid out so that the pool *is* a dense [B][N][H_kv][D] tensor (NHD
    pool, identity block table, full pages), compared with torch SDPA."""
    B, H_q, H_kv, D, P, N = 2, 8, 2, 64, 16, 64
    g = torch.Generator().manual_seed(16)
    q = torch.randn(B, H_q, D, generator=g).to(torch.bfloat16)
    k = torch.randn(B * N // P, P, H_kv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B * N // P, P, H_kv, D, generator=g).to(torch.bfloat16)
    bt = torch.arange(B * N // P, dtype=torch.int32).reshape(B, N // P)
    pr = O.problem(q, k, v, bt, [N] * B, 1.0 / math.sqrt(D), layout="NHD")
    got = O.paged_decode(pr, lib=lib)
    kd = k.to(torch.float64).reshape(B, N, H_kv, D).transpose(1, 2).repeat_interleave(H_q // H_kv, dim=1)
    vd = v.to(torch.float64).reshape(B, N, H_kv, D).transpose(1, 2).repeat_interleave(H_q // H_kv, dim=1)
    qd = q.to(torch.float64).unsqueeze(2)
    want = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, scale=1.0 / math.sqrt(D)).squeeze(2)
    assert np.allclose(got, want.numpy(), rtol=0, atol=1e-12), "sdpa_dense"


def gqa_replication(lib):
    w = W.make_custom([90, 17, 256], H_q=8, H_kv=2, D=64, seed=17, poison=False)
    got = O.paged_decode(_pr(w), lib=lib)
    G = w.G
    k1 = w.k_pool.repeat_interleave(G, dim=1)
    v1 = w.v_pool.repeat_interleave(G, dim=1)
    pr1 = O.problem(w.q, k1, v1, w.block_table, w.seq_lens, w.scale)
    want = O.paged_decode(pr1, lib=lib)
    assert np.array_equal(got, want), "gqa_replication"


def page_permutation(lib):
    w = W.make_custom([33, 250, 16, 500], H_q=8, H_kv=4, D=64, seed=18, poison=True)
    got = O.paged_decode(_pr(w), lib=lib)
    perm = torch.randperm(w.num_pages, generator=torch.Generator().manual_seed(99))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(w.num_pages)
    # new physical page j holds old page perm[j]; old page p now lives at inv[p]
    k2, v2 = w.k_pool[perm].clone(), w.v_pool[perm].clone()
    bt2 = inv[w.block_table.long()].to(torch.int32)
    pr2 = O.problem(w.q, k2, v2, bt2, w.seq_lens, w.scale)
    want = O.paged_decode(pr2, lib=lib)
    assert np.array_equal(got, want), "page_permutation"


def nan_poison(lib):
    lens = [1, 15, 16, 17, 300, 1023]
    clean = W.make_custom(lens, H_q=8, H_kv=2, D=128, seed=19, poison=False)
    dirty = W.make_custom(lens, H_q=8, H_kv=2, D=128, seed=19, poison=True)
    a = O.paged_decode(_pr(clean), lib=lib)
    b = O.paged_decode(_pr(dirty), lib=lib)
    assert np.isfinite(b).all(), "nan_poison: NaN reached the output"
    assert np.array_equal(a, b), "nan_poison"


def empty_row(lib):
    w = W.make_custom([0, 40, 0], H_q=4, H_kv=1, D=64, seed=20, poison=True)
    got = O.paged_decode(_pr(w), lib=lib)
    assert np.array_equal(got[0], np.zeros_like(got[0])), "empty_row"
    assert np.array_equal(got[2], np.zeros_like(got[2])), "empty_row"
    assert np.isfinite(got[1]).all() and np.abs(got[1]).sum() > 0, "empty_row"


def split_merge(lib):
    w = W.make_custom([700, 33, 1], H_q=8, H_kv=2, D=64, seed=21, poison=True, q_scale=8.0)
    pr = _pr(w)
    full = O.paged_decode(pr, lib=lib)
    for i, n in enumerate(w.seq_lens):
        pages = -(-n // w.P)
        for C in sorted({1, 2, 3, 7, -(-pages // 32), -(-pages // 2), pages}):
            C = max(1, C)
            span = C * w.P
            for hq in (0, w.H_q - 1):
                states = [O.partial_state(pr, i, hq, b, min(b + span, n), lib=lib) for b in range(0, n, span)]
                states.append(O.partial_state(pr, i, hq, n, n, lib=lib))  # an empty split
                ms, ls, accs = zip(*states)
                merged = O.merge_states(ms, ls, accs, lib=lib)
                assert np.allclose(merged, full[i, hq], rtol=0, atol=1e-12), ("split_merge", i, C, hq)


ATTENTION_PINS = (single_token, identical_keys, scale_zero, ones_values, dominant_key, sdpa_dense,
                  gqa_replication, page_permutation, nan_poison, empty_row, split_merge)


def run_all(lib):
    """Run every attention pin; return the names of those that fail."""
    failed = []
    for pin in ATTENTION_PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError) as e:  # a wrong oracle may also reject inputs
            failed.append(f"{pin.__name__}: {e}")
    return failed
