"""CPU oracle for paged GQA decode attention (TEST INFRASTRUCTURE ONLY).

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
legs may import this module.  It shares no code with the CUDA library: the
attention arithmetic lives in oracle/pkv_oracle.c (plain C, fp64), the host
scheduling pieces below are plain Python written from the pages' description.

Citations name the page and its section:
  [PKV]  "PersistentKV: Page-Aware Decode Scheduling for Long-Context LLM
         Serving on Commodity GPUs" (gist.science explainer), Technical summary.
Parity pins for every function here live in tests/oracle_pins.py.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import List, Optional, Sequence, Tuple

import numpy as np

from . import build_oracle

# Plan modes, as the pages name the three execution paths
# [PKV, Methodology 2 "Calibrated adaptive policy"].
NO_SPLIT = 0
SPLIT_S = 1
WORK_QUEUE = 2
BALANCED = 3  # the compact work queue, cut into equal shares for a fixed number of blocks
FLAG_SEPARATE_MERGE = 1
# a work-queue plan whose chunk is found per step from the lengths on the device:
# the plan carries the fill budget T instead of the chunk, (WORK_QUEUE, T, 0, flags)
FLAG_DEVICE_FILL = 32
INT32_MAX = 2**31 - 1

_lib = None


def load(path: Optional[str] = None):
    """Load (building if needed) the C oracle; `path` selects another build of it."""
    global _lib
    if path is None and _lib is not None:
        return _lib
    lib = ctypes.CDLL(path or build_oracle.build())
    p = ctypes.c_void_p
    i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
    common = [p, p, p, i64, i64, i64, p, i32, p, i32, i32, i32, i32, i32, f64]
    lib.oracle_paged_decode.argtypes = common + [p, i32]
    lib.oracle_paged_decode.restype = ctypes.c_int
    lib.oracle_paged_decode_pairs.argtypes = common + [p, i64, p, i32]
    lib.oracle_paged_decode_pairs.restype = ctypes.c_int
    lib.oracle_partial_state.argtypes = common + [i32, i32, i32, i32, p, p, p]
    lib.oracle_partial_state.restype = ctypes.c_int
    lib.oracle_merge_states.argtypes = [i32, p, p, p, i32, p]
    lib.oracle_merge_states.restype = ctypes.c_int
    if path is None:
        _lib = lib
    return lib


def _u16(t) -> np.ndarray:
    """bf16 tensor (torch) or uint16 array -> contiguous uint16 numpy array of bit patterns."""
    if isinstance(t, np.ndarray):
        assert t.dtype == np.uint16
        return np.ascontiguousarray(t)
    import torch

    assert t.dtype == torch.bfloat16, t.dtype
    return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _i32(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return np.ascontiguousarray(t, dtype=np.int32)
    try:
        import torch

        if isinstance(t, torch.Tensor):
            return np.ascontiguousarray(t.detach().cpu().numpy().astype(np.int32))
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(t, dtype=np.int32))


@dataclass
class Problem:
    """Raw inputs of one decode step, as bit patterns and integers.

    q: [B][H_q][D]; k_pool/v_pool: a pool addressed by element strides
    (s_page, s_head, s_tok), head_dim stride 1; block_table: [B][max_pages];
    seq_lens: [B]; P: tokens per page.
    """

    q: np.ndarray
    k_pool: np.ndarray
    v_pool: np.ndarray
    s_page: int
    s_head: int
    s_tok: int
    block_table: np.ndarray
    seq_lens: np.ndarray
    B: int
    H_q: int
    H_kv: int
    D: int
    P: int
    scale: float

    @property
    def max_pages(self) -> int:
        return int(self.block_table.shape[1]) if self.block_table.ndim == 2 else 0

    def _args(self):
        return (
            self.q.ctypes.data, self.k_pool.ctypes.data, self.v_pool.ctypes.data,
            self.s_page, self.s_head, self.s_tok,
            self.block_table.ctypes.data, self.max_pages, self.seq_lens.ctypes.data,
            self.B, self.H_q, self.H_kv, self.D, self.P, float(self.scale),
        )


def problem(q, k_pool, v_pool, block_table, seq_lens, scale: float, layout: str = "HND") -> Problem:
    """Build a Problem from torch tensors: bf16 q [B][H_q][D] and bf16 pools,
    [pages][H_kv][P][D] for layout "HND" or [pages][P][H_kv][D] for "NHD"."""
    B, H_q, D = (int(x) for x in q.shape)
    if layout == "HND":
        _, H_kv, P, D2 = (int(x) for x in k_pool.shape)
        strides = (H_kv * P * D, P * D, D)
    elif layout == "NHD":
        _, P, H_kv, D2 = (int(x) for x in k_pool.shape)
        strides = (P * H_kv * D, D, H_kv * D)
    else:
        raise ValueError(layout)
    assert D2 == D
    bt = _i32(block_table).reshape(B, -1)
    return Problem(_u16(q), _u16(k_pool), _u16(v_pool), int(strides[0]), int(strides[1]), int(strides[2]),
                   bt, _i32(seq_lens).reshape(-1), B, H_q, H_kv, D, P, float(scale))


def paged_decode(pr: Problem, n_threads: int = 1, lib=None) -> np.ndarray:
    """softmax(q K^T * scale) V per (row, query head), fp64 -> [B][H_q][D]."""
    lib = lib or load()
    out = np.zeros((pr.B, pr.H_q, pr.D), dtype=np.float64)
    rc = lib.oracle_paged_decode(*pr._args(), out.ctypes.data, int(n_threads))
    if rc != 0:
        raise ValueError("oracle_paged_decode rejected the problem")
    return out


def paged_decode_pairs(pr: Problem, pairs: Sequence[Tuple[int, int]], n_threads: int = 1, lib=None) -> np.ndarray:
    """Only the listed (row, query head) outputs -> [len(pairs)][D]."""
    lib = lib or load()
    pa = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
    out = np.zeros((pa.shape[0], pr.D), dtype=np.float64)
    rc = lib.oracle_paged_decode_pairs(*pr._args(), pa.ctypes.data, int(pa.shape[0]), out.ctypes.data, int(n_threads))
    if rc != 0:
        raise ValueError("oracle_paged_decode_pairs rejected the problem")
    return out


def partial_state(pr: Problem, row: int, hq: int, tok_begin: int, tok_end: int, lib=None):
    """(m, l, acc[D]) of one token range [PKV, Methodology 1 "Sequence splitting"]."""
    lib = lib or load()
    m = ctypes.c_double()
    l = ctypes.c_double()
    acc = np.zeros(pr.D, dtype=np.float64)
    rc = lib.oracle_partial_state(*pr._args(), row, hq, tok_begin, tok_end,
                                  ctypes.addressof(m), ctypes.addressof(l), acc.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_partial_state rejected the range")
    return m.value, l.value, acc


def merge_states(ms: Sequence[float], ls: Sequence[float], accs: Sequence[np.ndarray], lib=None) -> np.ndarray:
    """Exact merge of partial states [PKV, Methodology 1: "a separate merge kernel combines them exactly"]."""
    lib = lib or load()
    n = len(ms)
    D = int(accs[0].shape[0]) if n else 0
    m = np.ascontiguousarray(np.asarray(ms, dtype=np.float64))
    l = np.ascontiguousarray(np.asarray(ls, dtype=np.float64))
    a = np.ascontiguousarray(np.stack(accs).astype(np.float64)) if n else np.zeros((0, 0))
    out = np.zeros(D, dtype=np.float64)
    lib.oracle_merge_states(n, m.ctypes.data, l.ctypes.data, a.ctypes.data, D, out.ctypes.data)
    return out


# --------------------------------------------------------------------------
# Host scheduling: written from the pages in plain Python.


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def build_work_queue(seq_lens: Sequence[int], H_kv: int, P: int, chunk_pages: int):
    """Compact work queue [PKV, Methodology 1 "Compact work queue"; Key contributions
    "page-aware scheduling"].

    One item per (row i, KV head h, chunk c) whose token range is non-empty,
    in lexicographic (i, h, c) order.  Chunks are `chunk_pages` whole pages:
    chunk c covers tokens [c*C*P, min((c+1)*C*P, N_i)), so its bounds come
    from the row's real length N_i, never a padded one ("Row-local bounds").
    A row with N_i = 0 gets a single empty item (i, h, 0, 0) per head, so
    that its zero output is still written.

    Returns (items as a list of (row, kv_head, tok_begin, tok_end), indptr of
    length B*H_kv + 1 where items indptr[i*H_kv + h] .. indptr[i*H_kv + h + 1]
    belong to (i, h)).
    """
    if chunk_pages < 1 or H_kv < 1 or P < 1:
        raise ValueError("chunk_pages, H_kv and P must be positive")
    items: List[Tuple[int, int, int, int]] = []
    indptr = [0]
    span = chunk_pages * P
    for i, n in enumerate(seq_lens):
        n = int(n)
        if n < 0:
            raise ValueError("negative sequence length")
        for h in range(H_kv):
            if n == 0:
                items.append((i, h, 0, 0))
            else:
                c = 0
                while c * span < n:
                    items.append((i, h, c * span, min((c + 1) * span, n)))
                    c += 1
            indptr.append(len(items))
    return items, indptr


def build_balanced_queue(seq_lens: Sequence[int], H_kv: int, P: int, n_blocks: int):
    """Compact work queue cut into equal shares for `n_blocks` blocks.

    The (row, KV head) pairs are laid end to end in lexicographic order, each
    contributing ceil(N_i / P) pages; of the U pages in total, block b owns
    pages [floor(b*U/T), floor((b+1)*U/T)) (T = n_blocks).  Every maximal run
    of one pair's pages inside one block's share is an item
    (row, kv_head, tok_begin, tok_end), so items stay row-local and
    page-aligned [PKV, Methodology 1 "Compact work queue", "Row-local
    bounds"].  A row with N_i = 0 gets one empty item per head, owned by the
    last block whose share starts at or before the pair's position.

    Returns (items in lexicographic order, indptr over pairs as in
    build_work_queue, block_ptr of length T + 1: block b owns items
    block_ptr[b] .. block_ptr[b+1]).
    """
    if n_blocks < 1 or H_kv < 1 or P < 1:
        raise ValueError("n_blocks, H_kv and P must be positive")
    lens = [int(n) for n in seq_lens]
    if any(n < 0 for n in lens):
        raise ValueError("negative sequence length")
    T = n_blocks
    pages = [_ceil_div(n, P) for n in lens]
    U = H_kv * sum(pages)
    starts = [(b * U) // T for b in range(T + 1)]

    def owner(u):
        b = T - 1
        while starts[b] > u:
            b -= 1
        return b

    items, owners, indptr = [], [], [0]
    u = 0
    for i, n in enumerate(lens):
        for h in range(H_kv):
            if n == 0:
                items.append((i, h, 0, 0))
                owners.append(owner(u))
            else:
                x = u
                while x < u + pages[i]:
                    b = owner(x)
                    y = min(u + pages[i], starts[b + 1])
                    items.append((i, h, (x - u) * P, min((y - u) * P, n)))
                    owners.append(b)
                    x = y
            indptr.append(len(items))
            u += pages[i]
    block_ptr = [0] * (T + 1)
    k = 0
    for b in range(T + 1):
        while k < len(owners) and owners[k] < b:
            k += 1
        block_ptr[b] = k
    return items, indptr, block_ptr


def shared_prefixes(seq_lens: Sequence[int], block_table, P: int):
    """Groups of rows whose block tables start with the same physical pages
    ["Chapter 8 - Next-generation KV cache management", 8.1: reference-counted
    block sharing, best-of-8 over one prompt; 8.3: the first thousands of
    tokens repeat across requests and the block table makes them shared
    physical blocks].

    Rows with at least one full page and the same first physical page form a
    group (its lowest row leads); the group's shared length L (pages) is the
    number of leading table entries every member has in common with the
    leader, counting only pages that are full in every member, so no member's
    last, partial page falls inside the shared range.  Returns a list of
    (rows in ascending order, L) for every group of two or more rows with
    L >= 1."""
    lens = [int(n) for n in seq_lens]
    by_first = {}
    for i, n in enumerate(lens):
        if n >= P:
            by_first.setdefault(int(block_table[i][0]), []).append(i)
    groups = []
    for first in sorted(by_first, key=lambda f: by_first[f][0]):
        rows = by_first[first]
        if len(rows) < 2:
            continue
        lead = rows[0]
        L = lens[lead] // P
        for r in rows[1:]:
            full = lens[r] // P
            k = 0
            while k < min(full, L) and int(block_table[r][k]) == int(block_table[lead][k]):
                k += 1
            L = min(L, k)
        if L >= 1:
            groups.append((rows, L))
    return groups


def build_prefix_queue(seq_lens: Sequence[int], block_table, H_kv: int, P: int, chunk_pages: int,
                       max_members: int):
    """Compact work queue that stages shared prefix pages once for several rows.

    Items per (row i, KV head h), in lexicographic order as in
    build_work_queue: a row in a sharing group (shared_prefixes) with shared
    length L pages has its shared range [0, L*P) cut into chunks of C pages
    from 0, then the rest [L*P, N_i) cut into chunks of C pages from L*P;
    every other row is cut as in build_work_queue.  Row-local, page-aligned
    bounds as on the pages [PKV, Methodology 1 "Compact work queue",
    "Row-local bounds"].

    Units (what one block runs): for every group, KV head and shared chunk,
    the members' items of that chunk, in row order, in runs of at most
    `max_members`; every other item is a unit of its own.  The members of a
    unit cover the same tokens of the same KV head on the same physical
    pages, so one staging of each page serves all of them; each member still
    gets its own item, i.e. its own partial state, and its pair merges as in
    the plain queue.  Units are ordered by their first member's item.

    Returns (items, indptr over pairs, unit_ptr of length n_units + 1,
    unit_items: the members' item indices, unit by unit)."""
    if chunk_pages < 1 or H_kv < 1 or P < 1 or max_members < 1:
        raise ValueError("chunk_pages, H_kv, P and max_members must be positive")
    lens = [int(n) for n in seq_lens]
    if any(n < 0 for n in lens):
        raise ValueError("negative sequence length")
    span = chunk_pages * P
    shared = {}
    for g, (rows, L) in enumerate(shared_prefixes(lens, block_table, P)):
        for r in rows:
            shared[r] = (g, L)
    items, indptr = [], [0]
    chunk_item = {}  # (group, h, shared chunk c, row) -> item index
    for i, n in enumerate(lens):
        for h in range(H_kv):
            if n == 0:
                items.append((i, h, 0, 0))
            elif i in shared:
                g, L = shared[i]
                c = 0
                while c * span < L * P:
                    chunk_item[(g, h, c, i)] = len(items)
                    items.append((i, h, c * span, min((c + 1) * span, L * P)))
                    c += 1
                t = L * P
                while t < n:
                    items.append((i, h, t, min(t + span, n)))
                    t += span
            else:
                c = 0
                while c * span < n:
                    items.append((i, h, c * span, min((c + 1) * span, n)))
                    c += 1
            indptr.append(len(items))
    grouped = set(chunk_item.values())
    units = []
    keys = sorted({k[:3] for k in chunk_item})
    for key in keys:
        members = [chunk_item[key + (r,)] for r in sorted(r for (g, h, c, r) in chunk_item if (g, h, c) == key)]
        for k in range(0, len(members), max_members):
            units.append(members[k:k + max_members])
    units += [[x] for x in range(len(items)) if x not in grouped]
    units.sort(key=lambda u: u[0])
    unit_ptr, unit_items = [0], []
    for u in units:
        unit_items += u
        unit_ptr.append(len(unit_items))
    return items, indptr, unit_ptr, unit_items


@dataclass(frozen=True)
class Rule:
    """One row of a policy table: half-open ranges on B and N_max -> a plan."""

    b_lo: int
    b_hi: int
    nmax_lo: int
    nmax_hi: int
    mode: int
    num_splits: int = 1
    chunk_pages: int = 0
    flags: int = 0


def select_policy(seq_lens: Sequence[int], P: int, rules: Sequence[Rule], H_kv: int = 1) -> Tuple[int, int, int, int]:
    """Pick the execution path from (B, N_max) [PKV, Methodology 2 "Calibrated adaptive policy"].

    The first rule whose ranges hold (B, N_max) decides; no match, an empty
    batch or N_max = 0 means the single-kernel path.  Returns the plan
    (mode, num_splits, chunk_pages, flags):
      NO_SPLIT    -> (0, 1, 0, flags)
      SPLIT_S     -> C = ceil(pages_max / S), S' = ceil(pages_max / C): (1, S', C, flags)
      WORK_QUEUE  -> C from the rule,      S' = ceil(pages_max / C): (2, S', C, flags);
                     a rule with chunk_pages = 0 asks for the smallest C whose
                     queue has at most T = num_splits items (pages_max if none)
      BALANCED    -> T blocks from the rule's num_splits:              (3, T, 0, flags)
      a WORK_QUEUE rule with FLAG_DEVICE_FILL leaves the chunk to the device:
                     its fill budget T as given                         (2, T, 0, flags)
    where pages_max = ceil(N_max / P).
    """
    if P < 1:
        raise ValueError("page size must be positive")
    lens = [int(x) for x in seq_lens]
    if any(x < 0 for x in lens):
        raise ValueError("negative sequence length")
    B = len(lens)
    n_max = max(lens) if lens else 0
    pages_max = _ceil_div(n_max, P)
    chosen = None
    for r in rules:
        if r.mode not in (NO_SPLIT, SPLIT_S, WORK_QUEUE, BALANCED):
            raise ValueError("unknown mode in policy table")
        if r.mode in (SPLIT_S, BALANCED) and r.num_splits < 1:
            raise ValueError("SPLIT_S and BALANCED rules need num_splits >= 1")
        if r.mode == WORK_QUEUE and (r.chunk_pages < 0 or (r.chunk_pages == 0 and r.num_splits < 1)):
            raise ValueError("WORK_QUEUE rule needs chunk_pages >= 1, or 0 with num_splits >= 1")
        if r.flags & FLAG_DEVICE_FILL and (r.mode != WORK_QUEUE or r.chunk_pages != 0):
            raise ValueError("a device-fill rule is a WORK_QUEUE rule with chunk_pages = 0")
        if chosen is None and r.b_lo <= B < r.b_hi and r.nmax_lo <= n_max < r.nmax_hi:
            chosen = r
    if chosen is None or B == 0 or pages_max == 0:
        return (NO_SPLIT, 1, 0, 0)
    if chosen.mode == NO_SPLIT:
        return (NO_SPLIT, 1, 0, chosen.flags)
    if chosen.mode == BALANCED:
        return (BALANCED, chosen.num_splits, 0, chosen.flags)
    if chosen.flags & FLAG_DEVICE_FILL:
        return (WORK_QUEUE, chosen.num_splits, 0, chosen.flags)
    if chosen.mode == SPLIT_S:
        C = _ceil_div(pages_max, chosen.num_splits)
    elif chosen.chunk_pages > 0:
        C = chosen.chunk_pages
    else:
        # the first chunk size, counting up, whose queue fits T items
        C = pages_max
        for c in range(1, pages_max + 1):
            if fill_items(lens, H_kv, P, c) <= chosen.num_splits:
                C = c
                break
    return (chosen.mode, _ceil_div(pages_max, C), C, chosen.flags)


def fill_items(seq_lens: Sequence[int], H_kv: int, P: int, C: int) -> int:
    """Items of the compact queue at chunk size C (one per non-empty chunk of
    each (row, KV head), one empty item for a row with N_i = 0)."""
    return H_kv * sum(max(1, _ceil_div(_ceil_div(int(n), P), C)) for n in seq_lens)


def load_rules(path: str) -> List[Rule]:
    """Read a policy table (JSON: {"rules": [{b_lo, b_hi, nmax_lo, nmax_hi, mode, ...}]})."""
    import json

    with open(path) as f:
        doc = json.load(f)
    names = {"NO_SPLIT": NO_SPLIT, "SPLIT_S": SPLIT_S, "WORK_QUEUE": WORK_QUEUE, "BALANCED": BALANCED}
    out = []
    for r in doc["rules"]:
        mode = names[r["mode"]] if isinstance(r["mode"], str) else int(r["mode"])
        out.append(Rule(int(r["b_lo"]), int(r.get("b_hi", INT32_MAX)), int(r["nmax_lo"]),
                        int(r.get("nmax_hi", INT32_MAX)), mode, int(r.get("num_splits", 1)),
                        int(r.get("chunk_pages", 0)), int(r.get("flags", 0))))
    return out


@dataclass
class Counters:
    """Scheduler-induced workload counters of one decode step
    [PKV, Key contributions: "scheduler-induced workload counters"; Results:
    launch fan-out and merge-state traffic]."""

    launches: int
    work_items: int
    empty_items: int
    merge_state_bytes: int
    kv_bytes: int
    kv_bytes_streamed: int
    q_bytes: int
    out_bytes: int
    queue_bytes: int
    bucket_launches: int


def counters(seq_lens: Sequence[int], H_q: int, H_kv: int, D: int, P: int, plan) -> Counters:
    """Closed-form counters for a plan.

    launches: kernels per step (the attention kernel, plus the merge kernel
      when a split plan asks for a separate merge);
    work_items: blocks of the attention kernel; empty_items: those that only
      write the neutral state (or a zero output);
    merge_state_bytes: partial states written and read back by the merge,
      2 * slots * G * (D + 2) * 4 over every (row, head) pair with more than one slot;
    kv_bytes: K and V of the valid tokens; kv_bytes_streamed: whole pages;
    queue_bytes: items (16 B each) plus indptr (4 B per pair, +4; for BALANCED
      also 4 B per block, +4) sent to the device; none for a device-fill plan,
      whose blocks derive their items (counted at the chunk they find);
    bucket_launches: exact-length bucketing, one split and one merge launch per
      distinct non-zero length [PKV, Results: "16.00 -> 2.00 launches per step"].
    """
    mode, S, C, flags = plan
    lens = [int(x) for x in seq_lens]
    B = len(lens)
    G = H_q // H_kv
    state = G * (D + 2) * 4
    pages = [_ceil_div(n, P) for n in lens]
    if mode == NO_SPLIT:
        work = B * H_kv
        empty = H_kv * sum(1 for n in lens if n == 0)
        merge = 0
        qbytes = 0
        launches = 1
    elif mode == SPLIT_S:
        work = B * H_kv * S
        empty = H_kv * sum(S - min(S, _ceil_div(p, C)) for p in pages)
        merge = 2 * B * H_kv * S * state if S > 1 else 0
        qbytes = 0
        launches = 1 + (1 if flags & FLAG_SEPARATE_MERGE else 0)
    elif mode == WORK_QUEUE:
        device_fill = bool(flags & FLAG_DEVICE_FILL)
        if device_fill:
            # the chunk the device finds for these lengths: the fill rule with budget T = S
            pages_max = max(pages, default=0)
            C = pages_max
            for c in range(1, pages_max + 1):
                if fill_items(lens, H_kv, P, c) <= S:
                    C = c
                    break
            C = max(C, 1)
        per_pair = [max(1, _ceil_div(p, C)) for p in pages]
        work = H_kv * sum(per_pair)
        empty = H_kv * sum(1 for n in lens if n == 0)
        merge = 2 * H_kv * sum(k for k in per_pair if k > 1) * state
        qbytes = 0 if device_fill else 16 * work + 4 * (B * H_kv + 1)
        launches = 1 + (1 if flags & FLAG_SEPARATE_MERGE else 0)
    elif mode == BALANCED:
        items, indptr, _ = build_balanced_queue(lens, H_kv, P, S)
        per_pair = [indptr[k + 1] - indptr[k] for k in range(B * H_kv)]
        work = S
        empty = H_kv * sum(1 for n in lens if n == 0)
        merge = 2 * sum(k for k in per_pair if k > 1) * state
        qbytes = 16 * len(items) + 4 * (B * H_kv + 1) + 4 * (S + 1)
        launches = 1 + (1 if flags & FLAG_SEPARATE_MERGE else 0)
    else:
        raise ValueError("unknown mode")
    kv = sum(lens) * H_kv * 2 * D * 2
    kv_streamed = sum(pages) * P * H_kv * 2 * D * 2
    distinct = len({n for n in lens if n > 0})
    return Counters(launches, work, empty, merge, kv, kv_streamed, B * H_q * D * 2, B * H_q * D * 2,
                    qbytes, 2 * distinct)
