"""Seeded synthetic decode-step inputs.

This module only draws inputs: sequence lengths, a paged pool layout (block
table) and bf16 N(0,1) values for q, K and V.  It holds none of the attention
arithmetic, so both the CUDA path and the CPU oracle can be fed from it.

Named workloads (one decode step each; P = 16 tokens per page, bf16 values
drawn as fp32 N(0,1) and rounded to bf16, scale = 1/sqrt(head_dim)):

  tiny       B=1,  H_q=4,  H_kv=1, D=64,  N=512; 32 pages drawn from a 64-page pool
  long       B=1,  H_q=32, H_kv=8, D=128, N=32768; 2048 pages drawn from a
             4096-page pool (a random permutation); stated split S=32
  crossover  B=4,  H_q=32, H_kv=8, D=128, N_i ~ U[4096, 16384] (integers)
  mixed      B=8,  H_q=32, H_kv=8, D=128, N_i = floor(exp(U[ln 512, ln 32768])),
             moved off multiples of 16 so every row ends in a partial page
  prefix     B=64, H_q=64, H_kv=8, D=128, N_i = floor(exp(U[ln 256, ln 131072]));
             rows 0-15 share their first 128 physical pages (a 2048-token
             prefix) and have N_i >= 2049
  bimodal, uniform, zipf
             B=8, H_q=32, H_kv=8, D=128 traces in the style of the pages'
             study (their parameters are not published; see make())
  long_g1, long_g2, long_g8, long_g16
             the long context with H_q = 8, 16, 64, 128 query heads over
             the same 8 KV heads (G = 1, 2, 8, 16): the same K/V bytes, for
             measuring what the group size costs
  prefix_small
             the prefix workload's shape (B=64, G=8, 16 rows sharing a
             128-page prefix) with lengths log-uniform in [256, 16384], small
             enough for a profiler capture

For the last three the pool holds 1.25x the pages the rows need; a random
permutation of the pool is dealt to the rows in order, so every row's pages
are scattered.  Seeds: 20260622 calibrates the policy, 20260623 is reported.

With poison=True every pool page no row uses, every slot past a row's last
token in its tail page (unless another row that shares the page reads that
slot as one of its own tokens), and every block-table entry past a row's last
page (pointed at a poisoned page) holds bf16 NaN, so any read outside a row's
real tokens shows up in the output.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import torch

SEED_CALIBRATE = 20260622
SEED_REPORT = 20260623
PAGE = 16

NAMES = ("tiny", "long", "crossover", "mixed", "prefix", "bimodal", "uniform", "zipf", "long_g1", "long_g2",
         "long_g8", "long_g16", "prefix_small")


@dataclass
class Workload:
    name: str
    B: int
    H_q: int
    H_kv: int
    D: int
    P: int
    seq_lens: List[int]
    num_pages: int
    block_table: torch.Tensor  # int32 [B][max_pages]
    q: torch.Tensor            # bf16 [B][H_q][D]
    k_pool: torch.Tensor       # bf16 [num_pages][H_kv][P][D] ("HND") or [num_pages][P][H_kv][D] ("NHD")
    v_pool: torch.Tensor
    scale: float
    layout: str = "HND"
    split_s: Optional[int] = None
    shared_prefix_pages: int = 0
    shared_rows: int = 0
    seed: int = SEED_REPORT
    meta: dict = field(default_factory=dict)

    @property
    def G(self) -> int:
        return self.H_q // self.H_kv

    @property
    def max_pages(self) -> int:
        return int(self.block_table.shape[1])

    @property
    def seq_lens_tensor(self) -> torch.Tensor:
        return torch.tensor(self.seq_lens, dtype=torch.int32)

    def kv_bytes(self, unique: bool = False) -> int:
        """K+V bytes of the valid tokens (2 tensors * 2 bytes * D per token and KV head).
        unique=True counts the shared prefix pages once."""
        tokens = sum(self.seq_lens)
        if unique and self.shared_rows > 1:
            tokens -= (self.shared_rows - 1) * self.shared_prefix_pages * self.P
        return tokens * self.H_kv * 2 * self.D * 2

    def algorithmic_bytes(self, unique: bool = False) -> int:
        """Bytes a decode step must move: valid K/V + q + out."""
        return self.kv_bytes(unique) + 2 * self.B * self.H_q * self.D * 2


def _log_uniform(g: torch.Generator, n: int, lo: int, hi: int) -> List[int]:
    u = torch.rand(n, generator=g, dtype=torch.float64)
    return [int(math.floor(math.exp(math.log(lo) + float(x) * (math.log(hi) - math.log(lo))))) for x in u]


def _pages(n: int, P: int) -> int:
    return -(-n // P)


def make(name: str, seed: int = SEED_REPORT, device="cpu", poison: bool = False,
         layout: str = "HND", q_scale: float = 1.0) -> Workload:
    """One of the named workloads above."""
    g = torch.Generator("cpu").manual_seed(seed)
    split_s = None
    if name == "tiny":
        B, H_q, H_kv, D = 1, 4, 1, 64
        lens = [512]
        num_pages = 64
        perm = torch.randperm(num_pages, generator=g)
        tables = [perm[:32].tolist()]
        shared_pages = shared_rows = 0
    elif name == "long" or name.startswith("long_g"):
        B, H_kv, D = 1, 8, 128
        H_q = H_kv * (int(name[6:]) if name.startswith("long_g") else 4)
        lens = [32768]
        num_pages = 4096
        perm = torch.randperm(num_pages, generator=g)
        tables = [perm[:2048].tolist()]
        split_s = 32
        shared_pages = shared_rows = 0
    elif name in ("crossover", "mixed"):
        B, H_q, H_kv, D = (4 if name == "crossover" else 8), 32, 8, 128
        if name == "crossover":
            lens = torch.randint(4096, 16384 + 1, (B,), generator=g).tolist()
        else:
            lens = [n - 1 if n % PAGE == 0 else n for n in _log_uniform(g, B, 512, 32768)]
        return _finish(name, seed, device, poison, layout, q_scale, g, B, H_q, H_kv, D, lens)
    elif name in ("bimodal", "uniform", "zipf"):
        # B=8 traces shaped like the pages' study traces, whose parameters are
        # not published; these are generated and stated here:
        #   bimodal  4 rows U[256, 1024] and 4 rows U[16384, 32768], shuffled
        #   uniform  8 rows U[512, 32768]
        #   zipf     N_k = 32768 / k (k = 1..8) times U[0.9, 1.1]
        B, H_q, H_kv, D = 8, 32, 8, 128
        if name == "bimodal":
            lens = (torch.randint(256, 1024 + 1, (4,), generator=g).tolist() +
                    torch.randint(16384, 32768 + 1, (4,), generator=g).tolist())
            order = torch.randperm(B, generator=g).tolist()
            lens = [lens[k] for k in order]
        elif name == "uniform":
            lens = torch.randint(512, 32768 + 1, (B,), generator=g).tolist()
        else:
            jitter = (0.9 + 0.2 * torch.rand(B, generator=g, dtype=torch.float64)).tolist()
            lens = [max(1, int(32768 / (k + 1) * jitter[k])) for k in range(B)]
        return _finish(name, seed, device, poison, layout, q_scale, g, B, H_q, H_kv, D, lens)
    elif name in ("prefix", "prefix_small"):
        B, H_q, H_kv, D = 64, 64, 8, 128
        lens = _log_uniform(g, B, 256, 131072 if name == "prefix" else 16384)
        shared_rows, shared_pages = 16, 128
        lens = [max(n, shared_pages * PAGE + 1) if i < shared_rows else n for i, n in enumerate(lens)]
        return _finish(name, seed, device, poison, layout, q_scale, g, B, H_q, H_kv, D, lens,
                       shared_rows=shared_rows, shared_pages=shared_pages)
    else:
        raise ValueError(f"unknown workload {name!r}; known: {NAMES}")
    return _materialise(name, seed, device, poison, layout, q_scale, g, B, H_q, H_kv, D, lens, num_pages,
                        tables, split_s, shared_pages, shared_rows)


def make_custom(seq_lens: Sequence[int], H_q: int, H_kv: int, D: int, seed: int = SEED_REPORT,
                device="cpu", poison: bool = False, layout: str = "HND", q_scale: float = 1.0,
                shared_rows: int = 0, shared_pages: int = 0, slack: float = 1.25,
                name: str = "custom") -> Workload:
    """Any batch: pages scattered over a pool with `slack` x the needed pages."""
    g = torch.Generator("cpu").manual_seed(seed)
    return _finish(name, seed, device, poison, layout, q_scale, g, len(seq_lens), H_q, H_kv, D,
                   [int(n) for n in seq_lens], shared_rows=shared_rows, shared_pages=shared_pages,
                   slack=slack)


def _finish(name, seed, device, poison, layout, q_scale, g, B, H_q, H_kv, D, lens,
            shared_rows=0, shared_pages=0, slack=1.25):
    need = [_pages(n, PAGE) for n in lens]
    unique = shared_pages + sum(max(0, p - (shared_pages if i < shared_rows else 0)) for i, p in enumerate(need))
    num_pages = max(1, int(math.ceil(slack * unique)))
    perm = torch.randperm(num_pages, generator=g).tolist()
    shared = perm[:shared_pages]
    off = shared_pages
    tables = []
    for i, p in enumerate(need):
        if i < shared_rows:
            own = max(0, p - shared_pages)
            tables.append(shared[:min(p, shared_pages)] + perm[off:off + own])
            off += own
        else:
            tables.append(perm[off:off + p])
            off += p
    return _materialise(name, seed, device, poison, layout, q_scale, g, B, H_q, H_kv, D, lens, num_pages,
                        tables, None, shared_pages, shared_rows)


def _materialise(name, seed, device, poison, layout, q_scale, g, B, H_q, H_kv, D, lens, num_pages, tables,
                 split_s, shared_pages, shared_rows) -> Workload:
    P = PAGE
    max_pages = max([len(t) for t in tables] + [1])
    used = set(x for t in tables for x in t)
    unused = [x for x in range(num_pages) if x not in used]
    filler = unused[0] if (poison and unused) else 0
    bt = torch.full((B, max_pages), filler, dtype=torch.int32)
    for i, t in enumerate(tables):
        if t:
            bt[i, :len(t)] = torch.tensor(t, dtype=torch.int32)
    dev = torch.device(device)
    if dev.type == "cuda":
        gd = torch.Generator(dev).manual_seed(seed)
    else:
        gd = g
    q = (torch.randn((B, H_q, D), generator=gd, device=dev, dtype=torch.float32) * q_scale).to(torch.bfloat16)
    shape = (num_pages, H_kv, P, D)
    k_pool = torch.randn(shape, generator=gd, device=dev, dtype=torch.float32).to(torch.bfloat16)
    v_pool = torch.randn(shape, generator=gd, device=dev, dtype=torch.float32).to(torch.bfloat16)
    if poison:
        nan = float("nan")
        if unused:
            idx = torch.tensor(unused, dtype=torch.long, device=dev)
            k_pool[idx] = nan
            v_pool[idx] = nan
        # a row's partial last page is poisoned past its last token unless another
        # row reads that page further (a shared page one row ends inside)
        covered = {}
        for i, n in enumerate(lens):
            for j, page in enumerate(tables[i]):
                covered[page] = max(covered.get(page, 0), min(P, n - j * P))
        for i, n in enumerate(lens):
            if n % P and tables[i]:
                last = tables[i][-1]
                if covered[last] > n % P:
                    continue
                k_pool[last, :, n % P:, :] = nan
                v_pool[last, :, n % P:, :] = nan
    if layout == "NHD":
        k_pool = k_pool.permute(0, 2, 1, 3).contiguous()
        v_pool = v_pool.permute(0, 2, 1, 3).contiguous()
    elif layout != "HND":
        raise ValueError(layout)
    return Workload(name, B, H_q, H_kv, D, P, list(lens), num_pages, bt.to(dev), q, k_pool, v_pool,
                    1.0 / math.sqrt(D), layout, split_s, shared_pages, shared_rows, seed)
