"""Device timing of decode steps (CUDA events on the launching stream).

Three protocols:
  time_steady    K steps queued back to back between one pair of events,
                 consecutive steps reading different copies of the KV pool
                 (pool_copies) so that no step finds its pages in L2.  The K
                 steps are captured once in a CUDA graph and replayed, as a
                 serving loop replays its decode step, so that the host's
                 launch rate never paces the device;
  time_interleaved  the same K steps, each after a kernel that streams
                 through HBM (a projection's stand-in), minus that kernel alone;
  time_isolated  single cold steps, L2 flushed (Flush) before each, events
                 around the step alone.
"""
from __future__ import annotations

FLUSH_BYTES = 256 << 20


class Flush:
    """Evicts L2: writes a buffer larger than L2, then reads another one, so
    the next kernel finds neither its data nor dirty lines to write back."""

    def __init__(self, torch, device):
        self.a = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
        self.b = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=device)

    def __call__(self, i=0):
        self.a.fill_(i & 255)
        self.b.sum()


def n_pool_copies(w, l2_bytes=126 << 20) -> int:
    """How many copies of the KV pool put >= 3 L2 sizes of step data between
    two reads of the same copy (at most 8; 1 when one step already exceeds that)."""
    per_step = w.kv_bytes()
    return 1 if per_step >= 3 * l2_bytes else min(8, -(-3 * l2_bytes // per_step) + 1)


def pool_copies(w, torch, l2_bytes=126 << 20):
    """The pool and n_pool_copies(w) - 1 clones of it."""
    n = n_pool_copies(w, l2_bytes)
    return [(w.k_pool, w.v_pool)] + [(w.k_pool.clone(), w.v_pool.clone()) for _ in range(n - 1)]


def time_steady(w, dp, K, W, torch, bd, copies, graph=True):
    """Device time (ms) of K back-to-back steps, one event pair, rotating pool
    copies; the steps are replayed from a CUDA graph unless graph=False."""
    lens = torch.tensor(w.seq_lens, dtype=torch.int32, device=w.q.device)
    out = torch.empty_like(w.q)

    def step(i):
        k, v = copies[i % len(copies)]
        bd.paged_decode(w.q, k, v, w.block_table, lens, w.P, w.scale, plan=dp, out=out)

    for i in range(W):
        step(i)
    torch.cuda.synchronize()
    g = None
    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(K):
                step(W + i)
        g.replay()  # untimed: the first replay also uploads the graph
        torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(st)
    if graph:
        g.replay()
    else:
        for i in range(K):
            step(W + i)
    b.record(st)
    torch.cuda.synchronize()
    del g
    if bd.workspace_status(dp) != 0:
        raise RuntimeError("device error during the timed steps")
    return a.elapsed_time(b)


def time_interleaved(w, dp, K, W, torch, bd, copies, filler_bytes=64 << 20, lens_jitter=False):
    """Device time (ms) of K decode steps that each follow another kernel, as
    in a model where attention comes after a projection: every step is a
    filler kernel streaming filler_bytes through HBM (a copy: that many bytes
    read and as many written) then the decode step, all K captured in one CUDA
    graph; the filler alone, captured and timed the same way, is subtracted.
    With lens_jitter the filler also moves every row's length by one token
    (+1, then -1 on the next step), as a serving loop's lengths change on the
    device between steps.  Returns (decode ms for the K steps, filler ms)."""
    lens = torch.tensor(w.seq_lens, dtype=torch.int32, device=w.q.device)
    out = torch.empty_like(w.q)
    src = torch.empty(filler_bytes // 2, dtype=torch.bfloat16, device=w.q.device).normal_()
    dst = torch.empty_like(src)
    up = torch.tensor([1 if n + 1 <= w.max_pages * w.P else 0 for n in w.seq_lens], dtype=torch.int32,
                      device=w.q.device)

    def filler(i):
        dst.copy_(src)
        if lens_jitter:
            if i % 2 == 0:
                lens.add_(up)
            else:
                lens.sub_(up)

    def step(i):
        k, v = copies[i % len(copies)]
        filler(i)
        bd.paged_decode(w.q, k, v, w.block_table, lens, w.P, w.scale, plan=dp, out=out)

    def timed(body):
        for i in range(W):
            body(i)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(K):
                body(W + i)
        g.replay()
        torch.cuda.synchronize()
        st = torch.cuda.current_stream()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(st)
        g.replay()
        b.record(st)
        torch.cuda.synchronize()
        del g
        return a.elapsed_time(b)

    both = timed(step)
    alone = timed(filler)
    if bd.workspace_status(dp) != 0:
        raise RuntimeError("device error during the timed steps")
    return both - alone, alone


def time_isolated(w, dp, K, W, torch, bd, flush):
    """Per-step device times (ms) of single cold steps: L2 flushed, events around the step."""
    lens = torch.tensor(w.seq_lens, dtype=torch.int32, device=w.q.device)
    out = torch.empty_like(w.q)

    def step():
        bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table, lens, w.P, w.scale, plan=dp, out=out)

    for i in range(W):
        flush(i)
        step()
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    for i in range(K):
        flush(i)
        starts[i].record(st)
        step()
        ends[i].record(st)
    torch.cuda.synchronize()
    if bd.workspace_status(dp) != 0:
        raise RuntimeError("device error during the timed steps")
    return [s.elapsed_time(e) for s, e in zip(starts, ends)]
