"""ctypes binding of libpkv.so (include/pkv.h): argument marshalling only.

Every step of the decode path (policy, queue, kernels, merge) runs inside the
C-ABI library; this module converts torch tensors to raw pointers, allocates
caller-owned buffers with torch and passes torch's current CUDA stream.  If
the library is missing or cannot be loaded, every call raises PkvError.
"""
from __future__ import annotations

import ctypes
import json
import os
import weakref
from dataclasses import dataclass
from typing import List, Optional, Sequence

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpkv.so")

NO_SPLIT, SPLIT_S, WORK_QUEUE, BALANCED = 0, 1, 2, 3
FLAG_SEPARATE_MERGE, FLAG_NO_PDL, FLAG_DEEP_RING, FLAG_CLUSTER_MERGE, FLAG_PDL_EARLY = 1, 2, 4, 8, 16
FLAG_DEVICE_FILL = 32
FLAG_SHARED_PREFIX = 64
FILL_MAX_ROWS = 1024  # rows a device-fill plan can plan for on the device
INT32_MAX = 2**31 - 1
_MODE_NAMES = {"NO_SPLIT": NO_SPLIT, "SPLIT_S": SPLIT_S, "WORK_QUEUE": WORK_QUEUE, "BALANCED": BALANCED}

c_i32, c_i64, c_p, c_sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t


class PkvError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        name = _lib.pkv_status_string(status).decode() if _lib is not None else str(status)
        super().__init__(f"{what}: {name} ({status})" if what else f"{name} ({status})")


class Shape(ctypes.Structure):
    _fields_ = [("B", c_i32), ("H_q", c_i32), ("H_kv", c_i32), ("head_dim", c_i32), ("page_size", c_i32),
                ("max_pages_per_seq", c_i32), ("num_pool_pages", c_i32), ("reserved", c_i32),
                ("kv_stride_page", c_i64), ("kv_stride_head", c_i64), ("kv_stride_token", c_i64)]


class Plan(ctypes.Structure):
    _fields_ = [("mode", c_i32), ("num_splits", c_i32), ("chunk_pages", c_i32), ("flags", c_i32)]

    def tuple(self):
        return (self.mode, self.num_splits, self.chunk_pages, self.flags)

    def __repr__(self):
        return f"Plan{self.tuple()}"


class WorkItem(ctypes.Structure):
    _fields_ = [("row", c_i32), ("kv_head", c_i32), ("tok_begin", c_i32), ("tok_end", c_i32)]


class Rule(ctypes.Structure):
    _fields_ = [("b_lo", c_i32), ("b_hi", c_i32), ("nmax_lo", c_i32), ("nmax_hi", c_i32), ("mode", c_i32),
                ("num_splits", c_i32), ("chunk_pages", c_i32), ("flags", c_i32)]

    def tuple(self):
        return tuple(getattr(self, f) for f, _ in self._fields_)


class Counters(ctypes.Structure):
    _fields_ = [(n, c_i64) for n in ("launches", "work_items", "empty_items", "merge_state_bytes", "kv_bytes",
                                     "kv_bytes_streamed", "q_bytes", "out_bytes", "queue_bytes",
                                     "bucket_launches")]

    def as_dict(self):
        return {f: int(getattr(self, f)) for f, _ in self._fields_}


class HostTiming(ctypes.Structure):
    """Where one pkv_decode_host call's time went (pkv_host_timing), in microseconds."""
    _fields_ = [(n, ctypes.c_double) for n in ("host_plan_us", "host_enqueue_us", "host_wait_us", "host_unpack_us",
                                               "dev_h2d_us", "dev_kernel_us", "dev_d2h_us", "host_events_us")]

    def as_dict(self):
        return {f: float(getattr(self, f)) for f, _ in self._fields_}


class HostCall(ctypes.Structure):
    """pkv_host_call: the arguments of pkv_decode_host as one parameter block."""
    _fields_ = [("q_host", c_p), ("block_table_host", c_p), ("seq_lens_host", c_p), ("out_host", c_p),
                ("k_pool", c_p), ("v_pool", c_p), ("scale", ctypes.c_float), ("shape", c_p), ("rules", c_p),
                ("n_rules", c_i32), ("device_buffer", c_p), ("device_buffer_bytes", c_sz), ("host_staging", c_p),
                ("host_staging_bytes", c_sz), ("stream", c_p), ("plan_out", c_p), ("timing", c_p)]


_lib = None

# (name, restype, argtypes) of every function include/pkv.h declares
SIGNATURES = [
    ("pkv_version", ctypes.c_char_p, []),
    ("pkv_status_string", ctypes.c_char_p, [ctypes.c_int]),
    ("pkv_default_policy", ctypes.c_int, [c_p, c_i32, c_p]),
    ("pkv_select_policy", ctypes.c_int, [c_p, c_p, c_p, c_i32, c_p]),
    ("pkv_work_queue_size", ctypes.c_int, [c_p, c_p, c_i32, c_p]),
    ("pkv_build_work_queue", ctypes.c_int, [c_p, c_p, c_i32, c_p, c_i32, c_p, c_p]),
    ("pkv_balanced_queue_size", ctypes.c_int, [c_p, c_p, c_i32, c_p]),
    ("pkv_build_balanced_queue", ctypes.c_int, [c_p, c_p, c_i32, c_p, c_i32, c_p, c_p]),
    ("pkv_balanced_queue_capacity", ctypes.c_int, [c_p, c_i32, c_p]),
    ("pkv_build_balanced_queue_device", ctypes.c_int, [c_p, c_p, c_i32, c_p, c_i32, c_p, c_p, c_p]),
    ("pkv_fill_queue_capacity", ctypes.c_int, [c_p, c_i32, c_p]),
    ("pkv_build_fill_queue_device", ctypes.c_int, [c_p, c_p, c_i32, c_p, c_i32, c_p, c_p, c_p]),
    ("pkv_prefix_queue_size", ctypes.c_int, [c_p, c_p, c_p, c_i32, c_i32, c_p, c_p]),
    ("pkv_build_prefix_queue", ctypes.c_int, [c_p, c_p, c_p, c_i32, c_i32, c_p, c_i32, c_p, c_i32, c_p, c_p]),
    ("pkv_plan_counters", ctypes.c_int, [c_p, c_p, c_p, c_p]),
    ("pkv_workspace_bytes", ctypes.c_int, [c_p, c_p, c_i32, c_p]),
    ("pkv_workspace_init", ctypes.c_int, [c_p, c_sz, c_p]),
    ("pkv_workspace_status", ctypes.c_int, [c_p, c_p, c_p]),
    ("pkv_selftest_wait_timeout", ctypes.c_int, [c_p, c_sz, ctypes.c_uint32, c_p]),
    ("pkv_paged_decode", ctypes.c_int,
     [c_p, c_p, c_p, c_p, c_p, c_i32, ctypes.c_float, c_p, c_p, c_p, c_p, c_p, c_i32, c_p, c_sz, c_p]),
    ("pkv_paged_decode_noalloc", ctypes.c_int,
     [c_p, c_p, c_p, c_p, c_p, c_i32, ctypes.c_float, c_p, c_p, c_p, c_p, c_p, c_i32, c_p]),
    ("pkv_noalloc_status", ctypes.c_int, [c_p, c_p]),
    ("pkv_decode_host_bytes", ctypes.c_int, [c_p, c_p, c_p, c_i32, c_p, c_p]),
    ("pkv_decode_host", ctypes.c_int,
     [c_p, c_p, c_p, c_p, c_p, c_p, ctypes.c_float, c_p, c_p, c_i32, c_p, c_sz, c_p, c_sz, c_p, c_p]),
    ("pkv_decode_host_timed", ctypes.c_int,
     [c_p, c_p, c_p, c_p, c_p, c_p, ctypes.c_float, c_p, c_p, c_i32, c_p, c_sz, c_p, c_sz, c_p, c_p, c_p]),
    ("pkv_decode_host_call", ctypes.c_int, [c_p]),
    ("pkv_decode_host_replays", ctypes.c_int64, []),
]


def lib(path: Optional[str] = None):
    """Load libpkv.so (built by paged_kv_gqa_17_b200.build); raise if it is missing.
    With `path`, load that build instead and make it the one every later call uses."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise PkvError(-4, f"{p} is missing; build it with `python -m paged_kv_gqa_17_b200.build`")
    handle = ctypes.CDLL(p)
    for name, res, args in SIGNATURES:
        fn = getattr(handle, name)
        fn.restype = res
        fn.argtypes = args
    _lib = handle
    return handle


def _check(rc: int, what: str):
    if rc != 0:
        raise PkvError(rc, what)


def _ref(x):
    return ctypes.byref(x) if x is not None else None


def _lens_array(seq_lens) -> ctypes.Array:
    if isinstance(seq_lens, torch.Tensor):
        seq_lens = seq_lens.detach().cpu().tolist()
    vals = [int(v) for v in seq_lens]
    return (c_i32 * max(1, len(vals)))(*vals), len(vals)


def make_shape(B: int, H_q: int, H_kv: int, head_dim: int, page_size: int, max_pages: int, num_pool_pages: int,
               layout: str = "HND") -> Shape:
    P, D = page_size, head_dim
    if layout == "HND":
        strides = (H_kv * P * D, P * D, D)
    elif layout == "NHD":
        strides = (P * H_kv * D, D, H_kv * D)
    else:
        raise ValueError(layout)
    return Shape(B, H_q, H_kv, D, P, max_pages, num_pool_pages, 0, *strides)


def shape_of(q: torch.Tensor, k_pool: torch.Tensor, block_table: torch.Tensor, layout: str = "HND",
             v_pool: Optional[torch.Tensor] = None) -> Shape:
    """Shape of a decode step from q [B][H_q][D], a pool and block_table [B][max_pages].

    The pool strides are the tensor's own (in elements), so a pool that is a
    view into a larger cache needs no copy: K and V halves of one combined
    cache ([pages][2][H_kv][P][D] gives k = kv[:, 0], v = kv[:, 1]), or pages
    padded past their last row.  The head_dim axis must be contiguous; with
    `v_pool`, its shape and strides must equal k_pool's (one set of strides
    serves both pools).  Axes of extent 1 take the packed stride, which is
    never used to address an element."""
    if k_pool.dim() != 4:
        raise ValueError(f"k_pool must be 4-D, got shape {tuple(k_pool.shape)}")
    if v_pool is not None and (tuple(v_pool.shape) != tuple(k_pool.shape) or v_pool.stride() != k_pool.stride()):
        raise ValueError("k_pool and v_pool must have the same shape and strides")
    B, H_q, D = (int(x) for x in q.shape)
    if layout == "HND":
        (pages, H_kv, P, _), (sp, sh, st, sd) = k_pool.shape, k_pool.stride()
    elif layout == "NHD":
        (pages, P, H_kv, _), (sp, st, sh, sd) = k_pool.shape, k_pool.stride()
    else:
        raise ValueError(layout)
    if sd != 1 and D > 1:
        raise ValueError("the pool's head_dim axis must be contiguous (stride 1)")
    s = make_shape(B, H_q, int(H_kv), D, int(P), int(block_table.shape[1]), int(pages), layout)
    if pages > 1:
        s.kv_stride_page = sp
    if H_kv > 1:
        s.kv_stride_head = sh
    if P > 1:
        s.kv_stride_token = st
    return s


_DECODE_DTYPES = (torch.bfloat16, torch.bfloat16, torch.bfloat16, torch.bfloat16, torch.int32, torch.int32)


def _check_decode_tensors(q, k_pool, v_pool, block_table, seq_lens, out, shape: Shape):
    """Reject tensors whose type, layout or device differs from what the
    pointers passed to the library are taken to address.  One combined test
    (a few microseconds) passes every well-formed call; only a failing call
    runs the itemised checks that name the problem."""
    dev = q.get_device()
    kst = k_pool.stride()
    if ((q.dtype, out.dtype, k_pool.dtype, v_pool.dtype, block_table.dtype, seq_lens.dtype) == _DECODE_DTYPES
            and dev >= 0 and out.get_device() == dev and k_pool.get_device() == dev
            and v_pool.get_device() == dev and block_table.get_device() == dev and seq_lens.get_device() == dev
            and q.is_contiguous() and out.is_contiguous() and block_table.is_contiguous()
            and seq_lens.is_contiguous()
            and q.shape == (shape.B, shape.H_q, shape.head_dim) and out.shape == q.shape
            and block_table.shape == (shape.B, shape.max_pages_per_seq) and seq_lens.numel() >= shape.B
            and len(kst) == 4 and v_pool.stride() == kst and v_pool.shape == k_pool.shape
            and k_pool.shape[0] >= shape.num_pool_pages
            and (k_pool.shape[0] <= 1 or kst[0] == shape.kv_stride_page)
            and (kst[3] == 1 or shape.head_dim <= 1)):
        return
    _diagnose_decode_tensors(q, k_pool, v_pool, block_table, seq_lens, out, shape)
    raise ValueError("tensors do not match the plan's shape")


def _diagnose_decode_tensors(q, k_pool, v_pool, block_table, seq_lens, out, shape: Shape):
    for name, t, dt in (("q", q, torch.bfloat16), ("out", out, torch.bfloat16), ("k_pool", k_pool, torch.bfloat16),
                        ("v_pool", v_pool, torch.bfloat16), ("block_table", block_table, torch.int32),
                        ("seq_lens", seq_lens, torch.int32)):
        if t.dtype != dt:
            raise TypeError(f"{name} must be {dt}, got {t.dtype}")
    for name, t in (("q", q), ("out", out), ("block_table", block_table), ("seq_lens", seq_lens)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    want = (shape.B, shape.H_q, shape.head_dim)
    if tuple(q.shape) != want or tuple(out.shape) != want:
        raise ValueError(f"q and out must be {list(want)}, got {list(q.shape)} and {list(out.shape)}")
    if tuple(block_table.shape) != (shape.B, shape.max_pages_per_seq):
        raise ValueError(f"block_table must be [{shape.B}][{shape.max_pages_per_seq}], got {list(block_table.shape)}")
    if seq_lens.numel() < shape.B:
        raise ValueError(f"seq_lens holds {seq_lens.numel()} lengths for {shape.B} rows")
    if k_pool.dim() != 4 or tuple(v_pool.shape) != tuple(k_pool.shape) or v_pool.stride() != k_pool.stride():
        raise ValueError("k_pool and v_pool must be 4-D with the same shape and strides")
    if k_pool.shape[0] < shape.num_pool_pages or (k_pool.shape[0] > 1 and k_pool.stride(0) != shape.kv_stride_page):
        raise ValueError("the pools' pages differ from the plan's shape (page count or page stride)")
    if k_pool.stride(-1) != 1 and shape.head_dim > 1:
        raise ValueError("the pools' head_dim axis must be contiguous (stride 1)")
    dev = q.device
    if dev.type != "cuda":
        raise ValueError(f"q must be on a CUDA device, not {dev}")
    for name, t in (("out", out), ("k_pool", k_pool), ("v_pool", v_pool), ("block_table", block_table),
                    ("seq_lens", seq_lens)):
        if t.device != dev:
            raise ValueError(f"{name} is on {t.device}, q on {dev}")


def _check_host_call(q_host, block_table_host, seq_lens_host, out_host, k_pool, v_pool, shape: Shape,
                     device_index: int):
    """The tensors of a pkv_decode_host call: host q / out (bf16 [B][H_q][D]),
    host table (int32 [B][max_pages]) and lengths (int32, >= B), contiguous;
    pools on the decoder's CUDA device with the shape's page count and strides."""
    n_q = shape.B * shape.H_q * shape.head_dim
    for name, t, dt, n in (("q_host", q_host, torch.bfloat16, n_q), ("out_host", out_host, torch.bfloat16, n_q),
                           ("block_table_host", block_table_host, torch.int32, shape.B * shape.max_pages_per_seq),
                           ("seq_lens_host", seq_lens_host, torch.int32, None)):
        if t.dtype != dt:
            raise TypeError(f"{name} must be {dt}, got {t.dtype}")
        if t.device.type != "cpu":
            raise ValueError(f"{name} must be a host tensor, not on {t.device}")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if n is not None and t.numel() != n:
            raise ValueError(f"{name} holds {t.numel()} elements, the shape needs {n}")
    if seq_lens_host.numel() < shape.B:
        raise ValueError(f"seq_lens_host holds {seq_lens_host.numel()} lengths for {shape.B} rows")
    for name, t in (("k_pool", k_pool), ("v_pool", v_pool)):
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be torch.bfloat16, got {t.dtype}")
        if t.get_device() != device_index:
            raise ValueError(f"{name} must be on the decoder's device cuda:{device_index}")
    if k_pool.dim() != 4 or tuple(v_pool.shape) != tuple(k_pool.shape) or v_pool.stride() != k_pool.stride():
        raise ValueError("k_pool and v_pool must be 4-D with the same shape and strides")
    if k_pool.shape[0] < shape.num_pool_pages or (k_pool.shape[0] > 1 and k_pool.stride(0) != shape.kv_stride_page):
        raise ValueError("the pools' pages differ from the shape (page count or page stride)")
    if k_pool.stride(-1) != 1 and shape.head_dim > 1:
        raise ValueError("the pools' head_dim axis must be contiguous (stride 1)")


def rules_array(rules: Optional[Sequence]) -> tuple:
    """(ctypes array or None, count) from Rule structs, tuples or dicts."""
    if rules is None:
        return None, 0
    out = []
    for r in rules:
        if isinstance(r, Rule):
            out.append(r)
        elif isinstance(r, dict):
            mode = _MODE_NAMES[r["mode"]] if isinstance(r["mode"], str) else int(r["mode"])
            out.append(Rule(int(r["b_lo"]), int(r.get("b_hi", INT32_MAX)), int(r["nmax_lo"]),
                            int(r.get("nmax_hi", INT32_MAX)), mode, int(r.get("num_splits", 1)),
                            int(r.get("chunk_pages", 0)), int(r.get("flags", 0))))
        else:
            out.append(Rule(*[int(v) for v in r]))
    return (Rule * max(1, len(out)))(*out), len(out)


def load_rules(path: str) -> List[Rule]:
    """Read a policy table JSON ({"rules": [...]}) into Rule structs."""
    with open(path) as f:
        doc = json.load(f)
    arr, n = rules_array(doc["rules"])
    return [arr[i] for i in range(n)]


def default_rules() -> List[Rule]:
    L = lib()
    n = c_i32(0)
    L.pkv_default_policy(None, 0, ctypes.byref(n))
    arr = (Rule * max(1, n.value))()
    _check(L.pkv_default_policy(arr, n.value, ctypes.byref(n)), "pkv_default_policy")
    return [arr[i] for i in range(n.value)]


def select_policy(seq_lens_host, shape: Shape, rules=None) -> Plan:
    L = lib()
    lens, _ = _lens_array(seq_lens_host)
    arr, n = rules_array(rules)
    plan = Plan()
    _check(L.pkv_select_policy(lens, ctypes.byref(shape), arr, n, ctypes.byref(plan)), "pkv_select_policy")
    return plan


def build_work_queue(seq_lens_host, shape: Shape, chunk_pages: int):
    """-> (items int32 tensor [n][4] on the CPU, indptr int32 tensor [B*H_kv + 1])."""
    L = lib()
    lens, _ = _lens_array(seq_lens_host)
    n = c_i32(0)
    _check(L.pkv_work_queue_size(lens, ctypes.byref(shape), chunk_pages, ctypes.byref(n)), "pkv_work_queue_size")
    items = torch.zeros((max(1, n.value), 4), dtype=torch.int32)
    indptr = torch.zeros(shape.B * shape.H_kv + 1, dtype=torch.int32)
    _check(L.pkv_build_work_queue(lens, ctypes.byref(shape), chunk_pages, items.data_ptr(), n.value,
                                  indptr.data_ptr(), ctypes.byref(n)), "pkv_build_work_queue")
    return items[:n.value], indptr


def build_balanced_queue(seq_lens_host, shape: Shape, n_blocks: int):
    """-> (items int32 [n][4], indptr int32 [B*H_kv + 1 + n_blocks + 1]: pair offsets, then block offsets)."""
    L = lib()
    lens, _ = _lens_array(seq_lens_host)
    n = c_i32(0)
    _check(L.pkv_balanced_queue_size(lens, ctypes.byref(shape), n_blocks, ctypes.byref(n)),
           "pkv_balanced_queue_size")
    items = torch.zeros((max(1, n.value), 4), dtype=torch.int32)
    indptr = torch.zeros(shape.B * shape.H_kv + 1 + n_blocks + 1, dtype=torch.int32)
    _check(L.pkv_build_balanced_queue(lens, ctypes.byref(shape), n_blocks, items.data_ptr(), n.value,
                                      indptr.data_ptr(), ctypes.byref(n)), "pkv_build_balanced_queue")
    return items[:n.value], indptr


def build_prefix_queue(seq_lens_host, block_table_host, shape: Shape, chunk_pages: int, max_members: int):
    """-> (items int32 [n][4], indptr int32: pair offsets [B*H_kv + 1], unit offsets
    [n_units + 1], the units' member item indices [n]; n_units).  The queue that
    stages shared prefix pages once for several rows (pkv_build_prefix_queue)."""
    L = lib()
    lens, _ = _lens_array(seq_lens_host)
    bt = torch.as_tensor(block_table_host, dtype=torch.int32).cpu().contiguous()
    n, u = c_i32(0), c_i32(0)
    _check(L.pkv_prefix_queue_size(lens, bt.data_ptr(), ctypes.byref(shape), chunk_pages, max_members,
                                   ctypes.byref(n), ctypes.byref(u)), "pkv_prefix_queue_size")
    items = torch.zeros((max(1, n.value), 4), dtype=torch.int32)
    n_ptr = shape.B * shape.H_kv + 1 + u.value + 1 + n.value
    indptr = torch.zeros(n_ptr, dtype=torch.int32)
    _check(L.pkv_build_prefix_queue(lens, bt.data_ptr(), ctypes.byref(shape), chunk_pages, max_members,
                                    items.data_ptr(), n.value, indptr.data_ptr(), n_ptr, ctypes.byref(n),
                                    ctypes.byref(u)), "pkv_build_prefix_queue")
    return items[:n.value], indptr, int(u.value)


def balanced_queue_capacity(shape: Shape, n_blocks: int) -> int:
    L = lib()
    n = c_i32(0)
    _check(L.pkv_balanced_queue_capacity(ctypes.byref(shape), n_blocks, ctypes.byref(n)), "pkv_balanced_queue_capacity")
    return int(n.value)


def build_balanced_queue_device(seq_lens: torch.Tensor, shape: Shape, n_blocks: int, items: torch.Tensor,
                                indptr: torch.Tensor, workspace: torch.Tensor, stream=None) -> None:
    """pkv_build_balanced_queue_device: the balanced queue built on the GPU from
    device lengths into `items` / `indptr` (see include/pkv.h)."""
    L = lib()
    _check(L.pkv_build_balanced_queue_device(seq_lens.data_ptr(), ctypes.byref(shape), n_blocks, items.data_ptr(),
                                             int(items.shape[0]), indptr.data_ptr(), workspace.data_ptr(),
                                             _stream_ptr(stream)), "pkv_build_balanced_queue_device")


def fill_queue_capacity(shape: Shape, n_blocks: int) -> int:
    L = lib()
    n = c_i32(0)
    _check(L.pkv_fill_queue_capacity(ctypes.byref(shape), n_blocks, ctypes.byref(n)), "pkv_fill_queue_capacity")
    return int(n.value)


def build_fill_queue_device(seq_lens: torch.Tensor, shape: Shape, n_blocks: int, items: torch.Tensor,
                            indptr: torch.Tensor, workspace: torch.Tensor, stream=None) -> None:
    """pkv_build_fill_queue_device: the queue whose chunk fills one wave of
    n_blocks blocks, built on the GPU from device lengths (see include/pkv.h)."""
    L = lib()
    _check(L.pkv_build_fill_queue_device(seq_lens.data_ptr(), ctypes.byref(shape), n_blocks, items.data_ptr(),
                                         int(items.shape[0]), indptr.data_ptr(), workspace.data_ptr(),
                                         _stream_ptr(stream)), "pkv_build_fill_queue_device")


def plan_counters(seq_lens_host, shape: Shape, plan: Plan) -> dict:
    L = lib()
    lens, _ = _lens_array(seq_lens_host)
    c = Counters()
    _check(L.pkv_plan_counters(lens, ctypes.byref(shape), ctypes.byref(plan), ctypes.byref(c)), "pkv_plan_counters")
    return c.as_dict()


def workspace_bytes(shape: Shape, plan: Plan, n_items: int = 0) -> int:
    L = lib()
    b = c_sz(0)
    _check(L.pkv_workspace_bytes(ctypes.byref(shape), ctypes.byref(plan), n_items, ctypes.byref(b)),
           "pkv_workspace_bytes")
    return int(b.value)


def _stream_ptr(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


@dataclass
class DecodePlan:
    """Everything a decode step needs besides the tensors: the plan, the queue
    on the device (WORK_QUEUE, BALANCED) and a zeroed workspace.  Reusable for
    every step with the same sequence lengths and shape; with device_queue
    the queue comes from the device lengths at every step (built by a kernel
    of its own, or derived by each decode block under PKV_FLAG_DEVICE_FILL),
    so the plan serves any lengths up to the shape's maximum."""

    shape: Shape
    plan: Plan
    items: Optional[torch.Tensor]
    indptr: Optional[torch.Tensor]
    n_items: int
    workspace: torch.Tensor
    counters: dict
    device_queue: bool = False
    fill_blocks: int = 0  # device queue of a WORK_QUEUE plan: the wave it fills


def prefix_counters(seq_lens_host, shape: Shape, items: torch.Tensor, indptr: torch.Tensor, n_units: int,
                    flags: int = 0) -> dict:
    """Workload counters of a prefix-sharing plan, counted from its queue: one
    block per unit, a unit's pages streamed once for all its members."""
    lens = [int(n) for n in (seq_lens_host.tolist() if isinstance(seq_lens_host, torch.Tensor) else seq_lens_host)]
    B, H_kv, D, P = shape.B, shape.H_kv, shape.head_dim, shape.page_size
    G = shape.H_q // H_kv
    pairs = B * H_kv
    ptr = indptr.tolist()
    it = items.tolist()
    uptr = ptr[pairs + 1:pairs + 2 + n_units]
    uitems = ptr[pairs + 2 + n_units:]
    per_pair = [ptr[k + 1] - ptr[k] for k in range(pairs)]
    streamed = 0
    for u in range(n_units):
        _, _, tb, te = it[uitems[uptr[u]]]
        streamed += (-(-te // P) - tb // P) if te > tb else 0
    return {"launches": 1 + (1 if flags & FLAG_SEPARATE_MERGE else 0), "work_items": n_units,
            "empty_items": H_kv * sum(1 for n in lens if n == 0),
            "merge_state_bytes": 2 * sum(k for k in per_pair if k > 1) * G * (D + 2) * 4,
            "kv_bytes": sum(lens) * H_kv * 2 * D * 2, "kv_bytes_streamed": streamed * P * 2 * D * 2,
            "q_bytes": B * shape.H_q * D * 2, "out_bytes": B * shape.H_q * D * 2,
            "queue_bytes": 16 * len(it) + 4 * len(ptr), "bucket_launches": 2 * len({n for n in lens if n > 0})}


def plan_decode(seq_lens_host, shape: Shape, device, rules=None, plan: Optional[Plan] = None,
                device_queue: bool = False, fill_blocks: int = 296,
                device_fill: Optional[bool] = None, shared_prefix_table=None) -> DecodePlan:
    """Host planning for one batch: policy (unless `plan` is given), queue, workspace.

    shared_prefix_table (the host block table) asks for the queue that stages
    the prefix pages rows share once for several rows (pkv_build_prefix_queue
    at the plan's chunk; PKV_FLAG_SHARED_PREFIX); a NO_SPLIT plan stays as is.

    device_queue=True leaves the queue to the GPU, rebuilt from the device
    lengths by every paged_decode call (so one plan, or one captured CUDA
    graph, serves any lengths up to the shape's maximum): a BALANCED plan
    gets the balanced queue of its T blocks, a WORK_QUEUE plan the queue
    whose chunk fills one wave of `fill_blocks` blocks.  For the latter the
    decode blocks derive their own items (PKV_FLAG_DEVICE_FILL, one launch)
    where the plan allows it (B <= 1024, merge fused); device_fill=False
    asks for the builder kernel instead.  NO_SPLIT and SPLIT_S plans have no
    queue and read the lengths on the device anyway; they serve lengths up
    to those they were planned for (SPLIT_S: S' chunks of C pages)."""
    if plan is None:
        plan = select_policy(seq_lens_host, shape, rules)
    if shared_prefix_table is not None and plan.mode != NO_SPLIT or (plan.flags & FLAG_SHARED_PREFIX):
        # the prefix-sharing queue at the plan's chunk (a queue-free plan's whole rows otherwise)
        if shared_prefix_table is None:
            raise ValueError("a shared-prefix plan needs the host block table (shared_prefix_table)")
        lens = [int(n) for n in (seq_lens_host.tolist() if isinstance(seq_lens_host, torch.Tensor)
                                 else seq_lens_host)]
        pages_max = max([-(-n // shape.page_size) for n in lens] + [1])
        C = plan.chunk_pages if plan.mode in (SPLIT_S, WORK_QUEUE) and plan.chunk_pages > 0 else pages_max
        members = max(1, 16 // (shape.H_q // shape.H_kv))
        items_h, indptr_h, n_units = build_prefix_queue(lens, shared_prefix_table, shape, C, members)
        flags = (plan.flags | FLAG_SHARED_PREFIX) & ~(FLAG_DEVICE_FILL | FLAG_PDL_EARLY | FLAG_CLUSTER_MERGE)
        pplan = Plan(WORK_QUEUE, n_units, C, flags)
        n_items = int(items_h.shape[0])
        ws = torch.zeros(workspace_bytes(shape, pplan, n_items), dtype=torch.uint8, device=device)
        return DecodePlan(shape, pplan, items_h.to(device), indptr_h.to(device), n_items, ws,
                          prefix_counters(lens, shape, items_h, indptr_h, n_units, flags))
    if plan.mode == WORK_QUEUE and plan.flags & FLAG_DEVICE_FILL:
        device_queue, device_fill, fill_blocks = True, True, plan.num_splits
    if device_queue and plan.mode == WORK_QUEUE:
        fill_ok = shape.B <= FILL_MAX_ROWS and not plan.flags & FLAG_SEPARATE_MERGE
        if device_fill is None:
            device_fill = fill_ok
        if device_fill:
            if not fill_ok:
                raise ValueError("a device-fill plan needs B <= 1024 and the fused merge")
            dplan = Plan(WORK_QUEUE, fill_blocks, 0, plan.flags | FLAG_DEVICE_FILL)
            cap = max(fill_blocks, shape.B * shape.H_kv)
            ws = torch.zeros(workspace_bytes(shape, dplan, cap), dtype=torch.uint8, device=device)
            return DecodePlan(shape, dplan, None, None, cap, ws, plan_counters(seq_lens_host, shape, dplan), True,
                              fill_blocks)
    if device_queue and plan.mode in (WORK_QUEUE, BALANCED):
        pairs = shape.B * shape.H_kv
        if plan.mode == BALANCED:
            cap = balanced_queue_capacity(shape, plan.num_splits)
            n_ptr = pairs + 1 + plan.num_splits + 1
        else:
            cap = fill_queue_capacity(shape, fill_blocks)
            n_ptr = pairs + 1
        items = torch.zeros((cap, 4), dtype=torch.int32, device=device)
        indptr = torch.zeros(n_ptr, dtype=torch.int32, device=device)
        ws = torch.zeros(workspace_bytes(shape, plan, cap), dtype=torch.uint8, device=device)
        return DecodePlan(shape, plan, items, indptr, cap, ws, plan_counters(seq_lens_host, shape, plan), True,
                          fill_blocks if plan.mode == WORK_QUEUE else 0)
    items = indptr = None
    n_items = 0
    if plan.mode in (WORK_QUEUE, BALANCED):
        if plan.mode == WORK_QUEUE:
            items_h, indptr_h = build_work_queue(seq_lens_host, shape, plan.chunk_pages)
        else:
            items_h, indptr_h = build_balanced_queue(seq_lens_host, shape, plan.num_splits)
        n_items = int(items_h.shape[0])
        items = items_h.to(device)
        indptr = indptr_h.to(device)
    ws = torch.zeros(workspace_bytes(shape, plan, n_items), dtype=torch.uint8, device=device)
    return DecodePlan(shape, plan, items, indptr, n_items, ws, plan_counters(seq_lens_host, shape, plan))


def paged_decode(q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor, block_table: torch.Tensor,
                 seq_lens: torch.Tensor, page_size: int, scale: float, *, plan: Optional[DecodePlan] = None,
                 seq_lens_host=None, layout: str = "HND", rules=None, out: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    """out = softmax(scale * q K^T) V per (row, query head), read through the block table.

    q bf16 [B][H_q][D]; pools bf16 (layout "HND" [pages][H_kv][P][D] or "NHD"
    [pages][P][H_kv][D], any strides with a contiguous head_dim axis, see
    shape_of); block_table int32 [B][max_pages]; seq_lens int32 [B], all on one
    CUDA device.  Without `plan`, the policy and queue are built from
    `seq_lens_host` (or a host copy of seq_lens).  Tensors of another dtype,
    device or layout raise TypeError / ValueError before anything is launched.
    """
    L = lib()
    if plan is None:
        shape = shape_of(q, k_pool, block_table, layout, v_pool)
        host = seq_lens_host if seq_lens_host is not None else seq_lens.detach().cpu()
        plan = plan_decode(host, shape, q.device, rules)
    shape = plan.shape
    if out is None:
        out = torch.empty_like(q)
    _check_decode_tensors(q, k_pool, v_pool, block_table, seq_lens, out, shape)
    if plan.device_queue and plan.plan.mode == BALANCED:
        build_balanced_queue_device(seq_lens, shape, plan.plan.num_splits, plan.items, plan.indptr, plan.workspace,
                                    stream)
    elif plan.device_queue and plan.plan.flags & FLAG_DEVICE_FILL:
        pass  # every decode block derives its own item from the device lengths
    elif plan.device_queue:
        build_fill_queue_device(seq_lens, shape, plan.fill_blocks, plan.items, plan.indptr, plan.workspace, stream)
    rc = L.pkv_paged_decode(q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(), block_table.data_ptr(),
                            seq_lens.data_ptr(), page_size, float(scale), out.data_ptr(), ctypes.byref(shape),
                            ctypes.byref(plan.plan), plan.items.data_ptr() if plan.items is not None else None,
                            plan.indptr.data_ptr() if plan.indptr is not None else None, plan.n_items,
                            plan.workspace.data_ptr(), plan.workspace.numel(), _stream_ptr(stream))
    _check(rc, "pkv_paged_decode")
    return out


def paged_decode_noalloc(q: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor, block_table: torch.Tensor,
                         seq_lens: torch.Tensor, page_size: int, scale: float, plan: DecodePlan,
                         out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """pkv_paged_decode_noalloc: like paged_decode, but the library's own fixed
    scratch array replaces the plan's workspace (for callers that cannot
    allocate device memory; see include/pkv.h)."""
    L = lib()
    if out is None:
        out = torch.empty_like(q)
    _check_decode_tensors(q, k_pool, v_pool, block_table, seq_lens, out, plan.shape)
    rc = L.pkv_paged_decode_noalloc(q.data_ptr(), k_pool.data_ptr(), v_pool.data_ptr(), block_table.data_ptr(),
                                    seq_lens.data_ptr(), page_size, float(scale), out.data_ptr(),
                                    ctypes.byref(plan.shape), ctypes.byref(plan.plan),
                                    plan.items.data_ptr() if plan.items is not None else None,
                                    plan.indptr.data_ptr() if plan.indptr is not None else None, plan.n_items,
                                    _stream_ptr(stream))
    _check(rc, "pkv_paged_decode_noalloc")
    return out


def noalloc_status(stream=None) -> int:
    """Synchronize and return the raw device error mask the last
    pkv_paged_decode_noalloc call left in the library's scratch (0 = clean)."""
    L = lib()
    err = c_i32(0)
    rc = L.pkv_noalloc_status(_stream_ptr(stream), ctypes.byref(err))
    if rc not in (0, -5, -6):
        _check(rc, "pkv_noalloc_status")
    return int(err.value)


def workspace_status(plan: DecodePlan, stream=None) -> int:
    """Synchronize and return the raw device error mask of a plan's workspace (0 = clean)."""
    L = lib()
    err = c_i32(0)
    L.pkv_workspace_status(plan.workspace.data_ptr(), _stream_ptr(stream), ctypes.byref(err))
    return int(err.value)


def host_replays() -> int:
    """How many pkv_decode_host calls of this thread replayed a captured graph of their step."""
    return int(lib().pkv_decode_host_replays())


class HostDecoder:
    """Caller-owned buffers for pkv_decode_host, grown on demand: one device
    buffer (torch) and one page-locked host staging buffer.  Calls run on
    `stream` (default: the device's current stream when the decoder is made)
    unless a call passes its own.  The tensors of a call are checked (dtype,
    size, contiguity, pool strides and device) when a tensor object or shape
    is first seen; a serving loop that reuses its buffers pays only identity
    comparisons per step.  Checked tensors must not be resized in place."""

    def __init__(self, device, stream=None):
        self.device = torch.device(device)
        self.dev = torch.empty(0, dtype=torch.uint8, device=self.device)
        self.host = torch.empty(0, dtype=torch.uint8).pin_memory()
        self._stream = _stream_ptr(stream if stream is not None else torch.cuda.current_stream(self.device))
        self._fn = lib().pkv_decode_host
        self._fn_timed = lib().pkv_decode_host_timed
        self._fn_call = lib().pkv_decode_host_call
        self._plan = Plan()
        self._plan_ref = ctypes.byref(self._plan)
        self._bufs = (0, 0, 0, 0)
        self._checked = ()  # weak references to the tensors (and the shape) of the last checked call
        self._args = None   # the argument tuple of the last call with the checked tensors, its scale, no rules
        self._call = HostCall()  # the same arguments as a pkv_host_call block
        self._call_ref = ctypes.byref(self._call)

    def ensure(self, seq_lens_host, shape: Shape, rules=None):
        L = lib()
        lens, _ = _lens_array(seq_lens_host)
        arr, n = rules_array(rules)
        db, hb = c_sz(0), c_sz(0)
        _check(L.pkv_decode_host_bytes(lens, ctypes.byref(shape), arr, n, ctypes.byref(db), ctypes.byref(hb)),
               "pkv_decode_host_bytes")
        if self.dev.numel() < db.value:
            self.dev = torch.zeros(db.value, dtype=torch.uint8, device=self.device)
        if self.host.numel() < hb.value:
            self.host = torch.zeros(hb.value, dtype=torch.uint8).pin_memory()
        bufs = (self.dev.data_ptr(), self.dev.numel(), self.host.data_ptr(), self.host.numel())
        if bufs != self._bufs:  # the stored argument block names the old buffers
            self._bufs = bufs
            self._args = None

    def __call__(self, q_host: torch.Tensor, block_table_host: torch.Tensor, seq_lens_host: torch.Tensor,
                 out_host: torch.Tensor, k_pool: torch.Tensor, v_pool: torch.Tensor, scale: float, shape: Shape,
                 rules=None, stream=None, timing: Optional[HostTiming] = None) -> Plan:
        """One synchronized step; with `timing` (a HostTiming), pkv_decode_host_timed
        also fills in where the call's time went."""
        seen = self._checked
        if not (seen and seen[6] is shape and seen[0]() is q_host and seen[1]() is block_table_host
                and seen[2]() is seq_lens_host and seen[3]() is out_host and seen[4]() is k_pool
                and seen[5]() is v_pool):
            _check_host_call(q_host, block_table_host, seq_lens_host, out_host, k_pool, v_pool, shape,
                             self.dev.get_device())
            self._checked = tuple(weakref.ref(t) for t in (q_host, block_table_host, seq_lens_host, out_host,
                                                            k_pool, v_pool)) + (shape,)
            self._args = None
        elif rules is None and stream is None and self._args is not None and self._args[6] == scale:
            # the same checked tensors as the last call: its parameter block holds
            self._call.timing = None if timing is None else ctypes.addressof(timing)
            rc = self._fn_call(self._call_ref)
            if rc != 0:
                raise PkvError(rc, "pkv_decode_host")
            return Plan.from_buffer_copy(self._plan)
        arr, n = rules_array(rules) if rules is not None else (None, 0)
        dev, dev_n, host, host_n = self._bufs
        args = (q_host.data_ptr(), block_table_host.data_ptr(), seq_lens_host.data_ptr(), out_host.data_ptr(),
                k_pool.data_ptr(), v_pool.data_ptr(), float(scale), ctypes.byref(shape), arr, n, dev, dev_n,
                host, host_n, self._stream if stream is None else _stream_ptr(stream), self._plan_ref)
        if rules is None and stream is None:
            self._args = args
            c = self._call
            (c.q_host, c.block_table_host, c.seq_lens_host, c.out_host, c.k_pool, c.v_pool, c.scale) = args[:7]
            c.shape = ctypes.addressof(shape)
            c.rules, c.n_rules = None, 0
            (c.device_buffer, c.device_buffer_bytes, c.host_staging, c.host_staging_bytes, c.stream) = args[10:15]
            c.plan_out = ctypes.addressof(self._plan)
        rc = self._fn(*args) if timing is None else self._fn_timed(*args, ctypes.byref(timing))
        if rc != 0:
            raise PkvError(rc, "pkv_decode_host")
        return Plan.from_buffer_copy(self._plan)


def decode_host(*args, **kwargs):
    """One-shot pkv_decode_host with freshly allocated buffers (see HostDecoder)."""
    q_host, bt_host, lens_host, out_host, k_pool, v_pool, scale, shape = args[:8]
    dec = HostDecoder(k_pool.device)
    dec.ensure(lens_host, shape, kwargs.get("rules"))
    return dec(*args, **kwargs)
