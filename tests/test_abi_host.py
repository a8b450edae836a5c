"""The C-ABI library on the CPU: it loads, exports every declared symbol, and
its host planner (policy, queue, counters, workspace sizing) matches the
oracle's plain-Python versions bit for bit.  No GPU calls."""
import ctypes
import os
import random
import re
import subprocess

import pytest
import torch

from oracle import oracle as O
from paged_kv_gqa_17_b200 import binding as bd

from . import host_pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h")]


def declared_symbols():
    names = []
    for h in HEADERS:
        text = open(h).read()
        names += re.findall(r"PKV_API\s+[\w\s\*]+?\b(pkv_\w+)\s*\(", text)
    return names


@pytest.fixture(scope="module")
def L():
    from paged_kv_gqa_17_b200 import build

    build.build()
    return bd.lib()


def test_every_declared_symbol_is_exported(L):
    names = declared_symbols()
    assert len(names) >= 13
    for n in names:
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", bd.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\b(pkv_\w+)\b", out))
    assert set(names) <= exported
    # the binding wraps exactly the declared functions
    assert {s[0] for s in bd.SIGNATURES} == set(names)


def test_library_is_built_for_sm100a_only():
    out = subprocess.run(["cuobjdump", "--list-elf", bd.LIB_PATH], capture_output=True, text=True).stdout
    arches = set(re.findall(r"sm_(\d+a?)", out))
    assert arches == {"100a"}, arches


def test_version_and_status_strings(L):
    assert b"sm_100a" in L.pkv_version()
    assert L.pkv_status_string(0) == b"ok"
    assert L.pkv_status_string(-3) == b"buffer too small"


def _cases(seed, n=60):
    rng = random.Random(seed)
    for _ in range(n):
        B = rng.randint(0, 12)
        lens = [rng.choice([0, rng.randint(1, 40), rng.randint(1, 3000), rng.randint(1, 140000)]) for _ in range(B)]
        H_kv = rng.choice([1, 2, 4, 8])
        G = rng.choice([1, 2, 4, 8, 16])
        yield lens, H_kv, G, rng.choice([64, 128])


def _shape(lens, H_kv, G, D):
    return bd.make_shape(len(lens), H_kv * G, H_kv, D, 16, 1 + max([-(-n // 16) for n in lens] + [0]), 1)


def test_policy_matches_oracle_bit_exactly(L):
    tables = [bd.load_rules(os.path.join(ROOT, "paged_kv_gqa_17_b200", f))
              for f in ("policy_paper_rule.json", "policy_b200.json")]
    tables.append([bd.Rule(0, 3, 0, 5000, 1, 7, 0, 1), bd.Rule(3, 100, 100, 2**31 - 1, 2, 1, 5, 0)])
    tables += [[bd.Rule(0, 2**31 - 1, 0, 2**31 - 1, 2, T, 0, 4)] for T in (1, 37, 296)]  # queue filling T blocks
    for lens, H_kv, G, D in _cases(1):
        shape = _shape(lens, H_kv, G, D)
        for rules in tables:
            got = bd.select_policy(lens, shape, rules).tuple()
            want = O.select_policy(lens, 16, [O.Rule(*r.tuple()) for r in rules], H_kv)
            assert got == want, (lens, got, want)


def test_default_policy_is_the_committed_table(L):
    got = [r.tuple() for r in bd.default_rules()]
    want = [r.tuple() for r in bd.load_rules(os.path.join(ROOT, "paged_kv_gqa_17_b200", "policy_b200.json"))]
    assert got == want


def test_work_queue_matches_oracle_bit_exactly(L):
    for lens, H_kv, G, D in _cases(2):
        shape = _shape(lens, H_kv, G, D)
        for C in (1, 3, 16, 64):
            items, indptr = bd.build_work_queue(lens, shape, C)
            w_items, w_indptr = O.build_work_queue(lens, H_kv, 16, C)
            assert [tuple(x) for x in items.tolist()] == w_items
            assert indptr.tolist() == w_indptr


def test_balanced_queue_matches_oracle_bit_exactly(L):
    for lens, H_kv, G, D in _cases(4):
        shape = _shape(lens, H_kv, G, D)
        for T in (1, 3, 37, 296):
            items, indptr = bd.build_balanced_queue(lens, shape, T)
            w_items, w_indptr, w_bptr = O.build_balanced_queue(lens, H_kv, 16, T)
            assert [tuple(x) for x in items.tolist()] == w_items, (lens, T)
            assert indptr.tolist() == w_indptr + w_bptr, (lens, T)


def test_counters_match_oracle(L):
    for lens, H_kv, G, D in _cases(3):
        shape = _shape(lens, H_kv, G, D)
        for rules in ([bd.Rule(0, 2**31 - 1, 0, 2**31 - 1, m, 5, 7, f)
                       for m, f in ((0, 0), (1, 0), (1, 1), (2, 0), (2, 1), (3, 0), (3, 1))]):
            plan = bd.select_policy(lens, shape, [rules])
            got = bd.plan_counters(lens, shape, plan)
            want = O.counters(lens, H_kv * G, H_kv, D, 16, plan.tuple()).__dict__
            assert got == want, (lens, plan, got, want)


def test_workspace_bytes_cover_partial_states(L):
    shape = bd.make_shape(8, 32, 8, 128, 16, 2048, 9000)
    plan = bd.Plan(2, 64, 32, 0)
    n = 500
    b = bd.workspace_bytes(shape, plan, n)
    assert b >= 256 + 64 * 4 + n * 4 * 4 * 2 + n * 4 * 128 * 4
    assert b % 256 == 0


def test_host_rejects_bad_arguments(L):
    shape = bd.make_shape(2, 32, 8, 128, 16, 10, 100)
    lens, _ = bd._lens_array([5, -1])
    plan = bd.Plan()
    assert L.pkv_select_policy(lens, ctypes.byref(shape), None, 0, ctypes.byref(plan)) == -1
    bad = bd.make_shape(2, 30, 8, 128, 16, 10, 100)  # H_q not a multiple of H_kv
    lens, _ = bd._lens_array([5, 6])
    assert L.pkv_select_policy(lens, ctypes.byref(bad), None, 0, ctypes.byref(plan)) == -1
    rules, n = bd.rules_array([bd.Rule(0, 9, 0, 9, 1, 0, 0, 0)])
    assert L.pkv_select_policy(lens, ctypes.byref(shape), rules, n, ctypes.byref(plan)) == -1
    items = (bd.WorkItem * 1)()
    indptr = (ctypes.c_int32 * 17)()
    n_items = ctypes.c_int32(0)
    rc = L.pkv_build_work_queue(lens, ctypes.byref(shape), 1, items, 1, indptr, ctypes.byref(n_items))
    assert rc == -3 and n_items.value == 16  # capacity error reports the size needed
    assert L.pkv_build_work_queue(lens, ctypes.byref(shape), 0, items, 1, indptr, ctypes.byref(n_items)) == -1


def test_decode_rejects_unsupported_shapes_without_touching_the_gpu(L):
    """Shape checks run before any CUDA call, so they can be tested here."""
    plan = bd.Plan(0, 1, 0, 0)
    for shape, want in ((bd.make_shape(1, 4, 1, 96, 16, 4, 8), -2),    # head_dim 96
                        (bd.make_shape(1, 4, 1, 128, 32, 4, 8), -2),   # page size 32
                        (bd.make_shape(1, 34, 1, 128, 16, 4, 8), -2),  # G = 34
                        (bd.make_shape(1, 4, 3, 128, 16, 4, 8), -1)):  # H_q % H_kv != 0
        rc = L.pkv_paged_decode(None, None, None, None, None, shape.page_size, 1.0, None, ctypes.byref(shape),
                                ctypes.byref(plan), None, None, 0, None, 0, None)
        assert rc == want, (shape.head_dim, shape.page_size, rc)
    shape = bd.make_shape(1, 4, 1, 128, 16, 4, 8)
    rc = L.pkv_paged_decode(None, None, None, None, None, 8, 1.0, None, ctypes.byref(shape), ctypes.byref(plan),
                            None, None, 0, None, 0, None)
    assert rc == -1  # page_size argument disagrees with the shape
    wq = bd.Plan(2, 1, 4, 0)
    rc = L.pkv_paged_decode(None, None, None, None, None, 16, 1.0, None, ctypes.byref(shape), ctypes.byref(wq),
                            None, None, 0, None, 0, None)
    assert rc == -1  # work queue without items
    for bad_cluster in (bd.Plan(1, 17, 4, 8), bd.Plan(0, 1, 0, 8)):
        rc = L.pkv_paged_decode(None, None, None, None, None, 16, 1.0, None, ctypes.byref(shape),
                                ctypes.byref(bad_cluster), None, None, 0, None, 0, None)
        assert rc == -2  # cluster merge only for split-S with S <= 16


def test_host_pins_hold_for_the_c_planner(L):
    """The oracle's host pins, run against an adapter over the C planner."""

    class Adapter:
        NO_SPLIT, SPLIT_S, WORK_QUEUE, BALANCED, FLAG_SEPARATE_MERGE, INT32_MAX = 0, 1, 2, 3, 1, 2**31 - 1
        FLAG_DEVICE_FILL = 32
        Rule = O.Rule
        load_rules = staticmethod(O.load_rules)

        @staticmethod
        def build_work_queue(lens, H_kv, P, C):
            if C < 1:
                raise ValueError
            shape = bd.make_shape(len(lens), H_kv, H_kv, 64, P, 1, 1)
            items, indptr = bd.build_work_queue(lens, shape, C)
            return [tuple(x) for x in items.tolist()], indptr.tolist()

        @staticmethod
        def build_balanced_queue(lens, H_kv, P, T):
            if T < 1:
                raise ValueError
            shape = bd.make_shape(len(lens), H_kv, H_kv, 64, P, 1, 1)
            items, indptr = bd.build_balanced_queue(lens, shape, T)
            ptr = indptr.tolist()
            pairs = len(lens) * H_kv
            return [tuple(x) for x in items.tolist()], ptr[:pairs + 1], ptr[pairs + 1:]

        shared_prefixes = staticmethod(O.shared_prefixes)

        @staticmethod
        def build_prefix_queue(lens, bt, H_kv, P, C, M):
            if C < 1 or M < 1:
                raise ValueError
            width = max([len(r) for r in bt] + [1])
            table = torch.tensor([list(r) + [0] * (width - len(r)) for r in bt] or [[0]], dtype=torch.int32)
            shape = bd.make_shape(len(lens), H_kv, H_kv, 64, P, width, 1)
            items, indptr, n_units = bd.build_prefix_queue(lens, table, shape, C, M)
            pairs = len(lens) * H_kv
            ptr = indptr.tolist()
            return ([tuple(x) for x in items.tolist()], ptr[:pairs + 1], ptr[pairs + 1:pairs + 2 + n_units],
                    ptr[pairs + 2 + n_units:])

        @staticmethod
        def select_policy(lens, P, rules, H_kv=1):
            shape = bd.make_shape(len(lens), H_kv, H_kv, 64, P, 1, 1)
            try:
                return bd.select_policy(lens, shape, [r.__dict__ if hasattr(r, "__dict__") else r for r in rules]
                                        ).tuple()
            except bd.PkvError as e:
                raise ValueError(str(e))

        @staticmethod
        def counters(lens, H_q, H_kv, D, P, plan):
            shape = bd.make_shape(len(lens), H_q, H_kv, D, P, 1, 1)
            d = bd.plan_counters(lens, shape, bd.Plan(*plan))

            class C:
                pass

            c = C()
            c.__dict__.update(d)
            return c

    failed = host_pins.run_all(Adapter)
    assert not failed, failed


def test_device_queue_builder_host_checks(L):
    """The device-side builder rejects what it cannot do before queueing
    anything (no GPU needed for these paths)."""
    shape = bd.make_shape(4, 8, 2, 128, 16, 8, 10)
    cap = ctypes.c_int32(0)
    assert L.pkv_balanced_queue_capacity(ctypes.byref(shape), 37, ctypes.byref(cap)) == 0
    assert cap.value == 4 * 2 + 37
    assert L.pkv_balanced_queue_capacity(ctypes.byref(shape), 0, ctypes.byref(cap)) == -1
    # capacity below the bound
    assert L.pkv_build_balanced_queue_device(None, ctypes.byref(shape), 37, None, 44, None, None, None) == -3
    # missing buffers
    assert L.pkv_build_balanced_queue_device(None, ctypes.byref(shape), 37, None, 45, None, None, None) == -1
    # more rows than the one-block builder handles
    big = bd.make_shape(5000, 8, 2, 128, 16, 8, 10)
    assert L.pkv_build_balanced_queue_device(None, ctypes.byref(big), 37, None, 1 << 20, None, None, None) == -2
    # an empty batch queues nothing
    empty = bd.make_shape(0, 8, 2, 128, 16, 8, 10)
    assert L.pkv_build_balanced_queue_device(None, ctypes.byref(empty), 37, None, 0, None, None, None) == 0
    # the fill-one-wave builder: capacity max(T, B*H_kv), the same checks
    assert L.pkv_fill_queue_capacity(ctypes.byref(shape), 5, ctypes.byref(cap)) == 0 and cap.value == 8
    assert L.pkv_fill_queue_capacity(ctypes.byref(shape), 296, ctypes.byref(cap)) == 0 and cap.value == 296
    assert L.pkv_build_fill_queue_device(None, ctypes.byref(shape), 296, None, 295, None, None, None) == -3
    assert L.pkv_build_fill_queue_device(None, ctypes.byref(shape), 296, None, 296, None, None, None) == -1
    assert L.pkv_build_fill_queue_device(None, ctypes.byref(big), 296, None, 1 << 20, None, None, None) == -2
    assert L.pkv_build_fill_queue_device(None, ctypes.byref(empty), 296, None, 0, None, None, None) == 0


def test_prefix_queue_matches_oracle_bit_for_bit(L):
    """pkv_build_prefix_queue against the oracle's plain-Python builder on
    the seeded sharing cases: items, pair offsets, unit offsets and members."""
    for lens, bt, H_kv, P, C, M in host_pins._prefix_cases(seed=41, n=60):
        width = max(len(r) for r in bt)
        table = torch.tensor([list(r) for r in bt], dtype=torch.int32)
        shape = bd.make_shape(len(lens), H_kv, H_kv, 64, P, width, 1)
        items, indptr, n_units = bd.build_prefix_queue(lens, table, shape, C, M)
        o_items, o_indptr, o_uptr, o_uitems = O.build_prefix_queue(lens, bt, H_kv, P, C, M)
        assert [tuple(x) for x in items.tolist()] == o_items, (lens, bt, H_kv, P, C, M)
        assert indptr.tolist() == o_indptr + o_uptr + o_uitems, (lens, bt, H_kv, P, C, M)
        assert n_units == len(o_uptr) - 1


def test_prefix_plan_counters_recount(L):
    """The prefix plan's counters: one block per unit, a unit's pages once."""
    for lens, bt, H_kv, P, C, M in host_pins._prefix_cases(seed=43, n=30):
        if P != 16:
            continue
        width = max(len(r) for r in bt)
        table = torch.tensor([list(r) for r in bt], dtype=torch.int32)
        shape = bd.make_shape(len(lens), 4 * H_kv, H_kv, 64, P, width, 1)
        items, indptr, n_units = bd.build_prefix_queue(lens, table, shape, C, M)
        c = bd.prefix_counters(lens, shape, items, indptr, n_units)
        o_items, o_indptr, o_uptr, o_uitems = O.build_prefix_queue(lens, bt, H_kv, P, C, M)
        pages = 0
        for u in range(len(o_uptr) - 1):
            pages += len({(o_items[x][1], pg) for x in o_uitems[o_uptr[u]:o_uptr[u + 1]]
                          for pg in range(o_items[x][2] // P, -(-o_items[x][3] // P))})
        assert c["kv_bytes_streamed"] == pages * P * 2 * 64 * 2, (lens, bt, H_kv, C, M)
        assert c["work_items"] == len(o_uptr) - 1 and c["queue_bytes"] == 16 * len(o_items) + 4 * (
            len(o_indptr) + len(o_uptr) + len(o_uitems))
        plain = O.counters(lens, 4 * H_kv, H_kv, 64, P, (O.WORK_QUEUE, 1, C, 0))
        assert c["kv_bytes_streamed"] <= plain.kv_bytes_streamed


def test_host_call_block_matches_the_header(L, tmp_path):
    """bd.HostCall has pkv_host_call's size and field offsets (a C program
    compiled against the header prints them), and the parameter-block entry
    point rejects a NULL block before any CUDA call."""
    fields = [f for f, _ in bd.HostCall._fields_]
    src = tmp_path / "layout.c"
    src.write_text("#include <stddef.h>\n#include <stdio.h>\n#include \"pkv.h\"\nint main(void) {\n"
                   "  printf(\"%zu\", sizeof(pkv_host_call));\n"
                   + "".join(f"  printf(\" %zu\", offsetof(pkv_host_call, {f}));\n" for f in fields)
                   + "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    assert got == [ctypes.sizeof(bd.HostCall)] + [getattr(bd.HostCall, f).offset for f in fields]
    assert L.pkv_decode_host_call(None) == -1
