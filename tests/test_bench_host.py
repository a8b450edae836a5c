"""Host-side pieces of bench.py, without a GPU: the JSON description of
every plan family, the argument parser, and the reference arm's JSON line
(the oracle on the tiny workload)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from paged_kv_gqa_17_b200 import workloads as W  # noqa: E402


class _Plan:
    def __init__(self, mode, S, C, flags):
        self.mode, self.num_splits, self.chunk_pages, self.flags = mode, S, C, flags


@pytest.mark.parametrize("mode,name", [(0, "NO_SPLIT"), (1, "SPLIT_S"), (2, "WORK_QUEUE"), (3, "BALANCED")])
def test_describe_names_every_plan_family(mode, name):
    w = W.make("tiny")
    d = bench._describe(w, _Plan(mode, 4, 2, 0))
    assert d["plan"]["mode"] == name
    assert d["batch"] == 1 and d["tokens"] == 512
    json.dumps(d)


def test_parser_accepts_every_named_workload():
    for name in ("tiny", "long", "crossover", "mixed", "prefix", "bimodal", "uniform", "zipf"):
        assert bench.parse_args(["--workload", name]).workload == name
    a = bench.parse_args([])
    assert a.gpus == 1 and a.warmup >= 3 and a.workload == "long" and not a.no_graph


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "2", "--warmup", "1"], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "impl"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["unit"] == d["unit"]


def test_recorded_traffic_follows_the_kernel_source_hash(monkeypatch):
    """The roofline's traffic figure is reported only for the kernel sources
    it was captured on."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    assert rows, "profiles/traffic.txt lists no capture"
    name, digest, nbytes = rows[0]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: digest)
    assert bench.recorded_traffic(name) == int(nbytes)
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.recorded_traffic(name) is None
    assert bench.recorded_traffic("no-such-workload") is None



def test_calibration_row_replacement_keeps_the_other_rows_and_covers_the_grid():
    """calibrate --only-b: the re-measured row's rules replace exactly the
    old rules of that B range; together they still cover every (B, N_max)
    of the grid exactly once, and build_rules merges equal neighbours."""
    import json

    from paged_kv_gqa_17_b200 import calibrate as cal

    old = json.load(open(os.path.join(ROOT, "paged_kv_gqa_17_b200", "policy_b200.json")))["rules"]
    bi = cal.B_REP.index(8)
    best = {(bi, nj): (2, 1, 48, 4) if nj < 3 else (2, 296, 0, 0) for nj in range(len(cal.N_REP))}
    row = cal.build_rules(best, [bi])
    assert [(r["nmax_lo"], r["nmax_hi"]) for r in row] == [(0, 16384), (16384, 2**31 - 1)]
    assert row[0] == {"b_lo": 8, "b_hi": 16, "nmax_lo": 0, "nmax_hi": 16384, "mode": "WORK_QUEUE",
                      "chunk_pages": 48, "flags": 4}
    assert row[1]["num_splits"] == 296 and row[1]["chunk_pages"] == 0 and "flags" not in row[1]
    new = cal.replace_row(old, row, cal.B_EDGES[bi])
    assert [r for r in new if r["b_lo"] != 8] == [r for r in old if r["b_lo"] != 8]
    assert [r for r in new if r["b_lo"] == 8] == row
    for B in (1, 2, 3, 4, 7, 8, 15, 16, 31, 32, 64, 1000):
        for n in (0, 1023, 1024, 5000, 16383, 16384, 70000, 2**31 - 2):
            hits = [r for r in new if r["b_lo"] <= B < r["b_hi"] and r["nmax_lo"] <= n < r["nmax_hi"]]
            assert len(hits) == 1, (B, n, hits)
