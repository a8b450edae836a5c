"""Plant plausible mistakes in copies of the oracle; each must fail a pin.

The C oracle's source is patched textually, compiled into a temporary
directory and run through every attention pin; the Python host pieces are
patched the same way and run through the host pins.  Nothing here touches
the GPU or the CUDA library.
"""
import os
import subprocess
import sys

import pytest

from oracle import build_oracle

from . import host_pins, oracle_pins

HERE = os.path.dirname(os.path.abspath(__file__))
ORACLE_DIR = os.path.join(os.path.dirname(HERE), "oracle")

C_MUTANTS = {
    "kv head map uses modulo": ("return hq / G;", "return hq % pr->H_kv;"),
    "scale dropped": ("return pr->scale * dot;", "return dot;"),
    "slot off by one": ("int32_t slot = t % pr->P;", "int32_t slot = (t + 1) % pr->P;"),
    "exponent sign flipped": ("double w = exp(s[t] - M);", "double w = exp(M - s[t]);"),
    "normalised by N": ("out[d] /= Z;", "out[d] /= (double)N;"),
    "block table row stride": ("(int64_t)row * pr->max_pages", "(int64_t)row * pr->P"),
    "head and token strides swapped": ("(int64_t)h * pr->s_head + (int64_t)slot * pr->s_tok",
                                       "(int64_t)slot * pr->s_head + (int64_t)h * pr->s_tok"),
    "last token dropped": ("    for (int t = 0; t < N; ++t) {\n        double w = exp",
                           "    for (int t = 0; t + 1 < N; ++t) {\n        double w = exp"),
    "merge weight sign": ("double w = exp(m[i] - M);", "double w = exp(M - m[i]);"),
    "merge ignores l": ("L += w * l[i];", "L += l[i];"),
    "partial state drops max": ("double w = exp(logit(&pr, row, hq, t) - m);",
                                "double w = exp(logit(&pr, row, hq, t));"),
}

PY_MUTANTS = {
    "queue emits empty tail chunk": ("while c * span < n:", "while c * span <= n:"),
    "queue chunk not clipped": ("min((c + 1) * span, n)", "(c + 1) * span"),
    "policy range closed above": ("r.b_lo <= B < r.b_hi", "r.b_lo <= B <= r.b_hi"),
    "policy last match wins": ("if chosen is None and r.b_lo", "if r.b_lo"),
    "split count not tightened": ("return (chosen.mode, _ceil_div(pages_max, C), C, chosen.flags)",
                                  "return (chosen.mode, chosen.num_splits if chosen.mode == SPLIT_S else _ceil_div(pages_max, C), C, chosen.flags)"),
    "bucket launches count rows": ("2 * distinct)", "2 * B)"),
    "merge traffic counts single-chunk pairs": ("sum(k for k in per_pair if k > 1)", "sum(per_pair)"),
    "balanced owner off by one": ("        while starts[b] > u:", "        while starts[b] >= u and b > 0:"),
    "balanced share rounded up": ("starts = [(b * U) // T for b in range(T + 1)]",
                                  "starts = [min(U, -(-(b * U) // T)) for b in range(T + 1)]"),
    "balanced item not clipped to row": ("min((y - u) * P, n)", "(y - u) * P"),
    "fill rule allows one item too many": ("if fill_items(lens, H_kv, P, c) <= chosen.num_splits:",
                                           "if fill_items(lens, H_kv, P, c) <= chosen.num_splits + 1:"),
    "queue bytes miss the last pair offset": ("else 16 * work + 4 * (B * H_kv + 1)\n",
                                              "else 16 * work + 4 * B * H_kv\n"),
    "balanced queue bytes miss the block offsets": (" + 4 * (B * H_kv + 1) + 4 * (S + 1)", " + 4 * (B * H_kv + 1)"),
    "streamed bytes count valid tokens only": ("kv_streamed = sum(pages) * P * H_kv", "kv_streamed = sum(lens) * H_kv"),
    "balanced merge counts single-slot pairs": ("        merge = 2 * sum(k for k in per_pair if k > 1) * state",
                                                "        merge = 2 * sum(per_pair) * state"),
    "balanced work counts items": ("        work = S\n", "        work = len(items)\n"),
    "no-split empty rows not per head": ("work = B * H_kv\n        empty = H_kv * sum(",
                                         "work = B * H_kv\n        empty = sum("),
    "no-split work counts rows": ("        work = B * H_kv\n", "        work = B\n"),
    "device-fill counters count the queue bytes": ("qbytes = 0 if device_fill else 16 * work",
                                                   "qbytes = 16 * work"),
    "device-fill plan carries a chunk": ("        return (WORK_QUEUE, chosen.num_splits, 0, chosen.flags)\n",
                                         "        return (WORK_QUEUE, chosen.num_splits, 1, chosen.flags)\n"),
    "prefix shares the leader's partial last page": ("        L = lens[lead] // P\n",
                                                     "        L = -(-lens[lead] // P)\n"),
    "prefix counts a member's partial page": ("            while k < min(full, L) and", "            while k < L and"),
    "prefix groups rows without a full page": ("        if n >= P:\n            by_first", "        if n >= 1:\n            by_first"),
    "prefix tail chunks restart at zero": ("                t = L * P\n                while t < n:",
                                           "                t = 0\n                while t < n:"),
    "prefix units exceed the member cap": ("for k in range(0, len(members), max_members):\n            units.append(members[k:k + max_members])",
                                           "for k in range(0, len(members), max_members + 1):\n            units.append(members[k:k + max_members + 1])"),
    "fill rule ignores heads": ("    return H_kv * sum(max(1, _ceil_div(_ceil_div(int(n), P), C)) for n in seq_lens)",
                                "    return sum(max(1, _ceil_div(_ceil_div(int(n), P), C)) for n in seq_lens)"),
}


_RUNNER = """
import sys
sys.path.insert(0, {root!r})
from oracle import oracle as O
from tests import oracle_pins
failed = oracle_pins.run_all(O.load({lib!r}))
print("FAILED_PINS", len(failed))
for f in failed:
    print(" ", f[:200])
sys.exit(3 if failed else 0)
"""


@pytest.mark.parametrize("name", sorted(C_MUTANTS))
def test_c_oracle_mutant_is_caught(tmp_path, name):
    """Each mutant runs in its own process: an out-of-bounds read that crashes
    it counts as caught, like a failed pin."""
    old, new = C_MUTANTS[name]
    src = open(os.path.join(ORACLE_DIR, "pkv_oracle.c")).read()
    assert old in src, f"mutation site for {name!r} not found"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = build_oracle.build(str(path), str(tmp_path / "libmutant.so"), force=True)
    root = os.path.dirname(HERE)
    r = subprocess.run([sys.executable, "-c", _RUNNER.format(root=root, lib=lib)],
                       capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"planted mistake {name!r} passed every pin:\n{r.stdout}"


_PY_RUNNER = """
import sys, types
sys.path.insert(0, {root!r})
from tests import host_pins
mod = types.ModuleType("oracle._mutant")
mod.__dict__["__package__"] = "oracle"
sys.modules[mod.__name__] = mod  # dataclasses look their module up here
exec(compile(open({path!r}).read(), "oracle_mutant.py", "exec"), mod.__dict__)
failed = host_pins.run_all(mod)
print("FAILED_PINS", len(failed))
sys.exit(3 if failed else 0)
"""


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_py_oracle_mutant_is_caught(tmp_path, name):
    """Each mutant runs in its own process with a time limit: a mutant that
    never finishes (a loop that stops advancing) counts as caught."""
    old, new = PY_MUTANTS[name]
    src = open(os.path.join(ORACLE_DIR, "oracle.py")).read()
    assert old in src, f"mutation site for {name!r} not found"
    path = tmp_path / "oracle_mutant.py"
    path.write_text(src.replace(old, new))
    root = os.path.dirname(HERE)
    try:
        r = subprocess.run([sys.executable, "-c", _PY_RUNNER.format(root=root, path=str(path))],
                           capture_output=True, text=True, timeout=30)
    except subprocess.TimeoutExpired:
        return
    assert r.returncode != 0, f"planted mistake {name!r} passed every pin:\n{r.stdout}"
