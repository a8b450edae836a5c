"""Build libpkv.so in-tree: the CUDA kernels for sm_100a plus the host planner.

    python -m paged_kv_gqa_17_b200.build [--force] [--verbose]

nvcc compiles csrc/*.cu for sm_100a only (-gencode arch=compute_100a,code=sm_100a)
with -lineinfo; the CUDA runtime is linked statically, so the library only needs
the NVIDIA driver at run time.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libpkv.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    cand = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    return cand


POLICY_JSON = os.path.join(HERE, "policy_b200.json")
POLICY_INC = os.path.join(CSRC, "pkv_policy_table.inc")
_MODES = {"NO_SPLIT": "PKV_NO_SPLIT", "SPLIT_S": "PKV_SPLIT_S", "WORK_QUEUE": "PKV_WORK_QUEUE",
          "BALANCED": "PKV_BALANCED"}


def write_policy_table() -> str:
    """Turn policy_b200.json into the C initializer of the built-in table."""
    import json

    with open(POLICY_JSON) as f:
        doc = json.load(f)
    lines = ["// Generated from policy_b200.json by paged_kv_gqa_17_b200/build.py; edit the JSON instead.",
             "// b_lo, b_hi, nmax_lo, nmax_hi, mode, num_splits, chunk_pages, flags"]
    for r in doc["rules"]:
        lines.append("{%d, %d, %d, %d, %s, %d, %d, %d}," % (
            int(r["b_lo"]), int(r.get("b_hi", 2**31 - 1)), int(r["nmax_lo"]), int(r.get("nmax_hi", 2**31 - 1)),
            _MODES[r["mode"]], int(r.get("num_splits", 1)), int(r.get("chunk_pages", 0)), int(r.get("flags", 0))))
    text = "\n".join(lines) + "\n"
    old = open(POLICY_INC).read() if os.path.exists(POLICY_INC) else None
    if old != text:
        with open(POLICY_INC, "w") as f:
            f.write(text)
    return POLICY_INC


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _stale(out: str) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    deps = (sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.inc")) +
            glob.glob(os.path.join(INCLUDE, "*.h")) + [POLICY_JSON])
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, out: str = LIB, extra=()) -> str:
    write_policy_table()
    if not force and not _stale(out):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-shared", "-o", tmp, *sources(),
           "-cudart", "static"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
