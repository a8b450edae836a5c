"""B200-native paged GQA decode attention.

Single-token decode attention read straight through a paged KV cache's block
table, where G = H_q / H_kv query heads share each KV head: a split-S kernel
whose chunks produce partial softmax states, an exact merge, a compact work
queue (with a chunk that can fill one wave of the GPU, and a balanced cut for
a persistent grid, both also buildable on the device) and a calibrated policy
that picks the plan per batch.  Every step runs in the C-ABI library
`libpkv.so` (CUDA for sm_100a plus host C++); this package only marshals
arguments to it.

The CUDA library is loaded on first use of anything but `workloads`; if it is
missing or cannot find a GPU, the call raises instead of falling back.
"""
from . import workloads  # noqa: F401  (inputs only; no CUDA needed)

_LAZY = {
    "lib", "paged_decode", "plan_decode", "DecodePlan", "Shape", "Plan", "Rule",
    "select_policy", "build_work_queue", "workspace_bytes", "plan_counters",
    "load_rules", "default_rules", "decode_host", "PkvError",
    "NO_SPLIT", "SPLIT_S", "WORK_QUEUE", "BALANCED", "FLAG_SEPARATE_MERGE", "FLAG_NO_PDL", "FLAG_DEEP_RING",
    "build_balanced_queue", "paged_decode_noalloc", "shape_of", "HostDecoder", "FLAG_CLUSTER_MERGE",
    "FLAG_PDL_EARLY", "FLAG_DEVICE_FILL", "FLAG_SHARED_PREFIX", "build_prefix_queue", "HostTiming", "HostCall", "host_replays",
    "noalloc_status", "balanced_queue_capacity",
    "build_balanced_queue_device", "fill_queue_capacity", "build_fill_queue_device",
}


def __getattr__(name):
    if name in _LAZY:
        from . import binding

        return getattr(binding, name)
    raise AttributeError(name)
