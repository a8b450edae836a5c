"""Failure detection on the GPU without a fault: a bounded device wait that
runs out is reported through the workspace, and the context stays usable."""
import ctypes

import pytest
import torch

from paged_kv_gqa_17_b200 import binding as bd
from paged_kv_gqa_17_b200 import workloads as W

from .gpu_util import assert_close, oracle_full, run, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_gqa_17_b200 import build

    build.build()
    return bd.lib()


def test_wait_that_nobody_satisfies_times_out_and_is_reported(L):
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.pkv_selftest_wait_timeout(ws.data_ptr(), ws.numel(), 20000, stream) == 0  # 20 ms limit
    err = ctypes.c_int32(0)
    assert L.pkv_workspace_status(ws.data_ptr(), stream, ctypes.byref(err)) == -5  # PKV_ERR_TIMEOUT
    assert err.value & 1
    # cleared by a workspace init; the context is still usable for real work
    assert L.pkv_workspace_init(ws.data_ptr(), ws.numel(), stream) == 0
    assert L.pkv_workspace_status(ws.data_ptr(), stream, ctypes.byref(err)) == 0 and err.value == 0
    w = to_device(W.make_custom([300, 40], 8, 2, 64, seed=401, poison=True))
    got, _ = run(w)
    assert_close(got, oracle_full(w), "decode after a timed-out wait")


def test_selftest_rejects_unbounded_limits(L):
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    assert L.pkv_selftest_wait_timeout(ws.data_ptr(), ws.numel(), 0, None) == -1
    assert L.pkv_selftest_wait_timeout(ws.data_ptr(), ws.numel(), 2000001, None) == -1
