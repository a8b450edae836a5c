"""Pools that are views into a larger cache, through the C ABI: the K and V
halves of one combined cache (HND and NHD), rows padded past head_dim, and an
unused head per page.  The library takes the pools' strides from the shape,
so each must match the oracle (on packed copies of the same values) and give
the same bits as the same plan on packed pools."""
import pytest
import torch

from paged_kv_gqa_17_b200 import binding as bd
from paged_kv_gqa_17_b200 import workloads as W

from .gpu_util import assert_close, oracle_full, to_device

pytestmark = pytest.mark.gpu

ANY = (0, 2**31 - 1, 0, 2**31 - 1)
NAN = float("nan")

PLANS = {
    "nosplit": bd.Rule(*ANY, 0, 1, 0, 0),
    "split7": bd.Rule(*ANY, 1, 7, 0, 0),
    "split32_deep_sep": bd.Rule(*ANY, 1, 32, 0, 5),
    "wq3": bd.Rule(*ANY, 2, 1, 3, 0),
    "wqfill37": bd.Rule(*ANY, 2, 37, 0, 0),
    "bal37": bd.Rule(*ANY, 3, 37, 0, 0),
    "split16_cl": bd.Rule(*ANY, 1, 16, 0, 8),
}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_gqa_17_b200 import build

    build.build()
    bd.lib()


def combined(k, v):
    """K and V side by side in one cache: [pages][2][...]."""
    kv = torch.full((k.shape[0], 2) + tuple(k.shape[1:]), NAN, dtype=k.dtype, device=k.device)
    kv[:, 0] = k
    kv[:, 1] = v
    return kv[:, 0], kv[:, 1]


def padded_rows(k, v, pad=8):
    """Every (page, head, slot) row padded with NaN past head_dim."""
    out = []
    for t in (k, v):
        big = torch.full(tuple(t.shape[:-1]) + (t.shape[-1] + pad,), NAN, dtype=t.dtype, device=t.device)
        big[..., :t.shape[-1]] = t
        out.append(big[..., :t.shape[-1]])
    return out


def extra_head(k, v):
    """One unused (NaN) head after the real ones on every HND page."""
    out = []
    for t in (k, v):
        big = torch.full((t.shape[0], t.shape[1] + 1) + tuple(t.shape[2:]), NAN, dtype=t.dtype, device=t.device)
        big[:, :t.shape[1]] = t
        out.append(big[:, :t.shape[1]])
    return out


VIEWS = {
    "combined_hnd": ("HND", combined),
    "combined_nhd": ("NHD", combined),
    "padded_rows_hnd": ("HND", padded_rows),
    "padded_rows_nhd": ("NHD", padded_rows),
    "extra_head_hnd": ("HND", extra_head),
}


def decode(w, k, v, rule):
    shape = bd.shape_of(w.q, k, w.block_table, w.layout, v)
    dp = bd.plan_decode(w.seq_lens, shape, "cuda", rules=[rule])
    lens = torch.tensor(w.seq_lens, dtype=torch.int32, device="cuda")
    out = bd.paged_decode(w.q, k, v, w.block_table, lens, w.P, w.scale, plan=dp)
    torch.cuda.synchronize()
    assert bd.workspace_status(dp) == 0
    return out, dp


@pytest.mark.parametrize("plan", sorted(PLANS))
@pytest.mark.parametrize("view", sorted(VIEWS))
def test_pool_views_match_packed_pools_and_the_oracle(view, plan):
    layout, make = VIEWS[view]
    w = to_device(W.make_custom([1000, 4097, 77, 16, 0, 2500], 32, 8, 128, seed=150, poison=True, layout=layout))
    k, v = make(w.k_pool, w.v_pool)
    assert not k.is_contiguous()
    got, dp = decode(w, k, v, PLANS[plan])
    want, dq = decode(w, w.k_pool, w.v_pool, PLANS[plan])
    assert dp.plan.tuple() == dq.plan.tuple()
    assert torch.equal(got, want), f"{view}/{plan}: differs from the packed pools"
    assert_close(got.float().cpu().double().numpy(), oracle_full(w), f"{view}/{plan}")


def test_host_buffer_path_reads_a_combined_cache():
    w = to_device(W.make_custom([700, 33, 2049], 16, 4, 64, seed=151, poison=True))
    k, v = combined(w.k_pool, w.v_pool)
    shape = bd.shape_of(w.q, k, w.block_table, "HND", v)
    q_h = w.q.cpu().pin_memory()
    bt_h = w.block_table.cpu().pin_memory()
    lens_h = torch.tensor(w.seq_lens, dtype=torch.int32).pin_memory()
    out_h = torch.full_like(q_h, NAN).pin_memory()
    bd.decode_host(q_h, bt_h, lens_h, out_h, k, v, w.scale, shape)
    assert_close(out_h.float().double().numpy(), oracle_full(w), "host path, combined cache")


def test_device_tensors_of_the_wrong_type_are_refused_before_launch():
    w = to_device(W.make_custom([100, 200], 8, 2, 64, seed=152))
    shape = bd.shape_of(w.q, w.k_pool, w.block_table)
    dp = bd.plan_decode(w.seq_lens, shape, "cuda")
    with pytest.raises(TypeError):
        bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table,
                        torch.tensor(w.seq_lens, dtype=torch.int64, device="cuda"), 16, w.scale, plan=dp)
    with pytest.raises(ValueError):
        bd.paged_decode(w.q, w.k_pool, w.v_pool, w.block_table.cpu(),
                        torch.tensor(w.seq_lens, dtype=torch.int32, device="cuda"), 16, w.scale, plan=dp)
