"""The binding's argument marshalling on the CPU: pool strides read from the
tensors (views into combined or padded caches), and tensors of the wrong
type, layout or device rejected before anything reaches the library."""
import ctypes

import pytest
import torch

from paged_kv_gqa_17_b200 import binding as bd

BF16 = torch.bfloat16


@pytest.fixture(scope="module")
def L():
    from paged_kv_gqa_17_b200 import build

    build.build()
    return bd.lib()


def strides(s):
    return (s.kv_stride_page, s.kv_stride_head, s.kv_stride_token)


def test_contiguous_pools_give_the_packed_strides():
    q = torch.zeros(3, 32, 128, dtype=BF16)
    bt = torch.zeros(3, 9, dtype=torch.int32)
    for layout, pool in (("HND", torch.zeros(40, 8, 16, 128, dtype=BF16)),
                         ("NHD", torch.zeros(40, 16, 8, 128, dtype=BF16))):
        got = bd.shape_of(q, pool, bt, layout)
        want = bd.make_shape(3, 32, 8, 128, 16, 9, 40, layout)
        assert bytes(got) == bytes(want), layout


def test_views_into_a_combined_cache_keep_their_strides():
    H, P, D, pages = 8, 16, 128, 40
    q = torch.zeros(2, 32, D, dtype=BF16)
    bt = torch.zeros(2, 5, dtype=torch.int32)
    kv = torch.zeros(pages, 2, H, P, D, dtype=BF16)             # HND halves side by side
    s = bd.shape_of(q, kv[:, 0], bt, "HND", kv[:, 1])
    assert strides(s) == (2 * H * P * D, P * D, D) and s.num_pool_pages == pages
    kv = torch.zeros(pages, 2, P, H, D, dtype=BF16)             # NHD halves side by side
    s = bd.shape_of(q, kv[:, 0], bt, "NHD", kv[:, 1])
    assert strides(s) == (2 * P * H * D, D, H * D)
    padded = torch.zeros(pages, H, P, D + 8, dtype=BF16)        # rows padded past head_dim
    s = bd.shape_of(q, padded[..., :D], bt, "HND")
    assert strides(s) == (H * P * (D + 8), P * (D + 8), D + 8)
    wide = torch.zeros(pages, H + 1, P, D, dtype=BF16)          # an extra head per page
    s = bd.shape_of(q, wide[:, :H], bt, "HND")
    assert strides(s) == ((H + 1) * P * D, P * D, D)


def test_unit_axes_take_the_packed_stride():
    q = torch.zeros(1, 4, 64, dtype=BF16)
    bt = torch.zeros(1, 1, dtype=torch.int32)
    base = torch.zeros(2, 3, 16, 64, dtype=BF16)
    one = base[:1, 1:2]                                          # 1 page, 1 head, odd strides on both
    s = bd.shape_of(q, one, bt, "HND")
    assert strides(s) == (16 * 64, 16 * 64, 64)


def test_shape_of_rejects_pools_it_cannot_describe():
    q = torch.zeros(1, 4, 64, dtype=BF16)
    bt = torch.zeros(1, 4, dtype=torch.int32)
    k = torch.zeros(8, 1, 16, 64, dtype=BF16)
    with pytest.raises(ValueError):
        bd.shape_of(q, k.transpose(2, 3).contiguous().transpose(2, 3), bt)   # head_dim not contiguous
    with pytest.raises(ValueError):
        bd.shape_of(q, k, bt, "HND", torch.zeros(8, 1, 16, 72, dtype=BF16)[..., :64])  # V strides differ
    with pytest.raises(ValueError):
        bd.shape_of(q, k[0], bt)                                               # not 4-D
    with pytest.raises(ValueError):
        bd.shape_of(q, k, bt, "DHN")


def _args(B=2, H_q=8, H_kv=2, D=64, pages=10, max_pages=4):
    q = torch.zeros(B, H_q, D, dtype=BF16)
    k = torch.zeros(pages, H_kv, 16, D, dtype=BF16)
    v = torch.zeros_like(k)
    bt = torch.zeros(B, max_pages, dtype=torch.int32)
    lens = torch.zeros(B, dtype=torch.int32)
    return dict(q=q, k_pool=k, v_pool=v, block_table=bt, seq_lens=lens)


def _plan(a):
    shape = bd.shape_of(a["q"], a["k_pool"], a["block_table"])
    return bd.DecodePlan(shape, bd.Plan(0, 1, 0, 0), None, None, 0, torch.zeros(4096, dtype=torch.uint8), {})


def _decode(a, plan, out=None):
    return bd.paged_decode(a["q"], a["k_pool"], a["v_pool"], a["block_table"], a["seq_lens"], 16, 0.125,
                           plan=plan, out=out)


@pytest.mark.parametrize("bad, exc", [
    (dict(q=torch.zeros(2, 8, 64, dtype=torch.float16)), TypeError),
    (dict(k_pool=torch.zeros(10, 2, 16, 64, dtype=torch.float32)), TypeError),
    (dict(seq_lens=torch.zeros(2, dtype=torch.int64)), TypeError),
    (dict(block_table=torch.zeros(2, 4, dtype=torch.int64)), TypeError),
    (dict(q=torch.zeros(8, 2, 64, dtype=BF16).transpose(0, 1)), ValueError),       # not contiguous
    (dict(block_table=torch.zeros(4, 2, dtype=torch.int32).t()), ValueError),      # not contiguous
    (dict(block_table=torch.zeros(2, 5, dtype=torch.int32)), ValueError),          # other table width
    (dict(seq_lens=torch.zeros(1, dtype=torch.int32)), ValueError),                # too few lengths
    (dict(v_pool=torch.zeros(10, 2, 16, 72, dtype=BF16)[..., :64]), ValueError),   # V strides differ
    (dict(k_pool=torch.zeros(9, 2, 16, 64, dtype=BF16),
          v_pool=torch.zeros(9, 2, 16, 64, dtype=BF16)), ValueError),              # fewer pages than planned
    (dict(k_pool=torch.zeros(10, 3, 16, 64, dtype=BF16)[:, :2],
          v_pool=torch.zeros(10, 3, 16, 64, dtype=BF16)[:, :2]), ValueError),      # other page stride
    ({}, ValueError),                                                              # host tensors
])
def test_paged_decode_rejects_mismatched_tensors(L, bad, exc):
    a = _args()
    plan = _plan(a)
    a.update(bad)
    with pytest.raises(exc):
        _decode(a, plan)


def test_paged_decode_rejects_a_mismatched_out(L):
    a = _args()
    plan = _plan(a)
    with pytest.raises(ValueError):
        _decode(a, plan, out=torch.zeros(2, 8, 32, dtype=BF16))
    with pytest.raises(TypeError):
        _decode(a, plan, out=torch.zeros(2, 8, 64, dtype=torch.float32))


def test_combined_check_passes_exactly_the_calls_the_itemised_checks_pass(L, monkeypatch):
    """The one-expression test that passes well-formed calls and the itemised
    checks that name a problem agree: with every tensor taken to be on device
    0, the valid call passes the combined test, and each malformed one fails it
    and gets a specific error from the itemised checks."""
    monkeypatch.setattr(torch.Tensor, "get_device", lambda self: 0)
    a = _args()
    plan = _plan(a)
    out = torch.zeros(2, 8, 64, dtype=BF16)
    assert bd._check_decode_tensors(a["q"], a["k_pool"], a["v_pool"], a["block_table"], a["seq_lens"], out,
                                    plan.shape) is None
    bad_cases = [
        dict(q=torch.zeros(2, 8, 64, dtype=torch.float16)),
        dict(seq_lens=torch.zeros(2, dtype=torch.int64)),
        dict(q=torch.zeros(8, 2, 64, dtype=BF16).transpose(0, 1)),
        dict(block_table=torch.zeros(2, 5, dtype=torch.int32)),
        dict(seq_lens=torch.zeros(1, dtype=torch.int32)),
        dict(v_pool=torch.zeros(10, 2, 16, 72, dtype=BF16)[..., :64]),
        dict(k_pool=torch.zeros(9, 2, 16, 64, dtype=BF16), v_pool=torch.zeros(9, 2, 16, 64, dtype=BF16)),
        dict(k_pool=torch.zeros(10, 3, 16, 64, dtype=BF16)[:, :2], v_pool=torch.zeros(10, 3, 16, 64, dtype=BF16)[:, :2]),
        dict(k_pool=torch.zeros(10, 2, 64, 16, dtype=BF16).transpose(2, 3),
             v_pool=torch.zeros(10, 2, 64, 16, dtype=BF16).transpose(2, 3)),
        dict(k_pool=torch.zeros(10, 2, 16, 64, dtype=BF16)[0], v_pool=torch.zeros(10, 2, 16, 64, dtype=BF16)[0]),
    ]
    for bad in bad_cases:
        b = dict(a, **bad)
        args = (b["q"], b["k_pool"], b["v_pool"], b["block_table"], b["seq_lens"], out, plan.shape)
        with pytest.raises((TypeError, ValueError)) as e:
            bd._diagnose_decode_tensors(*args)
        assert "CUDA device" not in str(e.value), (bad, e.value)   # named before the device check
        with pytest.raises((TypeError, ValueError)):
            bd._check_decode_tensors(*args)


def _host_args(B=2, H_q=8, H_kv=2, D=64, pages=10, max_pages=4):
    a = _args(B, H_q, H_kv, D, pages, max_pages)
    shape = bd.shape_of(a["q"], a["k_pool"], a["block_table"])
    return dict(q_host=a["q"], block_table_host=a["block_table"], seq_lens_host=a["seq_lens"],
                out_host=torch.zeros_like(a["q"]), k_pool=a["k_pool"], v_pool=a["v_pool"]), shape


@pytest.mark.parametrize("bad, exc", [
    (dict(q_host=torch.zeros(2, 8, 64, dtype=torch.float16)), TypeError),
    (dict(q_host=torch.zeros(2, 8, 32, dtype=BF16)), ValueError),                 # too small: would overrun
    (dict(out_host=torch.zeros(1, 8, 64, dtype=BF16)), ValueError),
    (dict(out_host=torch.zeros(8, 2, 64, dtype=BF16).transpose(0, 1)), ValueError),
    (dict(block_table_host=torch.zeros(2, 3, dtype=torch.int32)), ValueError),
    (dict(block_table_host=torch.zeros(2, 4, dtype=torch.int64)), TypeError),
    (dict(seq_lens_host=torch.zeros(1, dtype=torch.int32)), ValueError),
    (dict(k_pool=torch.zeros(9, 2, 16, 64, dtype=BF16), v_pool=torch.zeros(9, 2, 16, 64, dtype=BF16)), ValueError),
    (dict(v_pool=torch.zeros(10, 2, 16, 64, dtype=torch.float32)), TypeError),
])
def test_host_call_checks_name_each_problem(monkeypatch, bad, exc):
    monkeypatch.setattr(torch.Tensor, "get_device", lambda self: 0)   # pools "on" cuda:0
    a, shape = _host_args()
    bd._check_host_call(**a, shape=shape, device_index=0)             # the well-formed call passes
    a.update(bad)
    with pytest.raises(exc):
        bd._check_host_call(**a, shape=shape, device_index=0)


def test_host_call_rejects_pools_off_the_decoders_device():
    a, shape = _host_args()                                           # CPU pools: get_device() == -1
    with pytest.raises(ValueError):
        bd._check_host_call(**a, shape=shape, device_index=0)


def test_host_decoder_checks_each_new_tensor_object_once(monkeypatch):
    """A HostDecoder checks a call's tensors when it first sees them; repeated
    calls with the same objects skip straight to the library, and a new object
    (or shape) is checked again before the library is reached."""
    monkeypatch.setattr(torch.Tensor, "get_device", lambda self: 0)
    checks, calls = [], []
    real = bd._check_host_call
    monkeypatch.setattr(bd, "_check_host_call", lambda *x, **k: (checks.append(1), real(*x, **k)))
    dec = object.__new__(bd.HostDecoder)                              # no CUDA here: set the fields by hand
    dec.dev = torch.zeros(1, dtype=torch.uint8)
    dec._stream, dec._bufs, dec._checked = 0, (0, 0, 0, 0), ()
    dec._plan = bd.Plan()
    dec._plan_ref = ctypes.byref(dec._plan)
    dec._fn = lambda *x: (calls.append(1), 0)[1]
    dec._fn_call = lambda ref: (calls.append(1), 0)[1]             # repeated calls: the parameter block
    dec._call = bd.HostCall()
    dec._call_ref = ctypes.byref(dec._call)
    a, shape = _host_args()
    args = [a[k] for k in ("q_host", "block_table_host", "seq_lens_host", "out_host", "k_pool", "v_pool")]

    def call(q=None, shp=None):
        dec(q if q is not None else args[0], *args[1:4], args[4], args[5], 0.125, shp or shape)

    call()
    call()
    call()
    assert len(checks) == 1 and len(calls) == 3
    assert dec._call.q_host == args[0].data_ptr() and dec._call.v_pool == args[5].data_ptr()
    assert dec._call.scale == 0.125 and dec._call.shape == ctypes.addressof(shape)
    call(q=args[0].clone())                                           # a new q object
    assert len(checks) == 2
    call(shp=bd.shape_of(a["q_host"], a["k_pool"], a["block_table_host"]))   # a new shape object
    assert len(checks) == 3 and len(calls) == 5
    with pytest.raises(ValueError):
        call(q=torch.zeros(2, 8, 32, dtype=BF16))                     # too small: stopped before the library
    assert len(calls) == 5
