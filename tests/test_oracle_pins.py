"""The CPU oracle against facts other than itself (no GPU)."""
import pytest

from oracle import oracle as O

from . import host_pins, oracle_pins

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")


@pytest.mark.parametrize("pin", oracle_pins.ATTENTION_PINS, ids=lambda f: f.__name__)
def test_attention_pin(olib, pin):
    pin(olib)


@pytest.mark.parametrize("pin", host_pins.HOST_PINS, ids=lambda f: f.__name__)
def test_host_pin(pin):
    pin(O)


def test_thread_count_does_not_change_result(olib):
    from paged_kv_gqa_17_b200 import workloads as W

    w = W.make_custom([300, 77, 1000], H_q=8, H_kv=2, D=64, seed=30, poison=True)
    pr = O.problem(w.q, w.k_pool, w.v_pool, w.block_table, w.seq_lens, w.scale)
    a = O.paged_decode(pr, n_threads=1)
    b = O.paged_decode(pr, n_threads=5)
    c = O.paged_decode_pairs(pr, [(2, 7), (0, 0), (1, 3)], n_threads=2)
    assert (a == b).all()
    assert (c[0] == a[2, 7]).all() and (c[1] == a[0, 0]).all() and (c[2] == a[1, 3]).all()


def test_oracle_rejects_bad_problems(olib):
    from paged_kv_gqa_17_b200 import workloads as W

    w = W.make_custom([40], H_q=4, H_kv=2, D=64, seed=31)
    pr = O.problem(w.q, w.k_pool, w.v_pool, w.block_table, w.seq_lens, w.scale)
    pr.seq_lens[0] = pr.max_pages * pr.P + 1  # longer than its block table
    with pytest.raises(ValueError):
        O.paged_decode(pr)
    with pytest.raises(ValueError):
        O.partial_state(pr, 0, 0, 0, 10**6)
