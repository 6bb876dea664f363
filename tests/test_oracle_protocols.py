"""Pins of the protocol simulator: exhaustive enumeration, schedules, planted bugs."""
import numpy as np
import pytest

from latency_self_synchronizing_b200.inputs import make_inputs
from oracle import exhaustive, protocols as P, simulator as S

SELF = list(P.SELF_SYNC)


def _x(seed, k, n, c):
    return make_inputs(seed=seed, k_ops=k, nranks=n, count=c)


@pytest.mark.parametrize("proto", SELF)
@pytest.mark.parametrize("n", [2, 3])
def test_every_landing_subset(proto, n):
    # 8 elements, except sentinel at N=3 (16 units -> 65536 subsets per
    # receiver and epoch) which uses 6 elements to keep the suite short
    count = 6 if (proto == P.SENTINEL and n == 3) else 8
    x = _x(11, 3, n, count)
    for epoch in (1, 2, 3, 4):
        stale = x[2] if epoch > 2 else None
        checked, v = exhaustive.landing_subsets(proto, x[epoch % 2], epoch, stale_inputs=stale)
        assert not v, v[:3]
        assert checked >= n


def test_landing_subsets_catch_missing_sentinel_reset():
    x = _x(12, 3, 2, 8)
    _, v = exhaustive.landing_subsets(P.SENTINEL, x[0], 3, stale_inputs=x[1], bug="no_reset")
    assert v


def test_ll_flag_from_two_epochs_ago_is_rejected():
    data = _x(13, 1, 1, 8)[0, 0]
    slot = P.initial_slot(P.LL, 8)
    for off, body in P.encode_all(P.LL, data, 5):
        slot[off:off + body.size] = body
    assert all(P.validate_unit(P.LL, slot, j, 5) for j in range(4))
    assert not any(P.validate_unit(P.LL, slot, j, 7) for j in range(4))
    assert not any(P.validate_unit(P.LL, P.initial_slot(P.LL, 8), j, 1) for j in range(4))


def test_encodings_layout():
    data = np.arange(1, 62, dtype=np.uint16)  # 61 elements: 2 LL128 lines, odd LL
    assert P.slot_bytes(P.LL, 61) == 8 * 31
    assert P.slot_bytes(P.LL128, 61) == 256
    assert P.slot_bytes(P.SENTINEL, 61) == 122
    off, body = P.encode_unit(P.LL, data, 30, 9)  # last LL unit: element 60 + pad
    assert off == 240 and list(body) == [61, 0, 0, 0, 9, 0, 0, 0]
    off, body = P.encode_unit(P.LL128, data, 1, 9)  # second line: element 60 + pad
    assert off == 128 and body[0] == 61 and not body[2:120].any()
    assert list(body[120:]) == [9, 0, 0, 0, 0, 0, 0, 0]
    assert P.expansion(P.LL, 1024) == 2.0
    assert abs(P.expansion(P.LL128, 60 * 1000) - 128 / 120) < 1e-12


def test_arrival_orders_all_ranks_identical():
    golden = np.array([[0x3F80], [0x33C0], [0xBF80]], dtype=np.uint16)  # order-sensitive
    combos, v = exhaustive.arrival_orders(golden)
    assert combos == 6 ** 3 and not v
    _, v = exhaustive.arrival_orders(golden, bug="arrival_order")
    assert v
    combos, v = exhaustive.arrival_orders(_x(14, 1, 2, 16)[0])
    assert combos == 4 and not v


@pytest.mark.parametrize("proto", SELF + [S.BARRIER_ONESHOT, S.BARRIER_TWOSHOT])
def test_every_interleaving_two_ranks(proto):
    x = _x(15, 3, 2, 2)
    states, v = exhaustive.explore_interleavings(proto, x)
    assert not v, v[:3]
    assert states > 10


@pytest.mark.parametrize("proto", SELF)
def test_every_interleaving_three_ranks_one_element(proto):
    x = _x(16, 2, 3, 1)
    states, v = exhaustive.explore_interleavings(proto, x, max_states=400_000)
    assert not v, v[:3]


@pytest.mark.parametrize("proto,bug", [
    ("ll", "single_buffer"), ("ll128", "single_buffer"), ("sentinel", "single_buffer"),
    ("sentinel", "no_reset"),
    ("barrier_oneshot", "no_bottom_barrier"), ("barrier_oneshot", "no_top_barrier"),
    ("barrier_twoshot", "no_mid_barrier"),
])
def test_interleaving_search_finds_planted_bug(proto, bug):
    x = _x(17, 3, 2, 2)
    _, v = exhaustive.explore_interleavings(proto, x, bug=bug)
    assert v


@pytest.mark.parametrize("proto", SELF + [S.BARRIER_ONESHOT, S.BARRIER_TWOSHOT])
@pytest.mark.parametrize("n", [2, 3, 5, 8])
def test_random_and_adversarial_schedules(proto, n):
    count = 61 if proto != P.SENTINEL else 13
    x = _x(100 + n, 3, n, count)
    for seed in range(2):
        _, v = S.run_chain(proto, x, seed=seed)
        assert not v, v[:3]
    _, v = S.run_chain(proto, x, seed=7, schedule="adversarial", slow_rank=n - 1)
    assert not v, v[:3]


@pytest.mark.parametrize("proto", SELF + [S.BARRIER_ONESHOT])
def test_allgather_schedules(proto):
    x = _x(21, 3, 4, 9)
    _, v = S.run_chain(proto, x, op="allgather", seed=3)
    assert not v, v[:3]
    _, v = S.run_chain(proto, x, op="allgather", seed=4, schedule="adversarial", slow_rank=0)
    assert not v, v[:3]


def test_arrival_order_bug_caught_by_simulator():
    x = np.zeros((2, 3, 1), dtype=np.uint16)
    x[:, :, 0] = [0x3F80, 0x33C0, 0xBF80]
    found = False
    for seed in range(30):
        _, v = S.run_chain(P.LL, x, seed=seed, bug="arrival_order")
        found |= bool(v)
    assert found


def test_first_epoch_and_parity_offset():
    x = _x(22, 4, 3, 5)
    _, v = S.run_chain(P.LL, x, first_epoch=1000, seed=1)
    assert not v


@pytest.mark.parametrize("proto", SELF + [S.BARRIER_ONESHOT, S.BARRIER_TWOSHOT])
def test_fifo_schedule_for_large_inputs(proto):
    x = _x(23, 2, 4, 300)
    _, v = S.run_fifo(proto, x)
    assert not v, v[:3]


@pytest.mark.parametrize("n,count,k", [(2, 2, 3), (3, 1, 2)])
def test_sentinel_reset_on_accept_every_interleaving(n, count, k):
    """The sentinel variant that writes the fill back in the same atomic step
    that accepts a unit (no separate reset pass) is as safe as resetting after
    the whole epoch: every interleaving, no violation."""
    x = _x(31 + n, k, n, count)
    states, v = exhaustive.explore_interleavings(P.SENTINEL, x, sentinel_reset="on_accept", max_states=400_000)
    assert not v, v[:3]
    _, v = exhaustive.explore_interleavings(P.SENTINEL, x, sentinel_reset="on_accept", bug="no_reset")
    assert v


@pytest.mark.parametrize("n", [2, 4, 8])
def test_sentinel_reset_on_accept_schedules(n):
    x = _x(40 + n, 3, n, 13)
    for seed in range(2):
        _, v = S.run_chain(P.SENTINEL, x, seed=seed, sentinel_reset="on_accept")
        assert not v, v[:3]
    _, v = S.run_chain(P.SENTINEL, x, seed=5, schedule="adversarial", slow_rank=0, sentinel_reset="on_accept")
    assert not v, v[:3]


@pytest.mark.parametrize("proto", ["ll_twoshot", "sentinel_twoshot"])
@pytest.mark.parametrize("n,count,k", [(2, 2, 3), (2, 4, 2)])
def test_selfsync_twoshot_every_interleaving(proto, n, count, k):
    """Reduce-scatter + all-gather, both self-synchronizing: every interleaving
    at two ranks (one-element shards so that every shard carries data)."""
    x = _x(50 + count, k, n, count)
    states, v = exhaustive.explore_interleavings(proto, x, max_states=200_000, vector=1)
    assert not v, v[:3]
    assert states > 10


def test_selfsync_twoshot_catches_missing_reset():
    x = _x(55, 3, 2, 2)
    _, v = exhaustive.explore_interleavings("sentinel_twoshot", x, bug="no_reset", vector=1)
    assert v


@pytest.mark.parametrize("proto", ["ll_twoshot", "sentinel_twoshot"])
@pytest.mark.parametrize("n", [2, 3, 5, 8])
def test_selfsync_twoshot_schedules(proto, n):
    x = _x(60 + n, 3, n, 100)  # vector-aligned shards as on the GPU, a ragged tail
    for seed in range(2):
        _, v = S.run_chain(proto, x, seed=seed)
        assert not v, v[:3]
    _, v = S.run_chain(proto, x, seed=9, schedule="adversarial", slow_rank=n - 1,
                       sentinel_reset="on_accept")
    assert not v, v[:3]


def test_oneshot_dual_buffer_every_interleaving_and_single_buffer_bug():
    """SiFAR's dual-buffered oneshot needs no bottom barrier; with one input
    buffer and no bottom barrier a fast rank overwrites an input a slow rank
    still pulls."""
    x = _x(70, 3, 2, 2)
    states, v = exhaustive.explore_interleavings("barrier_oneshot_db", x)
    assert not v and states > 10
    _, v = exhaustive.explore_interleavings("barrier_oneshot_db", x, bug="single_input_buffer")
    assert v
    for n in (3, 5, 8):
        y = _x(71, 4, n, 13)
        assert not S.run_chain("barrier_oneshot_db", y, seed=1)[1]
        assert not S.run_chain("barrier_oneshot_db", y, op="allgather", seed=2, schedule="adversarial",
                               slow_rank=0)[1]
