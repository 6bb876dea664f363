"""The latency floor microbenchmark (sfc_measure_floor): the fixed SM set,
every (pair, flag address) trial, and the order of its statistics."""
import pytest

from latency_self_synchronizing_b200 import _lib, api

pytestmark = pytest.mark.gpu


def test_floor_trials_and_statistics():
    f = api.measure_floor(200)
    n = _lib.SFC_FLOOR_SMS
    assert f["pairs"] == n * n * _lib.SFC_FLOOR_LOCATIONS
    ini, rsp = f["initiator_sm"], f["responder_sm"]
    assert len(set(ini + rsp)) == 2 * n
    merged = [x for pair in zip(ini, rsp) for x in pair]
    assert merged == sorted(merged)  # spread evenly over the sorted SM ids, alternating
    assert 0 < f["flag_rtt_ns_min_pair"] <= f["flag_rtt_ns_p10"] <= f["flag_rtt_ns_p50"]
    assert f["flag_rtt_ns_p50"] <= f["flag_rtt_ns_p90"] <= f["flag_rtt_ns_max_pair"]
    assert all(v > 0 for v in f["flag_rtt_ns_by_location"])
    # a round trip is two one-way trips through L2: longer than one L2 hit
    assert f["flag_rtt_ns_p50"] > f["l2_rtt_ns_p50"] > 0
    assert 0.5 < f["sm_clock_ghz"] < 3.0
    assert f["globaltimer_step_ns"] > 0


def test_floor_is_reproducible_within_a_process():
    a = api.measure_floor(300)["flag_rtt_ns_p50"]
    b = api.measure_floor(300)["flag_rtt_ns_p50"]
    assert abs(a - b) <= 0.25 * max(a, b)
