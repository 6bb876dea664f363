"""Pins of the speed-of-light formula and of the selector's argmin."""
import os

import pytest

from oracle import selector, sol

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "sol_example.txt")


def test_sol_worked_example():
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if line:
            rtt, store, want = map(float, line.split())
            assert sol.sol_latency(rtt, store) == pytest.approx(want, abs=1e-12)


def test_sol_rejects_negative():
    with pytest.raises(ValueError):
        sol.sol_latency(-1.0, 0.5)


def test_algorithmic_bytes_worked_examples():
    # 4 ranks x 2 KB, LL (expansion 2): 4 * (2 + 3*4 + 3*4 + 2) KB = 112 KB
    assert selector.algorithmic_bytes("ll", 1024, 4) == 112 * 1024
    # barrier oneshot: N (N + 1) S
    assert selector.algorithmic_bytes("barrier_oneshot", 1024, 4) == 4 * 5 * 2048
    # sentinel adds the reset: N (N - 1) S more than the same layout unreset
    s = 2048
    assert selector.algorithmic_bytes("sentinel", 1024, 4) == 4 * (s + 2 * 3 * s + s + 3 * s)
    # LL128 at 1 MB per rank, 8 ranks: lines of 60 elements, 128 bytes each
    count = 1 << 19
    lines = -(-count // 60)
    assert selector.algorithmic_bytes("ll128", count, 8) == 8 * (2 * count * 2 + 2 * 7 * 128 * lines)


NONE = [-1.0] * 24


def _tab(**pts):
    """table with p50 values at the given log2 sizes, e.g. _tab(b10=2.0)."""
    t = list(NONE)
    for k, v in pts.items():
        t[int(k[1:]) - 9] = v
    return t


def test_estimate_hand_examples():
    e = (0.0, 0.0, _tab(b10=2.0, b12=4.0, b14=10.0))
    # below the first measured size: held
    assert selector.estimate(e, "ll", 512, 4) == 2.0
    # exactly measured
    assert selector.estimate(e, "ll", 4096, 4) == 4.0
    # 2^11 is halfway (in log2) between 2^10 and 2^12: 3.0
    assert selector.estimate(e, "ll", 2048, 4) == pytest.approx(3.0)
    # 2^13 halfway between 2^12 (4) and 2^14 (10): 7.0
    assert selector.estimate(e, "ll", 8192, 4) == pytest.approx(7.0)
    # above the last: scaled by algorithmic bytes (sentinel-free LL: linear)
    b16 = selector.algorithmic_bytes("ll", 2 ** 15, 4)
    b14 = selector.algorithmic_bytes("ll", 2 ** 13, 4)
    assert selector.estimate(e, "ll", 2 ** 16, 4) == pytest.approx(10.0 * b16 / b14)
    # no table: alpha + beta * bytes
    assert selector.estimate((1.5, 1e-6, NONE), "ll", 1024, 4) == pytest.approx(
        1.5 + 1e-6 * selector.algorithmic_bytes("ll", 512, 4))
    assert selector.estimate((-1.0, 0.0, NONE), "ll", 1024, 4) is None


def test_choose_hand_examples():
    model = {"ll": (0.0, 0.0, _tab(b10=1.0, b20=50.0)),
             "barrier_twoshot": (0.0, 0.0, _tab(b10=5.0, b20=20.0))}
    assert selector.choose(model, 1024, 8) == "ll"
    assert selector.choose(model, 1 << 20, 8) == "barrier_twoshot"
    # crossing: ll 1 + 49 (k-1)/10, twoshot 5 + 15 (k-1)/10 -> equal at k = 1 + 4/34*10 (~2.18)
    assert selector.choose(model, 2 ** 11, 8) == "ll"
    assert selector.choose(model, 2 ** 12, 8) == "barrier_twoshot"


def test_choose_tie_breaks_on_bytes_then_order():
    flat = (0.0, 0.0, _tab(b12=3.0))
    # equal estimates: fewer bytes wins (sentinel moves fewer than LL)
    assert selector.choose({"ll": flat, "sentinel": flat}, 4096, 4) == "sentinel"
    assert selector.TIE_ORDER[0] == "sentinel"


def test_twoshot_never_chosen_for_allgather():
    model = {"barrier_twoshot": (0.0, 0.0, _tab(b10=0.1)), "ll": (0.0, 0.0, _tab(b10=5.0))}
    assert selector.choose(model, 1024, 4, op="allgather") == "ll"
