"""CPU-only checks of the C ABI: the library loads, exports every declared
symbol, and its host-side logic (selector, algorithmic bytes, status names)
agrees with the oracle's plain restatement. No kernel is launched."""
import os
import re

import pytest

from latency_self_synchronizing_b200 import _lib, api
from oracle import selector as osel

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "sfc.h")
PROTO_NAMES = {1: "ll", 2: "ll128", 3: "sentinel", 4: "barrier_oneshot", 5: "barrier_twoshot"}


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sfc_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    names = _declared()
    assert len(names) >= 20
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == {s[0] for s in _lib.SIGNATURES}


def test_status_strings():
    for s in api.Status:
        assert api.status_string(s)
    assert api.status_string(3) == "device wait timed out"


@pytest.mark.parametrize("op", ["allreduce", "allgather"])
@pytest.mark.parametrize("n", [2, 3, 4, 8])
def test_algorithmic_bytes_match_oracle(op, n):
    for count in [1, 7, 60, 61, 1024, 8192 * 8, 1 << 20, (1 << 25) + 3]:
        for p, name in PROTO_NAMES.items():
            if op == "allgather" and p == 5:
                assert api.algorithmic_bytes(op, p, count, n) == -1.0
                continue
            assert api.algorithmic_bytes(op, p, count, n) == pytest.approx(
                osel.algorithmic_bytes(name, count, n, op), rel=1e-12)


def _model_from(coeffs):
    m = api.default_cost_model()
    for op in range(2):
        for p in range(6):
            for n in range(9):
                m.c[op][p][n].alpha_us = -1.0
                m.c[op][p][n].beta_us_per_byte = 0.0
    for op in range(2):
        for p, name in PROTO_NAMES.items():
            if name in coeffs:
                for n in range(2, 9):
                    m.c[op][p][n].alpha_us, m.c[op][p][n].beta_us_per_byte = coeffs[name]
    return m


def test_selector_matches_oracle_argmin():
    coeffs = {"ll": (1.2, 1.0 / 3e6), "ll128": (2.0, 1.0 / 5e6), "sentinel": (2.6, 1.0 / 6e6),
              "barrier_oneshot": (3.5, 1.0 / 6e6), "barrier_twoshot": (5.0, 1.0 / 6.5e6)}
    m = _model_from(coeffs)
    for op in ("allreduce", "allgather"):
        for n in (2, 4, 8):
            for b in [1024 << i for i in range(17)]:
                got = api.select_protocol_model(m, op, b, n)
                want = osel.choose(coeffs, b // 2, n, op)
                assert PROTO_NAMES[int(got)] == want, (op, n, b)


def test_selector_ties_prefer_fewer_bytes():
    m = _model_from({"ll": (1.0, 0.0), "sentinel": (1.0, 0.0)})
    assert api.select_protocol_model(m, "allreduce", 4096, 4) == api.Protocol.SENTINEL


def test_default_model_chooses_a_real_protocol_everywhere():
    m = api.default_cost_model()
    for op in ("allreduce", "allgather"):
        for n in range(2, 9):
            for b in [1024 << i for i in range(17)]:
                p = api.select_protocol_model(m, op, b, n)
                assert p != api.Protocol.AUTO
                if op == "allgather":
                    assert p != api.Protocol.BARRIER_TWOSHOT
