"""CPU-only checks of the C ABI: the library loads, exports every declared
symbol, and its host-side logic (selector, algorithmic bytes, status names)
agrees with the oracle's plain restatement. No kernel is launched."""
import os
import re

import numpy as np
import pytest

from latency_self_synchronizing_b200 import _lib, api
from oracle import selector as osel

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "sfc.h")
PROTO_NAMES = {1: "ll", 2: "ll128", 3: "sentinel", 4: "barrier_oneshot", 5: "barrier_twoshot",
               6: "barrier_oneshot_db", 7: "ll_twoshot", 8: "sentinel_twoshot", 9: "ll128_fast"}
AR_ONLY = {5, 7, 8}


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


def test_debug_library_exports_the_same_symbols():
    """The bounds-checked build (built by __graft_entry__.build) is the same ABI."""
    import ctypes
    path = os.path.join(os.path.dirname(_lib.LIB_PATH), "libsfc_debug.so")
    if not os.path.exists(path):
        pytest.skip("libsfc_debug.so not built")
    lib = ctypes.CDLL(path)
    for n in _declared():
        assert hasattr(lib, n), n


def test_status_strings():
    for s in api.Status:
        assert api.status_string(s)
    assert api.status_string(3) == "device wait timed out"


@pytest.mark.parametrize("op", ["allreduce", "allgather"])
@pytest.mark.parametrize("n", [2, 3, 4, 8])
def test_algorithmic_bytes_match_oracle(op, n):
    for count in [1, 7, 60, 61, 1024, 8192 * 8, 1 << 20, (1 << 25) + 3]:
        for p, name in PROTO_NAMES.items():
            if op == "allgather" and p in AR_ONLY:
                assert api.algorithmic_bytes(op, p, count, n) == -1.0
                continue
            assert api.algorithmic_bytes(op, p, count, n) == pytest.approx(
                osel.algorithmic_bytes(name, count, n, op), rel=1e-12)


def _model_from(entries):
    """ctypes model from {proto: (alpha, beta, table)}; other protocols off."""
    m = api.default_cost_model()
    for op in range(2):
        for p in range(10):
            for n in range(9):
                m.c[op][p][n].alpha_us = -1.0
    for op in range(2):
        for p, name in PROTO_NAMES.items():
            if name in entries:
                a, b, tab = entries[name]
                for n in range(2, 9):
                    e = m.c[op][p][n]
                    e.alpha_us, e.beta_us_per_byte = a, b
                    for i in range(24):
                        e.table_us[i] = tab[i]
    return m


def _random_entries(rng):
    out = {}
    for name in PROTO_NAMES.values():
        tab = [-1.0] * 24
        for i in sorted(rng.choice(24, size=rng.integers(0, 8), replace=False)):
            tab[i] = float(rng.uniform(0.5, 500.0))
        out[name] = (float(rng.uniform(0, 5)), float(rng.uniform(0, 1e-6)), tab)
    return out


def test_cost_estimate_and_selector_match_oracle():
    rng = np.random.default_rng(0)
    sizes = [512 << i for i in range(20)] + [3000, 70000, 5_000_000, 1 << 33]
    for trial in range(20):
        entries = _random_entries(rng)
        m = _model_from(entries)
        for op in ("allreduce", "allgather"):
            for n in (2, 5, 8):
                for b in sizes:
                    for p, name in PROTO_NAMES.items():
                        if op == "allgather" and p in AR_ONLY:
                            continue
                        want = osel.estimate(entries[name], name, b, n, op)
                        got = api.cost_estimate(m, op, p, b, n)
                        assert got == pytest.approx(want, rel=1e-9), (trial, op, n, b, name)
                    got = api.select_protocol_model(m, op, b, n)
                    assert PROTO_NAMES[int(got)] == osel.choose(entries, b, n, op), (trial, op, n, b)


def test_selector_ties_prefer_fewer_bytes():
    flat = (0.0, 0.0, [2.0] + [-1.0] * 23)
    m = _model_from({"ll": flat, "sentinel": flat})
    assert api.select_protocol_model(m, "allreduce", 4096, 4) == api.Protocol.SENTINEL


def test_default_model_chooses_a_real_protocol_everywhere():
    m = api.default_cost_model()
    for op in ("allreduce", "allgather"):
        for n in range(2, 9):
            for b in [512 << i for i in range(20)]:
                p = api.select_protocol_model(m, op, b, n)
                assert p != api.Protocol.AUTO
                assert p != api.Protocol.LL128_FAST  # opt-in only
                if op == "allgather":
                    assert int(p) not in AR_ONLY


def test_one_load_ll128_is_opt_in():
    """The built-in model carries the one-load LL128's measured latencies but
    marks it unavailable; turning its entries on lets the selector take it
    where it measured fastest (eight ranks, 64 KiB per rank)."""
    m = api.default_cost_model()
    op, n, b = "allreduce", 8, 64 << 10
    e = m.c[int(api.as_op(op))][int(api.Protocol.LL128_FAST)][n]
    assert e.alpha_us < 0 and e.table_us[16 - 9] > 0  # 2^16 bytes measured
    assert api.cost_estimate(m, op, "ll128_fast", b, n) < 0
    assert api.select_protocol_model(m, op, b, n) != api.Protocol.LL128_FAST
    e.alpha_us = 0.0
    t_fast = api.cost_estimate(m, op, "ll128_fast", b, n)
    assert t_fast > 0
    assert all(t_fast < api.cost_estimate(m, op, p, b, n) for p in ("ll", "ll128", "sentinel"))
    assert api.select_protocol_model(m, op, b, n) == api.Protocol.LL128_FAST



def _prototypes():
    """name -> parameter count of every function the header declares."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"\b(sfc_[a-z_0-9]+)\s*\(([^;{]*?)\)\s*;", text):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_signatures_match_the_header():
    """Every ctypes signature has as many arguments as the C prototype."""
    protos = _prototypes()
    for name, _, args in _lib.SIGNATURES:
        assert name in protos, name
        assert len(args) == protos[name], (name, len(args), protos[name])


def _struct_fields(name):
    """Member names of `typedef struct { ... } name;` in declaration order."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    m = re.search(r"typedef struct \{([^}]*)\}\s*" + name + r";", text)
    assert m, name
    names = []
    for decl in m.group(1).split(";"):
        decl = re.sub(r"\[[^\]]*\]", "", decl).strip()
        if decl:
            first, *rest = decl.split(",")
            names.append(first.split()[-1].lstrip("*"))
            names += [r.strip().lstrip("*") for r in rest]
    return names


@pytest.mark.parametrize("cname,pyname", [("sfc_config", "Config"), ("sfc_cost_entry", "CostEntry"),
                                           ("sfc_floor_result", "FloorResult"), ("sfc_ll_view", "LLView")])
def test_binding_structs_match_the_header(cname, pyname):
    py = [f[0] for f in getattr(_lib, pyname)._fields_]
    assert _struct_fields(cname) == py


def _bare_communicator(n=2):
    """A Communicator with no context behind it: enough to reach the
    argument checks that run before any library call."""
    from latency_self_synchronizing_b200 import api

    class NoCalls:
        def __getattr__(self, name):
            def call(*args):
                raise AssertionError(f"{name} reached the library")
            call.__name__ = name
            return call

    c = api.Communicator.__new__(api.Communicator)
    c.nranks, c._device, c._ctx, c._lib = n, 0, None, NoCalls()
    c._ptrs_in, c._ptrs_out = [None] * n, [None] * n
    c._last, c._plans = None, []
    return c


def test_chain_rejects_host_tensors_the_kernel_would_dereference():
    """Pointer tables, skews and timing buffers are read or written by the
    GPU itself: host tensors are refused before anything is launched."""
    import torch

    c = _bare_communicator(2)
    table = torch.zeros(2 * 3, dtype=torch.int64)  # host memory
    with pytest.raises(ValueError, match="in_table"):
        c.allreduce_chain(table, table, 8, 3, protocol="ll")
    with pytest.raises(ValueError, match="timings"):
        c._timings_ptr(torch.zeros(4, dtype=torch.int64), 3)
    with pytest.raises(ValueError, match="skew_ns"):
        c._device_tensor(torch.zeros(6, dtype=torch.int32), (torch.int32,), 6, True, "skew_ns")
    assert c._timings_ptr(None, 3) is None


def test_host_chain_rejects_bad_host_operands():
    import torch

    c = _bare_communicator(2)
    good = torch.zeros(3, 2, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="in_host"):
        c.allreduce_chain_host(torch.zeros(3, 2, 8, dtype=torch.float32), good)
    with pytest.raises(ValueError, match="shape"):
        c.allreduce_chain_host(good, torch.zeros(3, 2, 9, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="timings"):
        c.allreduce_chain_host(good, good.clone(), timings=torch.zeros(4, dtype=torch.int64))


def test_single_ops_and_linear_reject_host_operands():
    import torch

    c = _bare_communicator(2)
    x = [torch.zeros(8, dtype=torch.bfloat16) for _ in range(2)]
    with pytest.raises(TypeError, match="CUDA"):
        c.allreduce(x, [t.clone() for t in x], protocol="ll")
    w = [torch.zeros(16, 8, dtype=torch.bfloat16) for _ in range(2)]
    y = [torch.zeros(16, dtype=torch.bfloat16) for _ in range(2)]
    with pytest.raises(ValueError, match="cuda:0"):
        c.linear_allreduce(w, x, y)


def test_pointer_table_refuses_host_tensors():
    import torch

    from latency_self_synchronizing_b200 import api

    with pytest.raises(TypeError, match="CUDA"):
        api.pointer_table([[torch.zeros(8, dtype=torch.bfloat16)]])
