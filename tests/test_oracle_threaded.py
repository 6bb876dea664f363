"""The concurrent CPU model (oracle/threaded.c): real threads, real atomics.

Its outputs are pinned to the closed forms (rank-order fp32 sum rounded once
to bf16; concatenation for the all-gather), under the interleavings the CPU
produces and under seeded start skews, over chains long enough that every
slot parity is reused many times. Two planted mistakes, made in a copy of the
C source compiled on the CPU, show that the checks notice a dropped sentinel
reset and a reduction in the wrong order.
"""
import os
import subprocess

import ctypes as C
import numpy as np
import pytest

from latency_self_synchronizing_b200.inputs import make_inputs
from oracle import reference, threaded

PROTOS = ["ll", "ll128", "sentinel", "barrier_oneshot"]


def _check_allreduce(out, x):
    k, n, _ = x.shape
    for kk in range(k):
        want = reference.allreduce(x[kk])
        for r in range(n):
            np.testing.assert_array_equal(out[kk, r], want, err_msg=f"op {kk} rank {r}")


@pytest.mark.parametrize("proto", PROTOS)
@pytest.mark.parametrize("n,count", [(2, 1), (3, 59), (4, 61), (5, 1001), (8, 120), (8, 257)])
def test_allreduce_matches_closed_form(proto, n, count):
    # counts: one element, LL's odd tail, LL128's partial and exact lines
    x = make_inputs(seed=100 + n, k_ops=12, nranks=n, count=count)
    out, secs = threaded.chain(proto, x)
    assert secs > 0
    _check_allreduce(out, x)


@pytest.mark.parametrize("proto", ["ll", "ll128", "sentinel"])
@pytest.mark.parametrize("n", [2, 4, 8])
def test_allgather_matches_concatenation(proto, n):
    x = make_inputs(seed=200 + n, k_ops=8, nranks=n, count=77, dist="uniform", params=(-4.0, 4.0))
    out, _ = threaded.chain(proto, x, op="allgather")
    for k in range(8):
        want = reference.allgather(x[k])
        for r in range(n):
            np.testing.assert_array_equal(out[k, r], want)


@pytest.mark.parametrize("proto", PROTOS)
def test_skewed_starts_change_nothing(proto):
    """Per-(operation, rank) start delays ~ Exp(mean 20 us): ranks run up to
    an epoch ahead, so slots of one parity are rewritten while the other is
    still being read; the bits stay the closed form's."""
    n, k, count = 4, 40, 300
    x = make_inputs(seed=300, k_ops=k, nranks=n, count=count)
    for s in range(3):
        skew = np.random.Generator(np.random.PCG64(s)).exponential(20e3, size=(k, n)).astype(np.uint32)
        out, _ = threaded.chain(proto, x, skew_ns=skew)
        _check_allreduce(out, x)


def test_rejects_bad_arguments():
    x = make_inputs(seed=1, k_ops=1, nranks=2, count=8)
    with pytest.raises(threaded.ThreadedError) as ei:
        threaded.chain("barrier_oneshot", x, op="allgather")
    assert ei.value.code == 1
    with pytest.raises(threaded.ThreadedError):
        threaded.chain("ll", x[:, :1])


def _mutant(tmp_path, old, new):
    src = open(os.path.join(os.path.dirname(threaded.__file__), "threaded.c")).read()
    assert src.count(old) == 1
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "mutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-pthread", "-ffp-contract=off", "-fPIC", "-shared",
                           "-o", str(so), str(path)])
    lib = C.CDLL(str(so))
    lib.sfo_threaded_chain.restype = C.c_int
    lib.sfo_threaded_chain.argtypes = [C.c_int, C.c_int, C.c_int, C.c_size_t, C.c_int, C.c_void_p, C.c_void_p,
                                       C.c_void_p, C.c_double, C.c_int, C.POINTER(C.c_double)]
    return lib


def _run(lib, proto, x, timeout_s=2.0):
    k, n, count = x.shape
    out = np.zeros_like(x)
    secs = C.c_double()
    rc = lib.sfo_threaded_chain(threaded.PROTOCOLS[proto], 0, n, count, k, x.ctypes.data, out.ctypes.data, None,
                                timeout_s, 0, C.byref(secs))
    return rc, out


def _matches(out, x):
    return all(np.array_equal(out[k, r], reference.allreduce(x[k]))
               for k in range(x.shape[0]) for r in range(x.shape[1]))


def test_planted_missing_sentinel_reset_is_caught(tmp_path):
    lib = _mutant(tmp_path, "atomic_store_explicit(&s->sent[base + j], (uint16_t)SENTINEL_BITS, "
                            "memory_order_relaxed);", "")
    x = make_inputs(seed=400, k_ops=6, nranks=3, count=64)
    rc, out = _run(lib, "sentinel", x)
    # without the reset epoch 3 takes epoch 1's values from the slot: wrong
    # sums, and the slots are not back at the pre-fill after the chain
    assert rc != 0 or not _matches(out, x)


def test_planted_reversed_reduction_order_is_caught(tmp_path):
    lib = _mutant(tmp_path,
                  "float acc = widen(src[0][i]);\n      for (int q = 1; q < n; ++q) acc = acc + widen(src[q][i]);",
                  "float acc = widen(src[n - 1][i]);\n      for (int q = n - 2; q >= 0; --q) acc = acc + widen(src[q][i]);")
    # fp32 sums of a few bf16 values of one scale are exact in any order, so
    # the planted order only shows where a small term is absorbed by a large
    # one: (2^27 - 2^27) + 1 = 1, but (1 - 2^27) + 2^27 = 0 in binary32
    x = make_inputs(seed=401, k_ops=2, nranks=3, count=64)
    x[:, 0, ::2] = 0x4D00  # +2^27
    x[:, 1, ::2] = 0xCD00  # -2^27
    x[:, 2, ::2] = 0x3F80  # 1.0
    rc, out = _run(lib, "ll", x)
    assert rc == 0
    assert not _matches(out, x)
