"""The concurrent CPU model (oracle/threaded.c): real threads, real atomics.

Its outputs are pinned to the closed forms (rank-order fp32 sum rounded once
to bf16; concatenation for the all-gather), under the interleavings the CPU
produces and under seeded delays, over chains long enough that every slot
parity is reused many times. Planted mistakes, made in a copy of the C source
compiled on the CPU, show that the checks notice a dropped sentinel reset, a
reduction in the wrong order, a single receive buffer in the oneshot, a
missing bottom barrier and a single input buffer in SiFAR's oneshot; two
further variants confirm readings of the pages: the barrier twoshot stays
correct without its bottom barrier, and the self-synchronizing twoshot with
a single buffer per phase.
"""
import os
import subprocess

import ctypes as C
import numpy as np
import pytest

from latency_self_synchronizing_b200.inputs import make_inputs
from oracle import reference, threaded

PROTOS = list(threaded.PROTOCOLS)


def _check_allreduce(out, x):
    k, n, _ = x.shape
    for kk in range(k):
        want = reference.allreduce(x[kk])
        for r in range(n):
            np.testing.assert_array_equal(out[kk, r], want, err_msg=f"op {kk} rank {r}")


@pytest.mark.parametrize("proto", PROTOS)
@pytest.mark.parametrize("n,count", [(2, 1), (3, 59), (4, 61), (5, 1001), (8, 120), (8, 257)])
def test_allreduce_matches_closed_form(proto, n, count):
    # counts: one element (empty twoshot shards), LL's odd tail, LL128's
    # partial and exact lines, shards that are not whole vectors
    x = make_inputs(seed=100 + n, k_ops=12, nranks=n, count=count)
    out, secs = threaded.chain(proto, x)
    assert secs > 0
    _check_allreduce(out, x)


@pytest.mark.parametrize("proto", threaded.ALLGATHER_PROTOCOLS)
@pytest.mark.parametrize("n", [2, 4, 8])
def test_allgather_matches_concatenation(proto, n):
    x = make_inputs(seed=200 + n, k_ops=8, nranks=n, count=77, dist="uniform", params=(-4.0, 4.0))
    out, _ = threaded.chain(proto, x, op="allgather")
    for k in range(8):
        want = reference.allgather(x[k])
        for r in range(n):
            np.testing.assert_array_equal(out[k, r], want)


@pytest.mark.parametrize("proto", PROTOS)
@pytest.mark.parametrize("after", [False, True])
def test_delays_change_nothing(proto, after):
    """Per-(operation, rank) delays ~ Exp(mean 20 us), before the operation
    or between a rank's pushes / top barrier and its reads: ranks run up to
    an epoch ahead, so slots of one parity are rewritten while the other is
    still being read; the bits stay the closed form's."""
    n, k, count = 4, 40, 300
    x = make_inputs(seed=300, k_ops=k, nranks=n, count=count)
    for s in range(3):
        skew = np.random.Generator(np.random.PCG64(s)).exponential(20e3, size=(k, n)).astype(np.uint32)
        out, _ = threaded.chain(proto, x, skew_ns=skew, skew_after=after)
        _check_allreduce(out, x)


def test_rejects_bad_arguments():
    x = make_inputs(seed=1, k_ops=1, nranks=2, count=8)
    for proto in ("barrier_oneshot", "barrier_twoshot", "ll_twoshot"):
        with pytest.raises(threaded.ThreadedError) as ei:
            threaded.chain(proto, x, op="allgather")
        assert ei.value.code == 1
    with pytest.raises(threaded.ThreadedError):
        threaded.chain("ll", x[:, :1])


# ---------------------------------------------------------------- variants

_SRC = os.path.join(os.path.dirname(threaded.__file__), "threaded.c")


def _variant(tmp_path, old, new, times=1):
    src = open(_SRC).read()
    assert src.count(old) == times, (old, src.count(old))
    path = tmp_path / "variant.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "variant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-pthread", "-ffp-contract=off", "-fPIC", "-shared",
                           "-o", str(so), str(path)])
    lib = C.CDLL(str(so))
    lib.sfo_threaded_chain.restype = C.c_int
    lib.sfo_threaded_chain.argtypes = threaded.ARGTYPES
    return lib


def _run(lib, proto, x, skew=None, after=0, timeout_s=2.0):
    k, n, count = x.shape
    out = np.zeros_like(x)
    secs = C.c_double()
    sk = None if skew is None else np.ascontiguousarray(skew, dtype=np.uint32)
    rc = lib.sfo_threaded_chain(threaded.PROTOCOLS[proto], 0, n, count, k, x.ctypes.data, out.ctypes.data,
                                None if sk is None else sk.ctypes.data, after, timeout_s, 0, C.byref(secs))
    return rc, out


def _matches(out, x):
    return all(np.array_equal(out[k, r], reference.allreduce(x[k]))
               for k in range(x.shape[0]) for r in range(x.shape[1]))


def _late_last_rank(k, n, ns=2_000_000):
    """The last rank reads 2 ms late in every operation; the others at once."""
    skew = np.zeros((k, n), dtype=np.uint32)
    skew[:, n - 1] = ns
    return skew


def test_planted_missing_sentinel_reset_is_caught(tmp_path):
    lib = _variant(tmp_path, "atomic_store_explicit(&z->e[base + j], (uint16_t)SENTINEL_BITS, "
                             "memory_order_relaxed);", "")
    x = make_inputs(seed=400, k_ops=6, nranks=3, count=64)
    rc, out = _run(lib, "sentinel", x)
    # without the reset epoch 3 takes epoch 1's values from the slot: wrong
    # sums, and the slots are not back at the pre-fill after the chain
    assert rc != 0 or not _matches(out, x)


def test_planted_reversed_reduction_order_is_caught(tmp_path):
    lib = _variant(tmp_path,
                   "float acc = widen(src[0][i]);\n  for (int q = 1; q < n; ++q) acc = acc + widen(src[q][i]);",
                   "float acc = widen(src[n - 1][i]);\n  for (int q = n - 2; q >= 0; --q) acc = acc + widen(src[q][i]);")
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


@pytest.mark.parametrize("proto", ["ll", "sentinel"])
def test_planted_single_receive_buffer_is_caught(tmp_path, proto):
    """One slot per source instead of one per epoch parity: the peers finish
    epoch e and push e+1 into the late reader's slot before it read e."""
    lib = _variant(tmp_path, "slot_base(z, recv, (int)(epoch & 1u), src)", "slot_base(z, recv, 0, src)", times=2)
    x = make_inputs(seed=402, k_ops=4, nranks=3, count=256)
    rc, out = _run(lib, proto, x, _late_last_rank(4, 3), after=1, timeout_s=0.5)
    assert rc != 0 or not _matches(out, x)


def test_planted_missing_bottom_barrier_is_caught(tmp_path):
    """The pull oneshot without its bottom barrier: a rank that finished
    operation k writes its next input over the buffer the late reader is
    about to read (the write-after-write hazard SiFAR names)."""
    lib = _variant(tmp_path, "return dual ? 0 : barrier(s, 2, r, epoch);", "return 0;")
    x = make_inputs(seed=403, k_ops=4, nranks=3, count=256)
    rc, out = _run(lib, "barrier_oneshot", x, _late_last_rank(4, 3), after=1)
    assert rc == 0
    assert not _matches(out, x)


def test_planted_single_input_buffer_in_dual_buffered_oneshot_is_caught(tmp_path):
    lib = _variant(tmp_path, "const int buf = dual ? (int)(epoch & 1u) : 0;", "const int buf = 0;")
    x = make_inputs(seed=404, k_ops=4, nranks=3, count=256)
    rc, out = _run(lib, "barrier_oneshot_db", x, _late_last_rank(4, 3), after=1)
    assert rc == 0
    assert not _matches(out, x)
    # the real dual buffering under the same delays
    out, _ = threaded.chain("barrier_oneshot_db", x, skew_ns=_late_last_rank(4, 3), skew_after=True)
    _check_allreduce(out, x)


def test_barrier_twoshot_needs_no_bottom_barrier(tmp_path):
    """Reading of the pages: in the pull twoshot the middle barrier of
    operation k and the top barrier of k+1 already order every reuse of the
    input and result buffers; without the bottom barrier the bits stay
    right under late readers and random delays."""
    lib = _variant(tmp_path, "  return barrier(s, 2, r, epoch);\n}", "  return 0;\n}")
    x = make_inputs(seed=405, k_ops=8, nranks=4, count=300)
    for after in (0, 1):
        rc, out = _run(lib, "barrier_twoshot", x, _late_last_rank(8, 4, 500_000), after=after)
        assert rc == 0 and _matches(out, x)
    for s in range(3):
        skew = np.random.Generator(np.random.PCG64(s)).exponential(20e3, size=(8, 4)).astype(np.uint32)
        rc, out = _run(lib, "barrier_twoshot", x, skew, after=s % 2)
        assert rc == 0 and _matches(out, x)


@pytest.mark.parametrize("proto", ["ll_twoshot", "sentinel_twoshot"])
def test_selfsync_twoshot_survives_a_single_buffer(tmp_path, proto):
    """Reading of the pages: in the self-synchronizing twoshot every slot of
    either phase is rewritten only after a full exchange of the other phase,
    so one buffer per phase already gives the right bits (the LL flags then
    end on the last epoch in one parity only, which the slot check reports)."""
    lib = _variant(tmp_path, "slot_base(z, recv, (int)(epoch & 1u), src)", "slot_base(z, recv, 0, src)", times=2)
    x = make_inputs(seed=406, k_ops=8, nranks=4, count=300)
    for after in (0, 1):
        rc, out = _run(lib, proto, x, _late_last_rank(8, 4, 500_000), after=after)
        assert rc in (0, 3) and _matches(out, x)


def _golden_cases():
    path = os.path.join(os.path.dirname(__file__), "golden", "rank_order_sum.txt")
    for line in open(path):
        line = line.split("#")[0].strip()
        if line:
            left, right = line.split("->")
            parts = left.split()
            n = int(parts[1])
            yield parts[0], [int(h, 16) for h in parts[2:2 + n]], int(right.split("|")[0], 16)


@pytest.mark.parametrize("proto", PROTOS)
def test_hand_derived_order_sensitive_cases(proto):
    """The hand-derived cases whose answer depends on the rank order give
    the derived bits on real threads too, whatever order the units land."""
    for name, xs, want in _golden_cases():
        n, count = len(xs), 97
        x = np.empty((6, n, count), dtype=np.uint16)
        x[:] = np.array(xs, dtype=np.uint16)[None, :, None]
        out, _ = threaded.chain(proto, x)
        assert np.all(out == want), (name, proto)
