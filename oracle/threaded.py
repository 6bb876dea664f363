"""Python side of the concurrent CPU model in ``threaded.c``.

TEST INFRASTRUCTURE ONLY: ``tests/`` and the CPU-baseline leg of ``bench.py``
use it; nothing on the product path does. The C file is compiled here with the
system C compiler (plain C11 + POSIX threads) into ``oracle/_build/`` on first
use, or by ``build()``.

Where the Python simulator replays chosen schedules of a model memory, this
runs the same protocols on real threads over real atomics (one thread per
rank), so the interleavings are whatever the CPU produces: a second,
independent check that the epoch-parity reuse and the sentinel reset need no
bottom barrier ("Why Microseconds Matter in AI Infrastructure", section
"Latency can matter more than bandwidth"; "flash-comm: Self-Synchronizing
Collective Communication for LLM Decoding", abstract), and a CPU baseline
that moves data between cores the way the GPU moves it between SMs.
"""

import ctypes as C
import os
import subprocess
import tempfile

import numpy as np

__all__ = ["PROTOCOLS", "ALLGATHER_PROTOCOLS", "ARGTYPES", "build", "chain", "ThreadedError"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "threaded.c")
_OUT = os.path.join(_HERE, "_build", "libsfo_threaded.so")

PROTOCOLS = {"ll": 1, "ll128": 2, "sentinel": 3, "barrier_oneshot": 4, "barrier_twoshot": 5,
             "barrier_oneshot_db": 6, "ll_twoshot": 7, "sentinel_twoshot": 8}
ALLGATHER_PROTOCOLS = ("ll", "ll128", "sentinel")
ARGTYPES = [C.c_int, C.c_int, C.c_int, C.c_size_t, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int,
            C.c_double, C.c_int, C.POINTER(C.c_double)]
_OPS = {"allreduce": 0, "allgather": 1}
_ERRORS = {1: "invalid arguments", 2: "a wait ran out", 3: "slots not left as the protocol requires",
           4: "out of memory", 5: "thread creation failed"}

_lib = None


class ThreadedError(RuntimeError):
    def __init__(self, code):
        super().__init__(f"threaded model: {_ERRORS.get(code, code)}")
        self.code = code


def build(force=False):
    """Compile threaded.c into oracle/_build/libsfo_threaded.so (if stale)."""
    if not force and os.path.exists(_OUT) and os.path.getmtime(_OUT) >= os.path.getmtime(_SRC):
        return _OUT
    os.makedirs(os.path.dirname(_OUT), exist_ok=True)
    fd, tmp = tempfile.mkstemp(suffix=".so", dir=os.path.dirname(_OUT))
    os.close(fd)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-pthread", "-ffp-contract=off", "-fno-fast-math",
                           "-Wall", "-Werror", "-fPIC", "-shared", "-o", tmp, _SRC])
    os.replace(tmp, _OUT)
    return _OUT


def _load():
    global _lib
    if _lib is None:
        lib = C.CDLL(build())
        lib.sfo_threaded_chain.restype = C.c_int
        lib.sfo_threaded_chain.argtypes = ARGTYPES
        _lib = lib
    return _lib


def chain(protocol, x, op="allreduce", skew_ns=None, skew_after=False, timeout_s=10.0):
    """Run len(x) chained operations (epochs 1..k) on x.shape[1] threads.

    x: uint16 bf16 bits [k, N, count]. skew_ns: optional uint32 [k, N], a
    delay of each rank in each operation: before it starts the operation, or
    with ``skew_after`` between its pushes (or its top barrier) and its
    first read, a late reader. Returns (out, seconds): out is
    [k, N, count] (all-reduce) or [k, N, N * count] (all-gather); seconds is
    the wall time of the whole chain."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    k, n, count = x.shape
    width = count if op == "allreduce" else n * count
    out = np.zeros((k, n, width), dtype=np.uint16)
    skew = None
    if skew_ns is not None:
        skew = np.ascontiguousarray(skew_ns, dtype=np.uint32)
        assert skew.shape == (k, n)
    secs = C.c_double(0.0)
    yield_polls = int(n > (os.cpu_count() or 1))
    rc = _load().sfo_threaded_chain(PROTOCOLS[protocol], _OPS[op], n, count, k, x.ctypes.data,
                                    out.ctypes.data, None if skew is None else skew.ctypes.data,
                                    int(bool(skew_after)), float(timeout_s), yield_polls, C.byref(secs))
    if rc != 0:
        raise ThreadedError(rc)
    return out, secs.value
