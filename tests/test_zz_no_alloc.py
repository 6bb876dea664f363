"""The allocation-free all-reduce entry point (sfc_allreduce_noalloc).

It serves callers that cannot call cudaMalloc when they need the collective:
code inside a custom allocator or an out-of-memory handler, a serving process
that reserved all device memory up front, a host library that may not own
allocations. Its scratch is a static device array shared by every call.

This file is collected last, so that a failure here comes after every other
test has run. Its tests call the entry point through the C ABI and check:
two calls in a row (the second must not be disturbed by what the first left
in the shared array) bit-exact to the oracle's closed form and to the
regular entry point; free device memory unchanged across warm calls; the
same in a fresh process whose first call is the documented set-up call; a
wait that runs out is reported by sfc_noalloc_status, not lost.
"""
import ctypes as C
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

from latency_self_synchronizing_b200 import _lib, api
from latency_self_synchronizing_b200.inputs import make_inputs
from oracle import reference

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bits(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def _stream():
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _status(lib):
    info = C.c_uint32(0)
    rc = lib.sfc_noalloc_status(_stream(), C.byref(info))
    return api.Status(rc), int(info.value)


@pytest.mark.parametrize("n,count", [(2, 8), (4, 1000), (8, 4096), (3, 4093), (5, 1)])
def test_noalloc_matches_oracle_and_regular_entry_twice(n, count):
    lib = _lib.load()
    assert lib.sfc_allreduce_noalloc(None, None, 0, 0, None) == 0  # set-up call
    comm = api.Communicator(n, 2 * count, protocols=["ll"])
    try:
        for call in range(2):
            x = make_inputs(seed=500 + 10 * n + call, k_ops=1, nranks=n, count=count)[0]
            ins = [torch.from_numpy(x[r].view(np.int16)).cuda().view(torch.bfloat16) for r in range(n)]
            ref = [torch.empty(count, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
            got = [torch.full((count,), 7.0, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
            comm.allreduce(ins, ref, protocol="ll")
            pin = (C.c_void_p * n)(*[t.data_ptr() for t in ins])
            pout = (C.c_void_p * n)(*[t.data_ptr() for t in got])
            rc = lib.sfc_allreduce_noalloc(pin, pout, n, count, _stream())
            assert rc == 0, api.status_string(rc)
            assert _status(lib)[0] == api.Status.OK
            assert comm.status()[0] == api.Status.OK
            want = reference.allreduce(x)
            for r in range(n):
                np.testing.assert_array_equal(_bits(got[r]), want, err_msg=f"call {call} rank {r} vs oracle")
                np.testing.assert_array_equal(_bits(got[r]), _bits(ref[r]), err_msg=f"call {call} rank {r}")
    finally:
        comm.close()


def test_noalloc_leaves_free_device_memory_unchanged():
    lib = _lib.load()
    n, count = 8, 4096
    assert lib.sfc_allreduce_noalloc(None, None, 0, 0, None) == 0
    x = make_inputs(seed=77, k_ops=1, nranks=n, count=count)[0]
    ins = [torch.from_numpy(x[r].view(np.int16)).cuda().view(torch.bfloat16) for r in range(n)]
    outs = [torch.empty(count, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    pin = (C.c_void_p * n)(*[t.data_ptr() for t in ins])
    pout = (C.c_void_p * n)(*[t.data_ptr() for t in outs])
    assert lib.sfc_allreduce_noalloc(pin, pout, n, count, _stream()) == 0  # warm
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert lib.sfc_allreduce_noalloc(pin, pout, n, count, _stream()) == 0
    assert _status(lib)[0] == api.Status.OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    want = reference.allreduce(x)
    for r in range(n):
        np.testing.assert_array_equal(_bits(outs[r]), want)


def _child(body, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    env["PYTHONPATH"] = ROOT + os.pathsep + env.get("PYTHONPATH", "")
    r = subprocess.run([sys.executable, "-c", textwrap.dedent(body)], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    return r


_CHILD_COMMON = """
    import ctypes as C
    import numpy as np
    import torch
    from latency_self_synchronizing_b200 import _lib, api
    from latency_self_synchronizing_b200.inputs import make_inputs
    from oracle import reference
    torch.cuda.set_device(0)
    lib = _lib.load()
    def stream():
        return C.c_void_p(torch.cuda.current_stream().cuda_stream)
    def status():
        info = C.c_uint32(0)
        return int(lib.sfc_noalloc_status(stream(), C.byref(info))), int(info.value)
    n, count = 4, 3000
    x = make_inputs(seed=31, k_ops=1, nranks=n, count=count)[0]
    ins = [torch.from_numpy(x[r].view(np.int16)).cuda().view(torch.bfloat16) for r in range(n)]
    outs = [torch.zeros(count, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    pin = (C.c_void_p * n)(*[t.data_ptr() for t in ins])
    pout = (C.c_void_p * n)(*[t.data_ptr() for t in outs])
    torch.cuda.synchronize()
"""


def test_noalloc_first_call_in_a_fresh_process():
    r = _child(_CHILD_COMMON + """
    assert lib.sfc_allreduce_noalloc(None, None, 0, 0, None) == 0   # the documented set-up call
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for call in range(2):
        assert lib.sfc_allreduce_noalloc(pin, pout, n, count, stream()) == 0
        assert status() == (0, 0)
        want = reference.allreduce(x)
        for t in outs:
            assert np.array_equal(t.cpu().view(torch.int16).numpy().view(np.uint16), want)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0, "device memory allocated after set-up"
    print("CHILD_OK")
    """)
    assert r.returncode == 0 and "CHILD_OK" in r.stdout, r.stdout + r.stderr


def test_noalloc_reports_a_wait_that_ran_out():
    # rank 1 pushes nothing (a host-side fault: the rank never arrives); its
    # peers' waits give up after 2 ms, which must reach sfc_noalloc_status
    r = _child(_CHILD_COMMON + """
    assert lib.sfc_allreduce_noalloc(pin, pout, n, count, stream()) == 0
    st, info = status()
    assert st == int(api.Status.TIMEOUT), (st, hex(info))
    assert (info >> 8) & 0xff != 1 and (info & 0xff) == 1, hex(info)   # a peer gave up waiting for rank 1
    assert status() == (0, 0)                # reading cleared it
    # while recorded, later calls exit at once and leave their outputs alone
    assert lib.sfc_allreduce_noalloc(pin, pout, n, count, stream()) == 0
    marker = [torch.full((count,), 3.0, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
    pm = (C.c_void_p * n)(*[t.data_ptr() for t in marker])
    assert lib.sfc_allreduce_noalloc(pin, pm, n, count, stream()) == 0
    torch.cuda.synchronize()
    assert all(bool((t == 3.0).all()) for t in marker)
    assert status()[0] == int(api.Status.TIMEOUT)
    print("CHILD_OK")
    """, env_extra={"SFC_NOALLOC_SILENT_RANK": "1", "SFC_TIMEOUT_MS": "2"})
    assert r.returncode == 0 and "CHILD_OK" in r.stdout, r.stdout + r.stderr


def test_noalloc_rejects_oversize():
    lib = _lib.load()
    n, count = 2, 4097
    bufs = [torch.empty(count, dtype=torch.bfloat16, device="cuda") for _ in range(2 * n)]
    pin = (C.c_void_p * n)(*[t.data_ptr() for t in bufs[:n]])
    pout = (C.c_void_p * n)(*[t.data_ptr() for t in bufs[n:]])
    rc = lib.sfc_allreduce_noalloc(pin, pout, n, count, _stream())
    assert rc == int(api.Status.INVALID)
