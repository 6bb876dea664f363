"""The allocation-free all-reduce entry point against the regular one.

sfc_allreduce_noalloc serves callers that cannot call cudaMalloc when they
need the collective (inside an allocator or out-of-memory path, or after
reserving all device memory up front); its scratch is a static device array.
This file is collected last so that a failure here comes after every other
test has run. Both entry points are called through the C ABI on the same
inputs, twice in a row (the second call must not be disturbed by what the
first left in the shared array), and must agree bit for bit, as every parity
test in this suite requires.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from latency_self_synchronizing_b200 import _lib, api
from latency_self_synchronizing_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("n,count", [(2, 8), (4, 1000), (8, 4096), (3, 4093)])
def test_noalloc_matches_regular_entry_point_twice(n, count):
    lib = _lib.load()
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
            stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
            rc = lib.sfc_allreduce_noalloc(pin, pout, n, count, stream)
            assert rc == 0, api.status_string(rc)
            torch.cuda.synchronize()
            assert comm.status()[0] == api.Status.OK
            for r in range(n):
                np.testing.assert_array_equal(_bits(got[r]), _bits(ref[r]), err_msg=f"call {call} rank {r}")
    finally:
        comm.close()


def test_noalloc_rejects_oversize():
    lib = _lib.load()
    n, count = 2, 4097
    bufs = [torch.empty(count, dtype=torch.bfloat16, device="cuda") for _ in range(2 * n)]
    pin = (C.c_void_p * n)(*[t.data_ptr() for t in bufs[:n]])
    pout = (C.c_void_p * n)(*[t.data_ptr() for t in bufs[n:]])
    rc = lib.sfc_allreduce_noalloc(pin, pout, n, count, C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == int(api.Status.INVALID)
