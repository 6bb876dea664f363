"""The host-buffer entry point (sfc_allreduce_chain_host) against the oracle.

The chain is split into up to 8 launches whose host<->device copies overlap
their neighbours on two copy streams; these tests cover every segment count,
a ragged size, two calls queued back to back without a synchronisation in
between (the second must not overwrite staging the first still uses),
staging growth, pageable host memory, and the per-operation completion
stamps across segment boundaries.
"""
import numpy as np
import pytest
import torch

from latency_self_synchronizing_b200 import api
from latency_self_synchronizing_b200.inputs import make_inputs
from oracle import reference

pytestmark = pytest.mark.gpu


def _host(bits, pinned=True):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.pin_memory() if pinned else t.clone()


def _want(x):
    return np.stack([reference.allreduce(x[k]) for k in range(x.shape[0])])


def _check(out, x):
    got = out.view(torch.int16).numpy().view(np.uint16)
    want = _want(x)
    for r in range(x.shape[1]):
        np.testing.assert_array_equal(got[:, r, :], want, err_msg=f"rank {r}")


@pytest.mark.parametrize("proto", ["sentinel", "ll", "barrier_oneshot_db"])
@pytest.mark.parametrize("k_ops", [1, 15, 16, 40, 129, 160])
def test_host_chain_matches_oracle(proto, k_ops):
    n, count = 4, 1000
    comm = api.Communicator(n, 2 * count)
    try:
        x = make_inputs(seed=k_ops, k_ops=k_ops, nranks=n, count=count, dist="normal", params=(1.0,))
        hin, hout = _host(x), torch.empty(k_ops, n, count, dtype=torch.bfloat16).pin_memory()
        tim = torch.zeros(k_ops + 1, dtype=torch.int64, device="cuda")
        comm.allreduce_chain_host(hin, hout, protocol=proto, timings=tim)
        torch.cuda.synchronize()
        st, info = comm.status()
        assert st == api.Status.OK, (st, hex(info))
        _check(hout, x)
        assert comm.next_epoch == 1 + k_ops
        t = tim.cpu().numpy().astype(np.uint64)
        assert np.all(t[1:] >= t[0]) and np.all(np.diff(t[1:].astype(np.int64)) >= 0)
    finally:
        comm.close()


def test_back_to_back_calls_growth_and_pageable():
    n = 8
    comm = api.Communicator(n, 1 << 15)
    try:
        xa = make_inputs(seed=1, k_ops=64, nranks=n, count=4099)
        xb = make_inputs(seed=2, k_ops=48, nranks=n, count=4099)
        ha, hb = _host(xa), _host(xb)
        oa = torch.empty(64, n, 4099, dtype=torch.bfloat16).pin_memory()
        ob = torch.empty(48, n, 4099, dtype=torch.bfloat16).pin_memory()
        comm.allreduce_chain_host(ha, oa, protocol="ll")
        comm.allreduce_chain_host(hb, ob, protocol="sentinel")  # queued behind the first, no sync
        torch.cuda.synchronize()
        assert comm.status()[0] == api.Status.OK
        _check(oa, xa)
        _check(ob, xb)
        # larger than any staging so far: staging grows; pageable host memory
        xc = make_inputs(seed=3, k_ops=100, nranks=n, count=16384)
        hc = _host(xc, pinned=False)
        oc = torch.empty(100, n, 16384, dtype=torch.bfloat16)
        comm.allreduce_chain_host(hc, oc, protocol="auto")
        torch.cuda.synchronize()
        assert comm.status()[0] == api.Status.OK
        _check(oc, xc)
        assert comm.next_epoch == 1 + 64 + 48 + 100
    finally:
        comm.close()
