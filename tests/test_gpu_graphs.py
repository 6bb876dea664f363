"""Device-epoch contexts: calls captured in a CUDA graph and replayed.

With sfc_config.device_epochs the epoch sequence lives on the device, so a
captured launch takes the next epoch each time it is replayed; outputs must
be bit-exact to the oracle on every replay, for LL (whose readiness flag is
the epoch) as well as the sentinel and barrier protocols, single calls and
chains, and eager calls must continue the same sequence.
"""
import numpy as np
import pytest
import torch

from latency_self_synchronizing_b200 import api
from latency_self_synchronizing_b200.inputs import make_inputs
from oracle import reference

from _gpu_helpers import Operands

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _fill(dst, bits):
    dst.copy_(torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16))


@pytest.mark.parametrize("protos", [("sentinel", "ll"), ("ll128_fast", "barrier_oneshot_db")])
def test_single_calls_replayed_from_a_graph(protos):
    n, count, reps = 4, 4099, 12
    comm = api.Communicator(n, 2 * count, device_epochs=True)
    try:
        assert comm.next_epoch == 0
        xs = [torch.empty(count, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
        ys = [torch.empty_like(x) for x in xs]
        zs = [torch.empty_like(x) for x in xs]
        data = make_inputs(seed=42, k_ops=reps + 1, nranks=n, count=count)
        for r in range(n):
            _fill(xs[r], data[0, r])
        comm.allreduce(xs, ys, protocol=protos[0])  # eager, before capture
        torch.cuda.synchronize()
        np.testing.assert_array_equal(_bits(ys[2]), reference.allreduce(data[0]))
        with pytest.raises(api.SfcError) as ei:  # device epochs take no explicit epoch
            comm.allreduce(xs, ys, protocol=protos[0], epoch=2)
        assert ei.value.status == api.Status.EPOCH
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            comm.allreduce(xs, ys, protocol=protos[0])
            comm.allreduce(xs, zs, protocol=protos[1])
        for i in range(1, reps + 1):
            for r in range(n):
                _fill(xs[r], data[i, r])
            g.replay()
            torch.cuda.synchronize()
            want = reference.allreduce(data[i])
            for r in range(n):
                np.testing.assert_array_equal(_bits(ys[r]), want, err_msg=f"replay {i} rank {r}")
                np.testing.assert_array_equal(_bits(zs[r]), want, err_msg=f"replay {i} rank {r}")
        comm.allreduce(xs, ys, protocol=protos[1])  # eager again: continues the sequence
        torch.cuda.synchronize()
        np.testing.assert_array_equal(_bits(ys[0]), reference.allreduce(data[reps]))
        st, info = comm.status()
        assert st == api.Status.OK, (st, hex(info))
        comm.reset()  # the device epoch goes back to 1
        comm.allreduce(xs, ys, protocol="ll")
        torch.cuda.synchronize()
        assert comm.status()[0] == api.Status.OK
        np.testing.assert_array_equal(_bits(ys[1]), reference.allreduce(data[reps]))
    finally:
        comm.close()


def test_chain_replayed_from_a_graph():
    n, count, k, reps = 8, 1000, 6, 5
    comm = api.Communicator(n, 2 * count, device_epochs=True)
    try:
        data = make_inputs(seed=7, k_ops=k * reps, nranks=n, count=count)
        ins = Operands(k, n, count)
        outs = Operands(k, n, count)
        view = ins.buf.view(k, n, ins.stride)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            comm.allreduce_chain(ins.table, outs.table, count, k, protocol="ll")
        for i in range(reps):
            host = np.zeros((k, n, ins.stride), dtype=np.uint16)
            host[:, :, :count] = data[i * k:(i + 1) * k]
            view.copy_(torch.from_numpy(host.view(np.int16)).cuda())
            g.replay()
            torch.cuda.synchronize()
            out = outs.bits()
            for kk in range(k):
                np.testing.assert_array_equal(out[kk, 3], reference.allreduce(data[i * k + kk]))
        assert comm.status()[0] == api.Status.OK
    finally:
        comm.close()
