"""GPU error paths: host-side rejections and bounded device waits.

Failures are made on the host (a rank told to stay silent, a wrong epoch, a
bad argument); the device waits run out after a short limit and report a
status the host reads, and the context stays usable after sfc_reset. No test
here faults, traps or hangs the GPU.
"""
import numpy as np
import pytest
import torch

from latency_self_synchronizing_b200 import api
from latency_self_synchronizing_b200.inputs import make_inputs
from oracle import reference

from _gpu_helpers import Operands, run_chain

pytestmark = pytest.mark.gpu


def _ops(x):
    return Operands(*x.shape, fill=x), Operands(*x.shape)


def test_wrong_epoch_rejected_on_host():
    comm = api.Communicator(2, 4096)
    try:
        x = make_inputs(seed=1, k_ops=1, nranks=2, count=64)
        ins, outs = _ops(x)
        with pytest.raises(api.SfcError) as ei:
            comm.allreduce(ins.tensors(0), outs.tensors(0), protocol="ll", epoch=5)
        assert ei.value.status == api.Status.EPOCH
        assert comm.launch_count == 0
    finally:
        comm.close()


def test_bad_arguments_rejected():
    comm = api.Communicator(2, 4096)
    try:
        x = make_inputs(seed=2, k_ops=1, nranks=2, count=64)
        ins, outs = _ops(x)
        with pytest.raises(api.SfcError) as ei:  # twoshot is not an all-gather
            comm.allgather(ins.tensors(0), [torch.empty(128, dtype=torch.bfloat16, device="cuda")] * 2,
                           protocol="twoshot")
        assert ei.value.status == api.Status.UNSUPPORTED
        big = Operands(1, 2, 4096)
        with pytest.raises(api.SfcError) as ei:  # larger than max_bytes_per_rank
            comm.allreduce(big.tensors(0), big.tensors(0), protocol="ll")
        assert ei.value.status == api.Status.INVALID
        with pytest.raises(api.SfcError) as ei:  # in-place (aliasing)
            comm.allreduce(ins.tensors(0), ins.tensors(0), protocol="ll")
        assert ei.value.status == api.Status.INVALID
        assert comm.launch_count == 0
    finally:
        comm.close()


@pytest.mark.parametrize("proto", ["ll", "ll128", "sentinel", "barrier_oneshot", "barrier_twoshot",
                                   "barrier_oneshot_db", "ll_twoshot", "sentinel_twoshot", "ll128_fast"])
def test_silent_rank_times_out_and_recovers(proto):
    comm = api.Communicator(4, 1 << 14, timeout_us=2000)
    try:
        x = make_inputs(seed=3, k_ops=3, nranks=4, count=4096)
        ins, outs = _ops(x)
        comm.set_silent_rank(2)
        comm.allreduce_chain(ins.table, outs.table, 4096, 3, protocol=proto)
        st, info = comm.status()
        assert st == api.Status.TIMEOUT
        # a poisoned context refuses new work until reset
        with pytest.raises(api.SfcError) as ei:
            comm.allreduce_chain(ins.table, outs.table, 4096, 3, protocol=proto)
        assert ei.value.status == api.Status.ABORTED
        comm.set_silent_rank(-1)
        comm.reset()
        assert comm.next_epoch == 1
        out = run_chain(comm, proto, x)
        for k in range(3):
            for r in range(4):
                np.testing.assert_array_equal(out[k, r], reference.allreduce(x[k]))
    finally:
        comm.close()


def test_sentinel_in_input_detected_with_debug_checks():
    comm = api.Communicator(2, 4096, debug_checks=True, timeout_us=5000)
    try:
        x = make_inputs(seed=4, k_ops=1, nranks=2, count=64)
        x[0, 1, 10] = 0xFFFF
        ins, outs = _ops(x)
        comm.allreduce_chain(ins.table, outs.table, 64, 1, protocol="sentinel")
        st, _ = comm.status()
        assert st == api.Status.SENTINEL_IN_INPUT
        comm.reset()
    finally:
        comm.close()


def test_zero_count_is_a_noop():
    comm = api.Communicator(2, 4096)
    try:
        e = comm.next_epoch
        empty = [torch.empty(0, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
        comm.allreduce(empty, [torch.empty(0, dtype=torch.bfloat16, device="cuda") for _ in range(2)],
                       protocol="ll")
        assert comm.next_epoch == e and comm.launch_count == 0
    finally:
        comm.close()
