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


def test_epoch_zero_means_next():
    """0 is never an epoch; every entry point reads it as the next one."""
    import ctypes as C
    comm = api.Communicator(2, 4096)
    try:
        x = make_inputs(seed=5, k_ops=3, nranks=2, count=64)
        ins, outs = _ops(x)
        lib = comm._lib
        for k in range(3):
            pi = (C.c_void_p * 2)(*[t.data_ptr() for t in ins.tensors(k)])
            po = (C.c_void_p * 2)(*[t.data_ptr() for t in outs.tensors(k)])
            assert lib.sfc_allreduce(comm._ctx, pi, po, 64, 0, int(api.Protocol.LL), 0, None) == 0
            assert comm.next_epoch == 2 + k
        torch.cuda.synchronize()
        assert comm.status()[0] == api.Status.OK
        for k in range(3):
            np.testing.assert_array_equal(outs.bits()[k, 0], reference.allreduce(x[k]))
        with pytest.raises(api.SfcError) as ei:  # an explicit stale epoch is still refused
            comm.allreduce(ins.tensors(0), outs.tensors(0), protocol="ll", epoch=1)
        assert ei.value.status == api.Status.EPOCH
    finally:
        comm.close()


def test_env_overrides(monkeypatch):
    """SFC_PROTOCOL forces what AUTO resolves to; SFC_TIMEOUT_MS bounds the
    device waits (a silent rank times out within it)."""
    import time
    monkeypatch.setenv("SFC_PROTOCOL", "barrier_oneshot_db")
    monkeypatch.setenv("SFC_TIMEOUT_MS", "3")
    comm = api.Communicator(4, 1 << 14)
    try:
        assert comm.select_protocol("allreduce", 2048) == api.Protocol.BARRIER_ONESHOT_DB
        assert comm.select_protocol("allgather", 2048) == api.Protocol.BARRIER_ONESHOT_DB
        x = make_inputs(seed=6, k_ops=2, nranks=4, count=1024)
        ins, outs = _ops(x)
        comm.allreduce_chain(ins.table, outs.table, 1024, 2, protocol="auto")
        torch.cuda.synchronize()
        assert comm.status()[0] == api.Status.OK
        for k in range(2):
            np.testing.assert_array_equal(outs.bits()[k, 1], reference.allreduce(x[k]))
        comm.set_silent_rank(1)
        t0 = time.perf_counter()
        comm.allreduce_chain(ins.table, outs.table, 1024, 2, protocol="ll")
        torch.cuda.synchronize()
        assert time.perf_counter() - t0 < 1.0
        assert comm.status()[0] == api.Status.TIMEOUT
        comm.set_silent_rank(-1)
        comm.reset()
    finally:
        comm.close()
    monkeypatch.setenv("SFC_PROTOCOL", "ll_twoshot")  # all-reduce only: all-gather keeps the selector
    monkeypatch.setenv("SFC_TIMEOUT_MS", "not a number")
    comm = api.Communicator(4, 1 << 14)
    try:
        assert comm.select_protocol("allreduce", 2048) == api.Protocol.LL_TWOSHOT
        assert comm.select_protocol("allgather", 2048) != api.Protocol.LL_TWOSHOT
    finally:
        comm.close()


def test_spent_epoch_sequence_is_refused_until_reset():
    """After epoch 2^32 - 1 the host sequence is spent: a wrap to 0 would
    validate against zero-filled LL flags, so every call is refused with
    SFC_ERR_EPOCH (nothing launched) until sfc_reset."""
    comm = api.Communicator(2, 4096)
    try:
        x = make_inputs(seed=9, k_ops=2, nranks=2, count=64)
        ins, outs = _ops(x)
        assert comm.reserve_epochs(0xFFFFFFFE) == 1  # epochs 1 .. 2^32 - 2, never launched
        assert comm.next_epoch == 0xFFFFFFFF
        comm.allreduce(ins.tensors(0), outs.tensors(0), protocol="ll")  # the last epoch
        torch.cuda.synchronize()
        assert comm.status()[0] == api.Status.OK
        np.testing.assert_array_equal(outs.bits()[0, 0], reference.allreduce(x[0]))
        assert comm.next_epoch == 0
        launches = comm.launch_count
        for proto in ("ll", "sentinel", "barrier_oneshot"):
            with pytest.raises(api.SfcError) as ei:
                comm.allreduce(ins.tensors(1), outs.tensors(1), protocol=proto)
            assert ei.value.status == api.Status.EPOCH
        with pytest.raises(api.SfcError) as ei:
            comm.reserve_epochs(1)
        assert ei.value.status == api.Status.EPOCH
        assert comm.launch_count == launches
        comm.reset()
        assert comm.next_epoch == 1
        comm.allreduce(ins.tensors(1), outs.tensors(1), protocol="ll")
        torch.cuda.synchronize()
        assert comm.status()[0] == api.Status.OK
        np.testing.assert_array_equal(outs.bits()[1, 1], reference.allreduce(x[1]))
    finally:
        comm.close()
