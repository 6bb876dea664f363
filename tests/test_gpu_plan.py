"""Prepared single collectives (sfc_plan_create / sfc_plan_launch): the same
bits as the closed form on every launch, the epoch sequence shared with the
other calls, operands fixed at creation while their contents change."""
import numpy as np
import pytest
import torch

from latency_self_synchronizing_b200 import api
from latency_self_synchronizing_b200.inputs import make_inputs
from oracle import reference

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _bits(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("proto", ["auto", "ll", "sentinel", "ll128", "barrier_oneshot", "barrier_twoshot",
                                   "barrier_oneshot_db", "ll_twoshot", "sentinel_twoshot"])
@pytest.mark.parametrize("n,count", [(2, 8), (4, 8192), (8, 4099)])
def test_plan_launches_match_the_closed_form(proto, n, count):
    comm = api.Communicator(n, 2 * count)
    try:
        x = make_inputs(seed=40 + n + count % 13, k_ops=4, nranks=n, count=count)
        ins = [_dev(x[0, r]) for r in range(n)]
        outs = [torch.empty(count, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
        plan = comm.plan(ins, outs, protocol=proto)
        for k in range(4):
            for r in range(n):  # new contents in the same buffers
                ins[r].copy_(_dev(x[k, r]))
            e = comm.next_epoch
            plan.launch()
            assert comm.next_epoch == e + 1
            if k == 1:  # a regular call in between continues the same sequence
                other = [torch.empty_like(t) for t in outs]
                comm.allreduce(ins, other, protocol=proto)
            torch.cuda.synchronize()
            assert comm.status()[0] == api.Status.OK
            want = reference.allreduce(x[k])
            for r in range(n):
                np.testing.assert_array_equal(_bits(outs[r]), want, err_msg=f"launch {k} rank {r}")
    finally:
        comm.close()


def test_plan_allgather_and_argument_checks():
    n, count = 4, 1000
    comm = api.Communicator(n, 2 * count)
    try:
        x = make_inputs(seed=3, k_ops=1, nranks=n, count=count)[0]
        ins = [_dev(x[r]) for r in range(n)]
        outs = [torch.empty(n * count, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
        plan = comm.plan(ins, outs, op="allgather", protocol="ll")
        plan.launch()
        plan.launch()
        torch.cuda.synchronize()
        assert comm.status()[0] == api.Status.OK
        for r in range(n):
            np.testing.assert_array_equal(_bits(outs[r]), reference.allgather(x))
        ar_outs = [torch.empty(count, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
        with pytest.raises(api.SfcError) as ei:  # an output that overlaps an input
            comm.plan(ins, [ins[0]] + ar_outs[1:], op="allreduce", protocol="ll")
        assert ei.value.status == api.Status.INVALID
        with pytest.raises(api.SfcError) as ei:  # allgather has no twoshot
            comm.plan(ins, outs, op="allgather", protocol="barrier_twoshot")
        assert ei.value.status == api.Status.UNSUPPORTED
    finally:
        comm.close()


def test_repeated_single_calls_on_the_same_tensors():
    """The binding skips its metadata checks when a call repeats the last
    call's tensor objects at the same addresses and sizes; any change makes
    it check again."""
    n, count = 4, 2048
    comm = api.Communicator(n, 2 * 4 * count)
    try:
        x = make_inputs(seed=77, k_ops=2, nranks=n, count=count)
        ins = [_dev(x[0, r]) for r in range(n)]
        outs = [torch.empty(count, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
        for k in range(2):
            for r in range(n):
                ins[r].copy_(_dev(x[k, r]))
            comm.allreduce(ins, outs, protocol="ll")  # the second call takes the short path
            torch.cuda.synchronize()
            for r in range(n):
                np.testing.assert_array_equal(_bits(outs[r]), reference.allreduce(x[k]))
        with pytest.raises(TypeError, match="CUDA"):  # another object: checked again
            comm.allreduce(ins, outs[:-1] + [torch.empty(count, dtype=torch.bfloat16)], protocol="ll")
        comm.allreduce(ins, outs, protocol="ll")
        outs[0].resize_(count // 2)  # same object, new size: checked again
        with pytest.raises(ValueError):
            comm.allreduce(ins, outs, protocol="ll")
        ins[1].resize_(count // 2)
        with pytest.raises(ValueError):
            comm.allreduce(ins, outs, protocol="ll")
        torch.cuda.synchronize()
        assert comm.status()[0] == api.Status.OK
    finally:
        comm.close()
