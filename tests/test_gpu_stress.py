"""Long-run robustness on the GPU: a million chained operations per
self-synchronizing protocol under random per-(operation, rank) start skew,
every output checked against the oracle, guard words intact afterwards.

The readiness logic is the part that could tear or race (a unit accepted
before all of it landed, a slot reused too early); the skew makes ranks
arrive in changing orders. Outputs are compared on the device with torch,
against expected values the CPU oracle computed for each distinct input set.
"""
import numpy as np
import pytest
import torch

from latency_self_synchronizing_b200 import api
from latency_self_synchronizing_b200.inputs import make_inputs
from oracle import reference

from _gpu_helpers import Operands

pytestmark = pytest.mark.gpu


def _run(proto, n, count, total_ops, skew_mean_ns, seed):
    sets = 64  # distinct input sets; operation i uses set i % 64 and output slot i % 64
    x = make_inputs(seed=seed, k_ops=sets, nranks=n, count=count)
    want = np.stack([reference.allreduce(x[s]) for s in range(sets)])  # [sets, count]
    comm = api.Communicator(n, 2 * count)
    try:
        ins = Operands(sets, n, count, fill=x)
        outs = Operands(sets, n, count)
        view = outs.buf.view(sets, n, outs.stride)[:, :, :count]
        want_dev = torch.from_numpy(want.view(np.int16)).cuda()[:, None, :].expand(sets, n, count)
        rng = np.random.default_rng(seed)
        skews = [torch.from_numpy(rng.exponential(skew_mean_ns, size=sets * n).astype(np.int32)).cuda()
                 for _ in range(16)]
        bad = torch.zeros((), dtype=torch.int64, device="cuda")
        launches = total_ops // sets
        for i in range(launches):
            comm.allreduce_chain(ins.table, outs.table, count, sets, protocol=proto, skew_ns=skews[i % 16])
            bad += (view != want_dev).sum()
            view.zero_()
        torch.cuda.synchronize()
        st, info = comm.status()
        assert st == api.Status.OK, (st, hex(info))
        assert int(bad) == 0, f"{int(bad)} wrong elements over {launches * sets} operations"
        assert comm.check_guards() == api.Status.OK
        assert comm.next_epoch == 1 + launches * sets
    finally:
        comm.close()


@pytest.mark.parametrize("proto", ["ll", "ll128", "sentinel", "ll_twoshot", "sentinel_twoshot", "ll128_fast"])
def test_million_ops_under_skew(proto):
    _run(proto, n=4, count=1000, total_ops=1_000_000, skew_mean_ns=300.0, seed=7)


@pytest.mark.parametrize("proto", ["ll", "sentinel", "ll128", "barrier_oneshot", "barrier_oneshot_db", "barrier_twoshot"])
def test_many_ops_eight_ranks(proto):
    _run(proto, n=8, count=4099, total_ops=1 << 17, skew_mean_ns=1000.0, seed=8)


@pytest.mark.parametrize("n,count", [(2, 60), (8, 600), (4, 120000)])
def test_ll128_one_load_tearing(n, count):
    """The one-load LL128 accepts data read in the same warp load as its flag;
    a torn line would show up here as a wrong element. Line-sized messages
    (one line, ten lines) and a large one, every output checked."""
    _run("ll128_fast", n=n, count=count, total_ops=1_000_000 if count < 100000 else 1 << 14,
         skew_mean_ns=200.0, seed=9 + n)


@pytest.mark.parametrize("proto", ["ll", "sentinel", "ll128_fast", "ll_twoshot", "sentinel_twoshot", "barrier_oneshot_db"])
@pytest.mark.parametrize("n", [3, 5, 6, 7])
def test_odd_rank_counts_under_skew(proto, n):
    """Rank counts the power-of-two cases do not reach (uneven twoshot shards,
    source indices that skip the own rank at every position), ragged size."""
    _run(proto, n=n, count=777, total_ops=1 << 15, skew_mean_ns=500.0, seed=20 + n)


@pytest.mark.parametrize("n,count", [(8, 32769), (4, 80000), (4, 65536), (2, 262147)])
def test_sentinel_load_polls_under_skew(n, count):
    """Large sentinel messages ((N - 1) x bytes >= 384 KB; 4 x 128 KB is the
    smallest power-of-two case) poll with loads and reset with stores behind
    a release fence: the resets must land before a writer reuses the slot two
    epochs later, under changing arrival orders."""
    _run("sentinel", n=n, count=count, total_ops=1 << 13, skew_mean_ns=2000.0, seed=30 + n)
