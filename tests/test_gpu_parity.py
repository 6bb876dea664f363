"""GPU parity: the CUDA library against the CPU oracle, bit for bit.

Every protocol, rank counts 2..8, ragged and multi-tile sizes, chained
epochs, both operations; the scratch invariants the protocols rely on; the
named workloads at their full sizes (sampled where the oracle would be slow).
All calls go through the C ABI (ctypes binding).
"""
import numpy as np
import pytest
import torch

from latency_self_synchronizing_b200 import api
from latency_self_synchronizing_b200.inputs import make_inputs
from oracle import protocols as OP
from oracle import reference
from oracle.bf16 import bf16_bits_to_f32

from _gpu_helpers import Operands, run_chain, slot_bytes

pytestmark = pytest.mark.gpu

AR_PROTOS = ["ll", "ll128", "sentinel", "barrier_oneshot", "barrier_twoshot", "barrier_oneshot_db", "ll_twoshot",
             "sentinel_twoshot", "ll128_fast"]
AG_PROTOS = ["ll", "ll128", "sentinel", "barrier_oneshot", "barrier_oneshot_db", "ll128_fast"]
RAGGED = [1, 7, 8, 9, 59, 60, 61, 255, 1000, 4099]


def _want_ar(x):
    return np.stack([reference.allreduce(x[k]) for k in range(x.shape[0])])


def _assert_ar(out, x):
    want = _want_ar(x)
    for r in range(x.shape[1]):
        np.testing.assert_array_equal(out[:, r, :], want, err_msg=f"rank {r}")


def _assert_ag(out, x):
    for k in range(x.shape[0]):
        want = reference.allgather(x[k])
        for r in range(x.shape[1]):
            np.testing.assert_array_equal(out[k, r], want, err_msg=f"op {k} rank {r}")


@pytest.fixture(scope="module")
def comms():
    made = {}

    def get(n, max_bytes=1 << 20, **kw):
        key = (n, max_bytes, tuple(sorted(kw.items())))
        if key not in made:
            made[key] = api.Communicator(n, max_bytes, **kw)
        return made[key]

    yield get
    for c in made.values():
        c.close()


@pytest.mark.parametrize("proto", AR_PROTOS)
@pytest.mark.parametrize("n", [2, 3, 4, 5, 6, 7, 8])
def test_allreduce_ragged_chain(comms, proto, n):
    comm = comms(n)
    for i, count in enumerate(RAGGED):
        x = make_inputs(seed=1000 * n + i, k_ops=3, nranks=n, count=count, dist="normal", params=(1.0,))
        _assert_ar(run_chain(comm, proto, x), x)


@pytest.mark.parametrize("proto", AG_PROTOS)
@pytest.mark.parametrize("n", [2, 3, 4, 5, 6, 7, 8])
def test_allgather_ragged_chain(comms, proto, n):
    comm = comms(n)
    for i, count in enumerate([1, 7, 8, 61, 1000, 4099]):
        x = make_inputs(seed=2000 * n + i, k_ops=3, nranks=n, count=count, dist="uniform", params=(-4.0, 4.0))
        _assert_ag(run_chain(comm, proto, x, op="allgather"), x)


@pytest.mark.parametrize("proto", AR_PROTOS)
def test_single_op_api_and_epoch_sequence(comms, proto):
    comm = api.Communicator(4, 1 << 16)
    try:
        for count in (8, 1000, 4096):
            x = make_inputs(seed=count, k_ops=1, nranks=4, count=count)
            ins = Operands(1, 4, count, fill=x)
            outs = Operands(1, 4, count)
            e = comm.next_epoch
            comm.allreduce(ins.tensors(0), outs.tensors(0), protocol=proto)
            assert comm.next_epoch == e + 1
            torch.cuda.synchronize()
            assert comm.status()[0] == api.Status.OK
            _assert_ar(outs.bits(), x)
    finally:
        comm.close()


def test_mixed_protocols_and_sizes_share_one_context(comms):
    """Epochs flow across calls with different protocols, sizes and CTA counts."""
    comm = comms(4, 1 << 20)
    rng = np.random.default_rng(5)
    for i in range(24):
        proto = AR_PROTOS[i % len(AR_PROTOS)]
        count = int(rng.choice([3, 64, 1000, 20000, 131072]))
        k = int(rng.integers(1, 5))
        x = make_inputs(seed=3000 + i, k_ops=k, nranks=4, count=count)
        _assert_ar(run_chain(comm, proto, x), x)
    for i in range(6):
        proto = AG_PROTOS[i % len(AG_PROTOS)]
        x = make_inputs(seed=3100 + i, k_ops=2, nranks=4, count=513)
        _assert_ag(run_chain(comm, proto, x, op="allgather"), x)


@pytest.mark.parametrize("proto", AR_PROTOS)
@pytest.mark.parametrize("ctas", [1, 3, 7])
def test_forced_cta_counts(proto, ctas):
    comm = api.Communicator(3, 1 << 18, ctas_per_rank=ctas)
    try:
        for count in (100, 20001):
            x = make_inputs(seed=ctas * 7 + count, k_ops=4, nranks=3, count=count)
            _assert_ar(run_chain(comm, proto, x), x)
    finally:
        comm.close()


def test_ll_flags_equal_last_epoch_of_each_parity(comms):
    n, count = 4, 1000
    comm = api.Communicator(n, 1 << 14)
    try:
        x = make_inputs(seed=77, k_ops=5, nranks=n, count=count)
        run_chain(comm, "ll", x)
        last = {1: comm.next_epoch - 1, 0: comm.next_epoch - 2}
        if last[1] % 2 == 0:
            last = {0: last[1], 1: last[0]}
        nvec = (count + 7) // 8
        for r in range(n):
            for par in (0, 1):
                for q in range(n):
                    if q == r:
                        continue
                    s = slot_bytes(comm, "ll", r, par, q)
                    words = s.view(np.uint32)
                    # GPU layout: 32-vector chunks of 1024 bytes; unit flags at odd words
                    used = np.zeros(words.size // 2, dtype=bool)
                    for v in range(nvec):
                        base = (v // 32) * 1024 + (v % 32) * 16
                        for half in (0, 512):
                            used[(base + half) // 8] = True
                            used[(base + half + 8) // 8] = True
                    flags = words[1::2][used]
                    assert np.all(flags == last[par]), (r, par, q)
    finally:
        comm.close()


@pytest.mark.parametrize("proto", ["sentinel", "sentinel_twoshot"])
def test_sentinel_slots_reset_after_chain(proto):
    n, count = 4, 3000
    comm = api.Communicator(n, 1 << 14)
    try:
        x = make_inputs(seed=78, k_ops=7, nranks=n, count=count)
        _assert_ar(run_chain(comm, proto, x), x)
        pars = (0, 1, 2, 3) if proto.endswith("twoshot") else (0, 1)  # twoshot: + all-gather slots
        for r in range(n):
            for par in pars:
                for q in range(n):
                    if q != r:
                        assert np.all(slot_bytes(comm, proto, r, par, q) == 0xFF)
    finally:
        comm.close()


def test_ll128_lines_carry_epoch_flag():
    n, count = 3, 600  # 10 lines
    comm = api.Communicator(n, 1 << 12)
    try:
        x = make_inputs(seed=79, k_ops=2, nranks=n, count=count)
        run_chain(comm, "ll128", x)
        e_last = comm.next_epoch - 1
        s = slot_bytes(comm, "ll128", 0, e_last & 1, 1)
        for line in range(10):
            flag = int(s[line * 128 + 120:line * 128 + 128].view(np.uint64)[0])
            assert flag == e_last
            lo, vals = OP.decode_unit(OP.LL128, s, line, count)
            np.testing.assert_array_equal(vals, x[1, 1, lo:lo + vals.size])
    finally:
        comm.close()


def test_fp64_bound_and_identical_ranks(comms):
    comm = comms(8)
    x = make_inputs(seed=81, k_ops=2, nranks=8, count=65536)
    out = run_chain(comm, "ll128", x)
    for k in range(2):
        got = bf16_bits_to_f32(out[k, 0]).astype(np.float64)
        assert np.all(np.abs(got - reference.allreduce_fp64(x[k])) <= reference.fp64_error_bound(x[k]))
        for r in range(8):
            np.testing.assert_array_equal(out[k, r], out[k, 0])


def test_order_sensitive_golden_on_gpu(comms):
    comm = comms(4)
    x = np.zeros((1, 4, 16), dtype=np.uint16)
    x[0, :, :] = np.array([0x3F80, 0x3B80, 0x3380, 0x3380], dtype=np.uint16)[:, None]
    for proto in AR_PROTOS:
        out = run_chain(comm, proto, x)
        assert np.all(out == 0x3F80), proto


# ----------------------------------------------------------- named workloads
def test_workload_ll_2k_full():
    """4 ranks, LL, 1024 elements, uniform[-1,1) seed 0, 100 chained ops."""
    comm = api.Communicator(4, 2048)
    try:
        x = make_inputs(seed=0, k_ops=100, nranks=4, count=1024, dist="uniform", params=(-1.0, 1.0))
        _assert_ar(run_chain(comm, "ll", x), x)
    finally:
        comm.close()


@pytest.mark.parametrize("tokens", [1, 2, 4, 8])
def test_workload_decode_h8192_sentinel_full(tokens):
    """4 ranks, sentinel, hidden 8192 x tokens, normal(0,1), 160 chained ops."""
    count = 8192 * tokens
    comm = api.Communicator(4, count * 2)
    try:
        x = make_inputs(seed=0, k_ops=160, nranks=4, count=count, dist="normal", params=(1.0,))
        _assert_ar(run_chain(comm, "sentinel", x), x)
    finally:
        comm.close()


@pytest.mark.parametrize("proto", ["ll128", "barrier_oneshot", "barrier_twoshot", "ll_twoshot", "sentinel_twoshot",
                                   "barrier_oneshot_db", "ll128_fast"])
@pytest.mark.parametrize("tokens", [1, 4, 16])
def test_workload_decode_h4096_full(proto, tokens):
    """8 ranks, hidden 4096 x tokens, normal(0,0.5), 64 chained ops."""
    count = 4096 * tokens
    comm = api.Communicator(8, count * 2)
    try:
        x = make_inputs(seed=0, k_ops=64, nranks=8, count=count, dist="normal", params=(0.5,))
        _assert_ar(run_chain(comm, proto, x), x)
    finally:
        comm.close()


@pytest.mark.parametrize("proto", AR_PROTOS)
@pytest.mark.parametrize("n", [2, 8])
def test_sweep_1mb_every_element(proto, n):
    """1 MB per rank (where the selector hands over to the barrier kernels):
    every element of every rank compared with the closed form."""
    count = (1 << 20) // 2
    comm = api.Communicator(n, 1 << 20, protocols=[proto])
    try:
        x = make_inputs(seed=(1 << 20) + n, k_ops=2, nranks=n, count=count)
        _assert_ar(run_chain(comm, proto, x), x)
    finally:
        comm.close()
        torch.cuda.empty_cache()


@pytest.mark.parametrize("n", [2, 4, 8])
def test_selected_protocol_16mb_every_element(n):
    """16 MB per rank with the protocol the selector picks there (and at
    1 MB): every element compared with the closed form."""
    nbytes = 16 << 20
    count = nbytes // 2
    probe = api.Communicator(n, 1 << 10)  # every protocol provisioned: the selector's own choice
    try:
        chosen = {probe.select_protocol("allreduce", b, n).name.lower() for b in (1 << 20, nbytes)}
    finally:
        probe.close()
    x = make_inputs(seed=nbytes + n, k_ops=2, nranks=n, count=count)
    want = _want_ar(x)
    for proto in sorted(chosen):
        comm = api.Communicator(n, nbytes, protocols=[proto])
        try:
            out = run_chain(comm, proto, x)
            for r in range(n):
                np.testing.assert_array_equal(out[:, r, :], want, err_msg=f"{proto} rank {r}")
        finally:
            comm.close()
            torch.cuda.empty_cache()


@pytest.mark.parametrize("proto", AR_PROTOS)
@pytest.mark.parametrize("n", [2, 8])
def test_sweep_64mb_sampled(proto, n):
    """64 MB per rank: every output compared at sampled indices (the head,
    the tail and 4096 random positions)."""
    nbytes = 64 << 20
    count = nbytes // 2
    comm = api.Communicator(n, nbytes, protocols=[proto])
    try:
        x = make_inputs(seed=nbytes + n, k_ops=2, nranks=n, count=count)
        out = run_chain(comm, proto, x)
        idx = np.unique(np.concatenate([np.arange(64), count - 64 + np.arange(64),
                                        np.random.default_rng(n).integers(0, count, 4096)]))
        for k in range(2):
            want = reference.allreduce(x[k][:, idx])
            for r in range(n):
                np.testing.assert_array_equal(out[k, r, idx], want)
    finally:
        comm.close()
        torch.cuda.empty_cache()


@pytest.mark.parametrize("proto", AG_PROTOS)
def test_workload_allgather_with_skew(proto):
    """8 ranks, every shard size 512 B .. 1 MB (powers of two), uniform[-4,4),
    exponential start skew (mean 2 us) per (op, rank); outputs equal to the
    closed form and bit-identical across 5 skew seeds."""
    n = 8
    for nbytes in [512 << i for i in range(12)]:
        count = nbytes // 2
        comm = api.Communicator(n, nbytes)
        try:
            x = make_inputs(seed=nbytes, k_ops=4, nranks=n, count=count, dist="uniform", params=(-4.0, 4.0))
            first = None
            for s in range(5):
                skew = np.random.default_rng(s).exponential(2000.0, size=4 * n).astype(np.int32)
                sk = torch.from_numpy(skew).cuda()
                out = run_chain(comm, proto, x, op="allgather", skew=sk)
                _assert_ag(out, x)
                if first is None:
                    first = out
                np.testing.assert_array_equal(out, first)
        finally:
            comm.close()


def test_timings_are_monotone(comms):
    comm = comms(4)
    x = make_inputs(seed=90, k_ops=20, nranks=4, count=8192)
    t = torch.zeros(21, dtype=torch.int64, device="cuda")
    run_chain(comm, "ll", x, timings=t)
    h = t.cpu().numpy().astype(np.uint64)
    assert np.all(np.diff(h[1:].astype(np.int64)) >= 0)
    assert h[1] >= h[0]


@pytest.mark.parametrize("proto", AR_PROTOS)
def test_guard_words_intact_after_large_chain(proto):
    comm = api.Communicator(8, 1 << 18, protocols=[proto])
    try:
        x = make_inputs(seed=91, k_ops=3, nranks=8, count=(1 << 17) - 3)
        _assert_ar(run_chain(comm, proto, x), x)
        assert comm.check_guards() == api.Status.OK
    finally:
        comm.close()


@pytest.mark.parametrize("proto", ["ll", "sentinel", "ll128_fast"])
@pytest.mark.parametrize("n", [4, 8])
def test_cta_size_boundary(comms, proto, n):
    """Messages up to 64 KB per rank at 4+ ranks run in 128-thread CTAs, larger
    ones in 256-thread CTAs; both sides of the boundary are bit-exact and both
    op kinds share one context and epoch sequence."""
    comm = comms(n, 1 << 17)
    for count, threads in [(32768, 128), (32769, 256), (8191, 128)]:
        assert comm.launch_shape("allreduce", proto, count)[1] == threads
        x = make_inputs(seed=count + n, k_ops=3, nranks=n, count=count)
        _assert_ar(run_chain(comm, proto, x), x)
        xg = make_inputs(seed=count + n + 1, k_ops=2, nranks=n, count=count // n)
        _assert_ag(run_chain(comm, proto, xg, op="allgather"), xg)


SPECIAL = np.array([0x0000, 0x8000, 0x0001, 0x8001, 0x007F, 0x807F, 0x0080, 0x8080, 0x7F7F, 0xFF7F, 0x7F00,
                    0xFF00, 0x3F80, 0xBF80, 0x7F80, 0xFF80], dtype=np.uint16)


def _special_inputs(seed, k, n, count):
    """bf16 edge values: signed zeros, subnormals (lost if anything flushed
    them), the smallest normal, the largest finite values (sums overflow to
    inf), infinities. An element with an infinite input gets only +inf and
    no large negative value, so no element meets +inf and -inf (a NaN, whose
    payload is not compared)."""
    rng = np.random.default_rng(seed)
    x = SPECIAL[rng.integers(0, len(SPECIAL), size=(k, n, count))]
    has_inf = np.broadcast_to(((x == 0x7F80) | (x == 0xFF80)).any(axis=1)[:, None, :], x.shape)
    x = np.where(has_inf & (x == 0xFF80), np.uint16(0x7F80), x)
    x = np.where(has_inf & ((x == 0xFF7F) | (x == 0xFF00)), np.uint16(0xBF80), x)
    return x


@pytest.mark.parametrize("proto", AR_PROTOS)
@pytest.mark.parametrize("n", [2, 3, 8])
def test_special_values_bit_exact(comms, proto, n):
    comm = comms(n)
    x = _special_inputs(seed=n * 31, k=2, n=n, count=4099)
    want = _want_ar(x)
    assert not np.any((want & 0x7FFF) > 0x7F80), "test inputs must not produce NaN"
    # the cases are present: subnormal or zero results, infinities, and -0 (n = 2)
    assert np.any((want & 0x7F80) == 0) and np.any((want & 0x7FFF) == 0x7F80)
    assert n != 2 or np.any(want == 0x8000)
    _assert_ar(run_chain(comm, proto, x), x)
