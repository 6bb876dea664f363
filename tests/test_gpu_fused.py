"""The fused row-parallel linear + all-reduce against the oracle
(oracle/linear.py): the exact value of the layer and the error bound of any
implementation that accumulates each partial in fp32 in its own order, rounds
it to bf16 and all-reduces the partials by the rank-order fold. The partial
products are fp32 accumulations whose order is the kernel's, so they are not
bit-exact to any plain definition; every rank's output must be bit-identical.
"""
import numpy as np
import pytest
import torch

from latency_self_synchronizing_b200 import api
from latency_self_synchronizing_b200.inputs import make_inputs
from oracle import linear
from oracle.bf16 import bf16_bits_to_f32

pytestmark = pytest.mark.gpu


def _bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _case(n, hidden, kdim, seed):
    w = make_inputs(seed=seed, k_ops=1, nranks=n, count=hidden * kdim, dist="normal", params=(0.05,))[0]
    x = make_inputs(seed=seed + 1, k_ops=1, nranks=n, count=kdim, dist="normal", params=(1.0,))[0]
    return w.reshape(n, hidden, kdim), x


# shapes cover every column split the launch picks (ks = 1, 2, 4, 8 warps per vector)
@pytest.mark.parametrize("n,hidden,kdim", [(2, 8, 8), (2, 1000, 512), (4, 8192, 7168), (8, 4096, 1024),
                                           (2, 64, 8192), (6, 1536, 4096), (3, 2056, 136), (8, 24, 8),
                                           (5, 2048, 1024), (7, 1536, 2048)])
def test_linear_allreduce_within_bound(n, hidden, kdim):
    w, x = _case(n, hidden, kdim, seed=hidden + kdim + n)
    comm = api.Communicator(n, hidden * 2, protocols=["ll"])
    try:
        W = [_bf16_dev(w[r]) for r in range(n)]
        X = [_bf16_dev(x[r]) for r in range(n)]
        Y = [torch.empty(hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
        for _ in range(2):  # two epochs in a row
            comm.linear_allreduce(W, X, Y)
            torch.cuda.synchronize()
            assert comm.status()[0] == api.Status.OK
            ys = [Y[r].cpu().view(torch.int16).numpy().view(np.uint16) for r in range(n)]
            for r in range(1, n):
                np.testing.assert_array_equal(ys[r], ys[0])
            exact = linear.linear_allreduce_fp64(w, x)[0]
            bound = linear.linear_allreduce_error_bound(w, x)[0]
            got = bf16_bits_to_f32(ys[0]).astype(np.float64)
            assert np.all(np.abs(got - exact) <= bound)
    finally:
        comm.close()


def test_linear_allreduce_shares_the_epoch_sequence():
    n, hidden, kdim = 4, 64, 64
    w, x = _case(n, hidden, kdim, seed=5)
    comm = api.Communicator(n, 4096)
    try:
        W = [_bf16_dev(w[r]) for r in range(n)]
        X = [_bf16_dev(x[r]) for r in range(n)]
        Y = [torch.empty(hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
        e = comm.next_epoch
        comm.linear_allreduce(W, X, Y)
        assert comm.next_epoch == e + 1
        first = comm.reserve_epochs(3)
        assert first == e + 1 and comm.next_epoch == e + 4
        with pytest.raises(api.SfcError) as ei:
            comm.linear_allreduce(W, X, Y, epoch=e)
        assert ei.value.status == api.Status.EPOCH
        comm.linear_allreduce(W, X, Y)  # LL flags of the reserved epochs never appeared: still fine
        torch.cuda.synchronize()
        assert comm.status()[0] == api.Status.OK
        view = comm.ll_view()
        assert view.nranks == n and view.slot_stride > 0
    finally:
        comm.close()


# several decode tokens in one pass over the weights: ragged shapes on the
# CUDA cores with token tiles 2, 4, 8 (extra tokens masked), 2-8 tokens on
# 16-aligned shapes on the tensor cores (16 x 8 tiles): 16-byte weight pieces
# where each warp owns whole tiles, 32-byte pieces where 2-4 warps share one
# (4 x 512 x 4096, 4 x 4096 x 2048, and 2 x 256 x 2080 with its 32-column rest);
# a 96 KB activation at 2 and 4 ranks takes one CTA an SM (2 x 512 x 6144 on
# 32-byte pieces, 4 x 3584 x 6144 on 16-byte pieces)
@pytest.mark.parametrize("n,hidden,kdim,tokens", [(2, 64, 512, 2), (4, 8192, 3584, 4), (8, 1024, 1024, 8),
                                                  (3, 2056, 136, 3), (4, 512, 4096, 5), (2, 1000, 2048, 7),
                                                  (8, 64, 8, 6), (5, 8192, 1024, 8), (3, 2064, 144, 3),
                                                  (4, 4096, 2048, 2), (3, 2064, 160, 3), (2, 1000, 512, 2),
                                                  (2, 256, 2080, 3), (2, 512, 6144, 8),
                                                  (4, 3584, 6144, 8)])
def test_linear_allreduce_tokens_within_bound(n, hidden, kdim, tokens):
    w, _ = _case(n, hidden, kdim, seed=hidden * 3 + kdim + n + tokens)
    x = make_inputs(seed=hidden + tokens, k_ops=1, nranks=n, count=tokens * kdim, dist="normal",
                    params=(1.0,))[0].reshape(n, tokens, kdim)
    comm = api.Communicator(n, tokens * hidden * 2, protocols=["ll"])
    try:
        W = [_bf16_dev(w[r]) for r in range(n)]
        X = [_bf16_dev(x[r]) for r in range(n)]
        Y = [torch.empty(tokens, hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
        for _ in range(2):
            comm.linear_allreduce(W, X, Y)
            torch.cuda.synchronize()
            assert comm.status()[0] == api.Status.OK
            ys = [Y[r].cpu().view(torch.int16).numpy().view(np.uint16) for r in range(n)]
            for r in range(1, n):
                np.testing.assert_array_equal(ys[r], ys[0])
            exact = linear.linear_allreduce_fp64(w, x)
            bound = linear.linear_allreduce_error_bound(w, x)
            got = bf16_bits_to_f32(ys[0]).reshape(tokens, hidden).astype(np.float64)
            assert np.all(np.abs(got - exact) <= bound)
    finally:
        comm.close()


def test_linear_allreduce_tokens_weights_16_byte_aligned():
    """Weights that start 16 bytes past a 32-byte boundary take the 16-byte
    pieces on a shape that otherwise reads 32-byte pieces; same bound."""
    n, hidden, kdim, tokens = 4, 4096, 2048, 2
    w, _ = _case(n, hidden, kdim, seed=77)
    x = make_inputs(seed=78, k_ops=1, nranks=n, count=tokens * kdim, dist="normal",
                    params=(1.0,))[0].reshape(n, tokens, kdim)
    comm = api.Communicator(n, tokens * hidden * 2, protocols=["ll"])
    try:
        W = []
        for r in range(n):
            big = torch.empty(hidden * kdim + 8, dtype=torch.bfloat16, device="cuda")
            assert big.data_ptr() % 32 == 0
            view = big[8:].view(hidden, kdim)  # 16 bytes in
            view.copy_(_bf16_dev(w[r]).view(hidden, kdim))
            W.append(view)
        X = [_bf16_dev(x[r]) for r in range(n)]
        Y = [torch.empty(tokens, hidden, dtype=torch.bfloat16, device="cuda") for _ in range(n)]
        comm.linear_allreduce(W, X, Y)
        torch.cuda.synchronize()
        assert comm.status()[0] == api.Status.OK
        ys = [Y[r].cpu().view(torch.int16).numpy().view(np.uint16) for r in range(n)]
        for r in range(1, n):
            np.testing.assert_array_equal(ys[r], ys[0])
        exact = linear.linear_allreduce_fp64(w, x)
        bound = linear.linear_allreduce_error_bound(w, x)
        got = bf16_bits_to_f32(ys[0]).reshape(tokens, hidden).astype(np.float64)
        assert np.all(np.abs(got - exact) <= bound)
    finally:
        comm.close()
