"""Pins of the row-parallel linear + all-reduce oracle (oracle/linear.py):
hand-worked values, index order, additivity over ranks and tokens, and the
error bound against simulated fp32 / bf16 arithmetic in several summation
orders (the bound must cover every one and still be far from vacuous)."""
import os

import numpy as np
import pytest

from latency_self_synchronizing_b200.inputs import make_inputs
from oracle import linear, reference
from oracle.bf16 import bf16_bits_to_f32, f32_to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "linear_allreduce.txt")


def _golden():
    cases = []
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if not line:
            continue
        head, w, x, y, a = [s.split() for s in line.split("|")]
        name, n, hidden, kdim, tokens = head[0], *map(int, head[1:])
        W = np.array([int(h, 16) for h in w], dtype=np.uint16).reshape(n, hidden, kdim)
        X = np.array([int(h, 16) for h in x], dtype=np.uint16).reshape(n, tokens, kdim)
        Y = np.array([float(v) for v in y]).reshape(tokens, hidden)
        A = np.array([float(v) for v in a]).reshape(n, tokens, hidden)
        cases.append((name, W, X, Y, A))
    return cases


@pytest.mark.parametrize("case", _golden(), ids=lambda c: c[0])
def test_worked_cases(case):
    _, W, X, Y, A = case
    np.testing.assert_array_equal(linear.linear_allreduce_fp64(W, X), Y)
    np.testing.assert_array_equal(linear.partial_magnitudes(W, X), A)
    assert linear.partials_fp64(W, X).shape == (W.shape[0], X.shape[1], W.shape[1])


def test_one_hot_tokens_pick_weight_columns():
    # non-square shapes: a transposed operand cannot even broadcast
    n, hidden, kdim = 3, 5, 7
    W = make_inputs(seed=11, k_ops=1, nranks=n, count=hidden * kdim, dist="normal", params=(1.0,))[0]
    W = W.reshape(n, hidden, kdim)
    for k in range(kdim):
        x = np.zeros((n, kdim), dtype=np.uint16)
        x[:, k] = 0x3F80  # 1.0
        d = linear.partials_fp64(W, x)[:, 0, :]
        np.testing.assert_array_equal(d, bf16_bits_to_f32(W[:, :, k]).astype(np.float64))


def test_additive_over_ranks_and_tokens():
    n, hidden, kdim, tokens = 4, 6, 40, 3
    W = make_inputs(seed=3, k_ops=1, nranks=n, count=hidden * kdim, dist="normal", params=(0.5,))[0]
    W = W.reshape(n, hidden, kdim)
    x = make_inputs(seed=4, k_ops=1, nranks=n, count=tokens * kdim, dist="normal", params=(1.0,))[0]
    x = x.reshape(n, tokens, kdim)
    full = linear.linear_allreduce_fp64(W, x)
    per_rank = sum(linear.linear_allreduce_fp64(W[r:r + 1], x[r:r + 1]) for r in range(n))
    np.testing.assert_allclose(full, per_rank, rtol=0, atol=1e-12)
    for t in range(tokens):
        np.testing.assert_array_equal(full[t], linear.linear_allreduce_fp64(W, x[:, t, :])[0])


def _simulated(W, x, order, rng):
    """One implementation: fp32 accumulation of the kdim products in `order`,
    bf16 rounding of every partial, rank-order fold of the partials."""
    n, hidden, kdim = W.shape
    tokens = x.shape[1]
    wf = bf16_bits_to_f32(W)
    xf = bf16_bits_to_f32(x)
    prod = np.einsum("rhk,rtk->rthk", wf.astype(np.float64), xf.astype(np.float64)).astype(np.float32)
    if order == "forward":
        idx = [np.arange(kdim)]
    elif order == "reverse":
        idx = [np.arange(kdim)[::-1]]
    elif order == "random":
        idx = [rng.permutation(kdim)]
    else:
        idx = None
    if idx is not None:
        acc = np.zeros(prod.shape[:-1], dtype=np.float32)
        for k in idx[0]:
            acc = np.add(acc, prod[..., k], dtype=np.float32)
    else:  # pairwise tree
        cur = prod
        while cur.shape[-1] > 1:
            if cur.shape[-1] % 2:
                cur = np.concatenate([cur, np.zeros(cur.shape[:-1] + (1,), np.float32)], axis=-1)
            cur = np.add(cur[..., 0::2], cur[..., 1::2], dtype=np.float32)
        acc = cur[..., 0]
    p = f32_to_bf16_bits(acc)  # [n, tokens, hidden]
    y = np.stack([reference.allreduce(p[:, t, :]) for t in range(tokens)])
    return bf16_bits_to_f32(y).astype(np.float64)


@pytest.mark.parametrize("n,hidden,kdim,tokens", [(2, 16, 64, 1), (4, 8, 512, 2), (8, 4, 1000, 1), (3, 12, 200, 3)])
def test_bound_covers_simulated_arithmetic(n, hidden, kdim, tokens):
    rng = np.random.default_rng(n * 1000 + kdim)
    W = make_inputs(seed=kdim, k_ops=1, nranks=n, count=hidden * kdim, dist="normal", params=(0.05,))[0]
    W = W.reshape(n, hidden, kdim)
    x = make_inputs(seed=kdim + 1, k_ops=1, nranks=n, count=tokens * kdim, dist="normal", params=(1.0,))[0]
    x = x.reshape(n, tokens, kdim)
    D = linear.linear_allreduce_fp64(W, x)
    bound = linear.linear_allreduce_error_bound(W, x)
    a = linear.partial_magnitudes(W, x).sum(axis=0)
    worst = 0.0
    for order in ("forward", "reverse", "random", "pairwise"):
        y = _simulated(W, x, order, rng)
        assert np.all(np.abs(y - D) <= bound), order
        worst = max(worst, float(np.max(np.abs(y - D) / bound)))
    # not vacuous: far below the magnitudes involved
    assert np.all(bound <= 2.0 ** -5 * (np.abs(D) + a))
    assert worst > 0.0


def test_bound_catches_a_dropped_product_block():
    # a partial that misses 8 of its products (one 16-byte piece of a weight
    # row) leaves the bound for most outputs
    n, hidden, kdim = 4, 64, 256
    W = make_inputs(seed=21, k_ops=1, nranks=n, count=hidden * kdim, dist="normal", params=(0.05,))[0]
    W = W.reshape(n, hidden, kdim)
    x = make_inputs(seed=22, k_ops=1, nranks=n, count=kdim, dist="normal", params=(1.0,))[0]
    D = linear.linear_allreduce_fp64(W, x)[0]
    bound = linear.linear_allreduce_error_bound(W, x)[0]
    Wd = W.copy()
    Wd[1, :, 8:16] = 0
    wrong = linear.linear_allreduce_fp64(Wd, x)[0]
    assert np.mean(np.abs(wrong - D) > bound) > 0.5


def test_gamma():
    assert linear.gamma(0, 2.0 ** -24) == 0.0
    assert linear.gamma(1, 0.5) == 1.0
    with pytest.raises(ValueError):
        linear.gamma(4, 0.25)
