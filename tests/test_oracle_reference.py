"""Pins of the closed forms: worked cases, the fp64 bound, brute force."""
import itertools
import os

import numpy as np

from latency_self_synchronizing_b200.inputs import make_inputs
from oracle import reference
from oracle.bf16 import bf16_bits_to_f32

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "rank_order_sum.txt")


def _cases():
    out = []
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if not line:
            continue
        left, right = line.split("->")
        parts = left.split()
        n = int(parts[1])
        xs = [int(h, 16) for h in parts[2:2 + n]]
        want, wrong = [int(h, 16) for h in right.replace("|", " ").split()]
        out.append((parts[0], xs, want, wrong))
    return out


def test_order_sensitive_worked_cases():
    for name, xs, want, wrong in _cases():
        x = np.array(xs, dtype=np.uint16).reshape(-1, 1)
        got = int(reference.allreduce(x)[0])
        assert got == want, (name, hex(got))
        assert got != wrong


def test_fp64_bound_random():
    for n in range(2, 9):
        x = make_inputs(seed=n, k_ops=1, nranks=n, count=4096, dist="normal", params=(1.0,))[0]
        out = bf16_bits_to_f32(reference.allreduce(x)).astype(np.float64)
        err = np.abs(out - reference.allreduce_fp64(x))
        assert np.all(err <= reference.fp64_error_bound(x))


def test_fp64_bound_catches_a_dropped_term():
    x = make_inputs(seed=9, k_ops=1, nranks=4, count=4096)[0]
    dropped = reference.allreduce(x[:3])
    err = np.abs(bf16_bits_to_f32(dropped).astype(np.float64) - reference.allreduce_fp64(x))
    assert np.any(err > reference.fp64_error_bound(x))


def test_two_ranks_is_the_correctly_rounded_sum():
    # N=2: one fp32 add of two bf16 values whose exact sum fits in fp32, so the
    # result must be the bf16 nearest (ties to even) to the exact sum
    rng = np.random.default_rng(3)
    x = make_inputs(seed=4, k_ops=1, nranks=2, count=20000)[0]
    exact = bf16_bits_to_f32(x).astype(np.float64).sum(axis=0)
    b = reference.allreduce(x).astype(np.int64)
    v = bf16_bits_to_f32(b.astype(np.uint16)).astype(np.float64)
    for step in (-1, 1):
        w = bf16_bits_to_f32((b + step).astype(np.uint16)).astype(np.float64)
        ok = np.isfinite(w) & (np.sign(w) == np.sign(v))
        assert np.all(np.abs(v - exact)[ok] <= np.abs(w - exact)[ok])
    del rng


def test_negative_zero_and_subnormals():
    x = np.full((4, 3), 0x8000, dtype=np.uint16)  # -0 everywhere
    assert np.all(reference.allreduce(x) == 0x8000)
    y = np.array([[0x0001], [0x0001]], dtype=np.uint16)  # 2^-133 twice
    assert int(reference.allreduce(y)[0]) == 0x0002
    z = np.array([[0x8000], [0x0000]], dtype=np.uint16)  # -0 + +0 = +0
    assert int(reference.allreduce(z)[0]) == 0x0000


def test_overflow_goes_to_infinity():
    big = np.array([[0x7F7F], [0x7F7F]], dtype=np.uint16)  # bf16 max twice
    assert int(reference.allreduce(big)[0]) == 0x7F80


def test_brute_force_tiny():
    # every triple from a small value set: the fold equals a direct
    # left-to-right evaluation with Python floats rounded to fp32 per step
    vals = [0x3F80, 0xBF80, 0x3B80, 0x3380, 0x33C0, 0x4000, 0x0001, 0x8000]
    for t in itertools.product(vals, repeat=3):
        x = np.array(t, dtype=np.uint16).reshape(3, 1)
        f = [float(v) for v in bf16_bits_to_f32(np.array(t, dtype=np.uint16))]
        acc = np.float32(f[0])
        for v in f[1:]:
            acc = np.float32(float(acc) + v)  # exact in fp64, one rounding to fp32
        want = reference.f32_to_bf16_bits(np.array([acc], dtype=np.float32))[0]
        assert reference.allreduce(x)[0] == want


def test_allgather_is_concatenation():
    x = make_inputs(seed=5, k_ops=1, nranks=3, count=7)[0]
    g = reference.allgather(x)
    assert g.shape == (21,)
    for q in range(3):
        assert np.array_equal(g[7 * q:7 * (q + 1)], x[q])


def test_all_ranks_identical():
    x = make_inputs(seed=6, k_ops=1, nranks=5, count=33)[0]
    outs = reference.allreduce_all_ranks(x)
    assert all(np.array_equal(outs[0], outs[r]) for r in range(5))
