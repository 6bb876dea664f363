"""Closed forms of what the collectives compute.

All-reduce: every rank r receives, for every element i,

    out[r][i] = bf16_RNE( (...((f32(x_0[i]) + f32(x_1[i])) + f32(x_2[i])) ...) + f32(x_{N-1}[i]) )

with binary32 round-to-nearest-even additions taken in rank order 0..N-1,
starting from x_0 (not from 0.0, so that an all -0 input stays -0), and one
final rounding to bf16. "flash-comm: Self-Synchronizing Collective
Communication for LLM Decoding", abstract: the reduction order is fixed and
independent of the order in which data arrives, so every rank obtains the same
result. Because the order is fixed, the result is one definite bit pattern,
which is what the GPU path must reproduce bit for bit.

All-gather: every rank receives the concatenation in[0] || in[1] || ... ||
in[N-1] (same abstract: the mechanism also serves a standalone all-gather).
"""

import numpy as np

from .bf16 import bf16_bits_to_f32, f32_to_bf16_bits  # noqa: F401 (re-exported)

__all__ = [
    "allreduce",
    "allreduce_all_ranks",
    "allgather",
    "allreduce_fp64",
    "fp64_error_bound",
    "rank_order_sum_f32",
]


def rank_order_sum_f32(inputs):
    """fp32 fold of N bf16 rows in rank order 0..N-1; returns float32 [count]."""
    x = np.asarray(inputs, dtype=np.uint16)
    if x.ndim != 2 or x.shape[0] < 1:
        raise ValueError("inputs must be [N, count] bf16 bit patterns")
    acc = bf16_bits_to_f32(x[0]).copy()
    with np.errstate(over="ignore", invalid="ignore"):  # IEEE inf / NaN results are wanted
        for q in range(1, x.shape[0]):
            acc = np.add(acc, bf16_bits_to_f32(x[q]), dtype=np.float32)
    return acc


def allreduce(inputs):
    """All-reduce result (identical on every rank): bf16 bits [count]."""
    return f32_to_bf16_bits(rank_order_sum_f32(inputs))


def allreduce_all_ranks(inputs):
    """The N per-rank outputs, [N, count]; every row equals ``allreduce``."""
    x = np.asarray(inputs, dtype=np.uint16)
    row = allreduce(x)
    return np.broadcast_to(row, x.shape).copy()


def allgather(inputs):
    """All-gather result for every rank: bf16 bits [N * count]."""
    x = np.asarray(inputs, dtype=np.uint16)
    return x.reshape(-1).copy()


def allreduce_fp64(inputs):
    """Exact-as-fp64 sum of the bf16 inputs (float64 [count])."""
    x = np.asarray(inputs, dtype=np.uint16)
    return bf16_bits_to_f32(x).astype(np.float64).sum(axis=0)


def fp64_error_bound(inputs):
    """Componentwise bound 2^-7 * N * sum_r |x_r| on |out - sum64|.

    The required accuracy is "within 2^-7 * N relative error of an fp64 sum";
    taken componentwise against sum |x_r| because a bound relative to |sum|
    cannot hold under cancellation. It covers the N-1 fp32 roundings
    (each at most 2^-24 relative to a partial sum bounded by sum |x_r|) and
    the final bf16 rounding (at most 2^-8 relative).
    """
    x = np.asarray(inputs, dtype=np.uint16)
    n = x.shape[0]
    mag = np.abs(bf16_bits_to_f32(x).astype(np.float64)).sum(axis=0)
    return (2.0 ** -7) * n * mag
