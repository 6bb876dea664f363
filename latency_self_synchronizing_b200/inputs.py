"""Seeded synthetic inputs shared by the tests, the bench and the CPU oracle.

This module holds none of the collective's arithmetic: it only draws numbers.
Each (operation k, rank r) gets its own PCG64 stream, spawned from
``numpy.random.SeedSequence(seed)`` in row-major (k, r) order, so an input
does not depend on how many other inputs are drawn. fp32 samples are narrowed
to bf16 by torch's CPU conversion (a library routine, round to nearest even);
the results are returned as uint16 bit patterns, shape [K, N, count].

Distributions follow the tensor-parallel decode traffic the pages motivate
("Why Microseconds Matter in AI Infrastructure", section "Latency can matter
more than bandwidth": small per-layer all-reduces of activations).
"""

import numpy as np
import torch

__all__ = ["make_inputs", "bf16_bits", "SENTINEL_BITS"]

SENTINEL_BITS = 0xFFFF


def bf16_bits(f32):
    """fp32 array -> bf16 bit patterns (uint16) via torch's RNE conversion."""
    t = torch.from_numpy(np.ascontiguousarray(f32, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def _draw(gen, dist, count, params):
    if dist == "uniform":
        lo, hi = params
        return gen.uniform(lo, hi, count).astype(np.float32)
    if dist == "normal":
        (sigma,) = params
        return (gen.standard_normal(count, dtype=np.float32) * np.float32(sigma)).astype(np.float32)
    raise ValueError(f"unknown distribution {dist!r}")


def make_inputs(seed, k_ops, nranks, count, dist="normal", params=(1.0,)):
    """uint16 [k_ops, nranks, count] of bf16 bits; never the sentinel pattern."""
    children = np.random.SeedSequence(seed).spawn(k_ops * nranks)
    out = np.empty((k_ops, nranks, count), dtype=np.uint16)
    for k in range(k_ops):
        for r in range(nranks):
            gen = np.random.Generator(np.random.PCG64(children[k * nranks + r]))
            out[k, r] = bf16_bits(_draw(gen, dist, count, params))
    if np.any(out == SENTINEL_BITS):  # finite samples never round to it
        raise AssertionError("input generator produced the sentinel pattern")
    return out
