"""bfloat16 <-> binary32 codec written from the IEEE 754 definitions.

bfloat16 is the upper half of an IEEE 754 binary32 word: 1 sign bit, the same
8 exponent bits, 7 fraction bits. The set of bf16 values is therefore exactly
the set of binary32 values whose low 16 bits are zero, including subnormals,
infinities and NaNs. Widening (bf16 -> f32) appends 16 zero bits and is exact.

Narrowing with round-to-nearest, ties-to-even (IEEE 754 clause 4.3.1) picks,
of the two neighbouring bf16 values that bracket the binary32 value, the
nearer one, and on a tie the one whose last fraction bit is 0. For finite
values of one sign the binary32 bit pattern is monotone in magnitude, so the
two neighbours are the patterns ``hi = bits >> 16`` and ``hi + 1`` and the
distance to the lower one is the low 16 bits (``0x8000`` is the exact middle).
Rounding up may carry out of the fraction into the exponent; past the largest
finite exponent that carry produces the infinity pattern, which is what
round-to-nearest prescribes on overflow. NaN inputs are kept NaN with the sign
and the quiet bit set.

Used for the one final rounding of the fp32 rank-order sum ("flash-comm:
Self-Synchronizing Collective Communication for LLM Decoding", abstract:
identical results on every rank) and to widen bf16 inputs to fp32.
"""

import numpy as np

__all__ = ["f32_to_bf16_bits", "bf16_bits_to_f32", "BF16_SENTINEL"]

# The receive-buffer pre-fill of the sentinel protocol: a negative NaN
# ("Why Microseconds Matter in AI Infrastructure", section "Latency can matter
# more than bandwidth"). Sign 1, exponent all ones, fraction all ones.
BF16_SENTINEL = 0xFFFF


def f32_to_bf16_bits(x):
    """binary32 values -> bf16 bit patterns (uint16), round to nearest even."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    bits = x.view(np.uint32).astype(np.uint64)  # room for the carry
    hi = bits >> 16
    lo = bits & 0xFFFF
    odd = hi & 1
    round_up = (lo > 0x8000) | ((lo == 0x8000) & (odd == 1))
    out = hi + round_up.astype(np.uint64)
    is_nan = (bits & 0x7FFFFFFF) > 0x7F800000
    out = np.where(is_nan, hi | 0x0040, out)
    return out.astype(np.uint16)


def bf16_bits_to_f32(b):
    """bf16 bit patterns (uint16) -> exact binary32 values."""
    b = np.ascontiguousarray(np.asarray(b, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32)
