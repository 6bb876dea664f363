"""Row-parallel linear layer followed by its all-reduce: exact value and the
error bound a bf16 / fp32 implementation must stay within.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The layer is the tensor-parallel decode step the pages build on: every rank r
holds its slice W_r (bf16 [hidden, kdim]) of the weight and its slice x_r
(bf16 [tokens, kdim]) of the activation, computes the partial product
d_r = x_r W_r^T, and the partials are all-reduced so that every rank holds
y = sum_r d_r ("SiFAR: Synchronization-Free All-Reduce for Low-Latency LLM
Inference", introduction: the all-reduce that follows each tensor-parallel
layer). "Why Microseconds Matter in AI Infrastructure", section "Communication
is becoming part of GPU execution", puts the low-latency send / receive /
reduce inside the kernel that produces the data; the fused layer does that,
so the partials never reach global memory and cannot be compared on their
own.

What an implementation computes and how far it may be from the exact value:

* p_r = bf16_RNE(acc_r), where acc_r is an fp32 accumulation of the kdim
  products W_r[h, k] * x_r[t, k] in an order the implementation chooses
  (every product of two bf16 values is exact in fp32). Any summation order of
  kdim terms whose partial sums are rounded to a precision with unit roundoff
  u is within gamma_kdim(u) * a_r of the exact sum, with
  gamma_m(u) = m u / (1 - m u) and a_r = sum_k |W_r[h, k] x_r[t, k]|
  (the standard bound for any summation tree: no path through it has more
  than kdim roundings). u = 2^-24 for round-to-nearest fp32 adds; the bound
  here takes u = 2^-23, which also covers accumulators that truncate to fp32
  precision instead of rounding to nearest. The bf16 rounding of acc_r adds
  at most 2^-8 |acc_r| <= 2^-8 (|d_r| + gamma a_r).
* y = bf16_RNE(fold_fp32(p_0, ..., p_{N-1})), the rank-order all-reduce of
  the partials (the closed form in ``reference``): N - 1 fp32 adds, each
  within 2^-24 of a partial sum bounded by sum_r |p_r|, then one bf16
  rounding within 2^-8 of the fp32 result.

Hence |y - D| <= E + F + 2^-8 (|D| + E + F) with D = sum_r d_r,
E = sum_r e_r, e_r = 2^-8 |d_r| + (1 + 2^-8) gamma_kdim a_r, and
F = gamma_{N-1}(2^-24) sum_r (|d_r| + e_r). The library primitive used for
the exact value is a float64 product (every bf16 product and every partial
sum of the test sizes is exact or within 2^-53 relative in float64, far
below the bound).
"""

import numpy as np

from .bf16 import bf16_bits_to_f32

__all__ = ["partials_fp64", "partial_magnitudes", "linear_allreduce_fp64", "linear_allreduce_error_bound", "gamma"]

U_ACC = 2.0 ** -23  # unit roundoff assumed for the kdim-term accumulation
U_F32 = 2.0 ** -24  # fp32 round-to-nearest adds of the all-reduce fold
U_BF16 = 2.0 ** -8  # one rounding to bf16 (8 significant bits)


def gamma(m, u):
    """gamma_m(u) = m u / (1 - m u): the relative error bound of m roundings."""
    mu = m * u
    if mu >= 1.0:
        raise ValueError("gamma undefined: m * u >= 1")
    return mu / (1.0 - mu)


def _as_f64(bits):
    return bf16_bits_to_f32(np.asarray(bits, dtype=np.uint16)).astype(np.float64)


def _shapes(W, x):
    W = np.asarray(W, dtype=np.uint16)
    x = np.asarray(x, dtype=np.uint16)
    if W.ndim != 3:
        raise ValueError("W must be [N, hidden, kdim] bf16 bit patterns")
    if x.ndim == 2:
        x = x[:, None, :]
    if x.ndim != 3 or x.shape[0] != W.shape[0] or x.shape[2] != W.shape[2]:
        raise ValueError("x must be [N, kdim] or [N, tokens, kdim] matching W")
    return W, x


def partials_fp64(W, x):
    """d[r, t, h] = sum_k W[r, h, k] * x[r, t, k] in float64 ([N, tokens, hidden])."""
    W, x = _shapes(W, x)
    wf, xf = _as_f64(W), _as_f64(x)
    return np.einsum("rhk,rtk->rth", wf, xf)


def partial_magnitudes(W, x):
    """a[r, t, h] = sum_k |W[r, h, k] * x[r, t, k]| in float64."""
    W, x = _shapes(W, x)
    wf, xf = np.abs(_as_f64(W)), np.abs(_as_f64(x))
    return np.einsum("rhk,rtk->rth", wf, xf)


def linear_allreduce_fp64(W, x):
    """D[t, h] = sum_r d[r, t, h]: the exact value every rank's output
    approximates ([tokens, hidden])."""
    return partials_fp64(W, x).sum(axis=0)


def linear_allreduce_error_bound(W, x):
    """Componentwise bound on |y - D| for any implementation that rounds each
    partial to bf16 after an fp32 accumulation in any order and all-reduces
    the partials by the rank-order fold ([tokens, hidden])."""
    W, x = _shapes(W, x)
    n, _, kdim = W.shape
    d = partials_fp64(W, x)
    a = partial_magnitudes(W, x)
    g = gamma(kdim, U_ACC)
    e = U_BF16 * np.abs(d) + (1.0 + U_BF16) * g * a
    E = e.sum(axis=0)
    F = gamma(max(n - 1, 0), U_F32) * (np.abs(d) + e).sum(axis=0)
    D = d.sum(axis=0)
    return E + F + U_BF16 * (np.abs(D) + E + F)
