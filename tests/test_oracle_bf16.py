"""Pins of the oracle's bf16 codec against IEEE 754 and a library routine."""
import os

import numpy as np
import torch

from oracle.bf16 import BF16_SENTINEL, bf16_bits_to_f32, f32_to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "bf16_rne.txt")


def _golden():
    rows = []
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if line:
            f, b = line.split()[:2]
            rows.append((int(f, 16), int(b, 16)))
    return rows


def test_worked_values():
    rows = _golden()
    f = np.array([r[0] for r in rows], dtype=np.uint32).view(np.float32)
    got = f32_to_bf16_bits(f)
    for (fb, want), g in zip(rows, got):
        assert int(g) == want, (hex(fb), hex(int(g)), hex(want))


def test_matches_torch_rne_on_random_bit_patterns():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 2**32, size=200_000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    keep = ~np.isnan(f)
    f = f[keep]
    ours = f32_to_bf16_bits(f)
    lib = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, lib)


def test_nearest_by_brute_force():
    # the chosen bf16 is never farther from x than either bf16 neighbour
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(5000) * 10.0 ** rng.integers(-30, 30, 5000)).astype(np.float32)
    b = f32_to_bf16_bits(x).astype(np.int64)
    v = bf16_bits_to_f32(b.astype(np.uint16)).astype(np.float64)
    for step in (-1, 1):
        w = bf16_bits_to_f32((b + step).astype(np.uint16)).astype(np.float64)
        ok = np.isfinite(w)
        d_v = np.abs(v - x.astype(np.float64))
        d_w = np.abs(w - x.astype(np.float64))
        assert np.all(d_v[ok] <= d_w[ok])
        tie = ok & (d_v == d_w)
        assert np.all((b[tie] & 1) == 0)  # ties go to even


def test_widening_is_exact_and_round_trips():
    b = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    f = bf16_bits_to_f32(b)
    back = f32_to_bf16_bits(f)
    nan = np.isnan(f)
    assert np.array_equal(back[~nan], b[~nan])
    assert np.all(np.isnan(bf16_bits_to_f32(back[nan])))


def test_sentinel_is_negative_nan():
    v = bf16_bits_to_f32(np.array([BF16_SENTINEL], dtype=np.uint16))[0]
    assert np.isnan(v)
    assert (BF16_SENTINEL >> 15) == 1


def test_no_flush_to_zero_in_fp32_adds():
    tiny = np.array([1], dtype=np.uint32).view(np.float32)  # 2^-149
    s = np.add(tiny, tiny, dtype=np.float32)
    assert s.view(np.uint32)[0] == 2  # 2^-148, not 0
