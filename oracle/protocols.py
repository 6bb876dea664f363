"""Byte-level readiness encodings: LL, LL128 and sentinel.

Each encoding turns one source's bf16 chunk into *units*: the pieces a writer
stores atomically and a reader validates on its own. The receiver keeps one
slot per (parity, source); a unit is accepted when it validates against the
epoch being received.

Readings of the pages taken here ("Why Microseconds Matter in AI
Infrastructure", section "Latency can matter more than bandwidth", which names
LL flag packing, the LL128 design and the sentinel method but gives no
layouts):

* LL -- data and a readiness flag travel in one atomic store. Unit = 8 bytes,
  little endian: a 32-bit data word holding bf16 elements 2j (low half) and
  2j+1 (high half), then a 32-bit flag equal to the epoch. An odd count pads
  the last high half with +0. Valid iff flag == epoch.
* LL128 -- a 128-byte line: 120 bytes of data (60 bf16 elements, zero padded
  at the tail) followed by an 8-byte flag word whose value is the epoch (low
  32 bits = epoch, high 32 bits = 0). The line is the unit. Valid iff the
  flag word == epoch.
* Sentinel -- the raw bf16 element is the unit; the slot is pre-filled with
  the negative-NaN pattern 0xFFFF and an element is valid iff it differs from
  it. After consuming, the reader writes 0xFFFF back.

The epoch is a 32-bit counter starting at 1, so zero-filled memory never
validates for LL / LL128.
"""

import numpy as np

from .bf16 import BF16_SENTINEL

__all__ = [
    "LL",
    "LL128",
    "SENTINEL",
    "SELF_SYNC",
    "LL128_ELEMS_PER_LINE",
    "unit_count",
    "slot_bytes",
    "initial_slot",
    "encode_unit",
    "encode_all",
    "validate_unit",
    "decode_unit",
    "unit_elements",
    "reset_unit_bytes",
    "expansion",
]

LL = "ll"
LL128 = "ll128"
SENTINEL = "sentinel"
SELF_SYNC = (LL, LL128, SENTINEL)

LL_UNIT_BYTES = 8
LL128_LINE_BYTES = 128
LL128_DATA_BYTES = 120
LL128_ELEMS_PER_LINE = LL128_DATA_BYTES // 2  # 60


def unit_count(proto, count):
    """Number of units that carry ``count`` bf16 elements."""
    if proto == LL:
        return (count + 1) // 2
    if proto == LL128:
        return (count + LL128_ELEMS_PER_LINE - 1) // LL128_ELEMS_PER_LINE
    if proto == SENTINEL:
        return count
    raise ValueError(proto)


def unit_bytes(proto):
    return {LL: LL_UNIT_BYTES, LL128: LL128_LINE_BYTES, SENTINEL: 2}[proto]


def slot_bytes(proto, count):
    return unit_count(proto, count) * unit_bytes(proto)


def expansion(proto, count):
    """Encoded bytes per data byte (e in the roofline accounting)."""
    if count == 0:
        return 0.0
    return slot_bytes(proto, count) / (2.0 * count)


def initial_slot(proto, count):
    """Slot contents before any epoch: zeros (LL, LL128) or sentinel fill."""
    n = slot_bytes(proto, count)
    if proto == SENTINEL:
        return np.full(n, 0xFF, dtype=np.uint8)
    return np.zeros(n, dtype=np.uint8)


def unit_elements(proto, count, j):
    """Element indices [lo, hi) that unit j carries (real elements only)."""
    if proto == LL:
        lo = 2 * j
        return lo, min(lo + 2, count)
    if proto == LL128:
        lo = LL128_ELEMS_PER_LINE * j
        return lo, min(lo + LL128_ELEMS_PER_LINE, count)
    if proto == SENTINEL:
        return j, j + 1
    raise ValueError(proto)


def _u16_le(vals):
    v = np.asarray(vals, dtype=np.uint16)
    out = np.empty(2 * v.size, dtype=np.uint8)
    out[0::2] = (v & 0xFF).astype(np.uint8)
    out[1::2] = (v >> 8).astype(np.uint8)
    return out


def _u32_le(x):
    x = int(x) & 0xFFFFFFFF
    return np.array([(x >> (8 * i)) & 0xFF for i in range(4)], dtype=np.uint8)


def _u64_le(x):
    x = int(x) & 0xFFFFFFFFFFFFFFFF
    return np.array([(x >> (8 * i)) & 0xFF for i in range(8)], dtype=np.uint8)


def _read_u32(buf, off):
    b = buf[off:off + 4]
    return int(b[0]) | (int(b[1]) << 8) | (int(b[2]) << 16) | (int(b[3]) << 24)


def _read_u64(buf, off):
    lo = _read_u32(buf, off)
    hi = _read_u32(buf, off + 4)
    return lo | (hi << 32)


def encode_unit(proto, data, j, epoch):
    """(byte offset, bytes) of unit j of ``data`` (bf16 bits) at ``epoch``."""
    data = np.asarray(data, dtype=np.uint16)
    count = data.size
    lo, hi = unit_elements(proto, count, j)
    if proto == LL:
        elems = np.zeros(2, dtype=np.uint16)  # pad element = +0
        elems[: hi - lo] = data[lo:hi]
        body = np.concatenate([_u16_le(elems), _u32_le(epoch)])
        return LL_UNIT_BYTES * j, body
    if proto == LL128:
        elems = np.zeros(LL128_ELEMS_PER_LINE, dtype=np.uint16)
        elems[: hi - lo] = data[lo:hi]
        body = np.concatenate([_u16_le(elems), _u64_le(epoch & 0xFFFFFFFF)])
        return LL128_LINE_BYTES * j, body
    if proto == SENTINEL:
        return 2 * j, _u16_le(data[lo:hi])
    raise ValueError(proto)


def encode_all(proto, data, epoch):
    """Every unit of ``data``: list of (offset, bytes)."""
    data = np.asarray(data, dtype=np.uint16)
    return [encode_unit(proto, data, j, epoch) for j in range(unit_count(proto, data.size))]


def validate_unit(proto, slot, j, epoch):
    """Readiness test of unit j against ``epoch`` (the receiver's poll)."""
    if proto == LL:
        return _read_u32(slot, LL_UNIT_BYTES * j + 4) == (epoch & 0xFFFFFFFF)
    if proto == LL128:
        return _read_u64(slot, LL128_LINE_BYTES * j + LL128_DATA_BYTES) == (epoch & 0xFFFFFFFF)
    if proto == SENTINEL:
        off = 2 * j
        return (int(slot[off]) | (int(slot[off + 1]) << 8)) != BF16_SENTINEL
    raise ValueError(proto)


def decode_unit(proto, slot, j, count):
    """(lo, values) -- the real elements unit j carries, as bf16 bits."""
    lo, hi = unit_elements(proto, count, j)
    n = hi - lo
    if proto == LL:
        off = LL_UNIT_BYTES * j
    elif proto == LL128:
        off = LL128_LINE_BYTES * j
    elif proto == SENTINEL:
        off = 2 * j
    else:
        raise ValueError(proto)
    b = slot[off:off + 2 * n]
    vals = (b[0::2].astype(np.uint16) | (b[1::2].astype(np.uint16) << 8)).astype(np.uint16)
    return lo, vals


def reset_unit_bytes(proto, j):
    """(offset, bytes) the sentinel reader writes back after consuming unit j."""
    if proto != SENTINEL:
        raise ValueError("only the sentinel protocol resets its receive buffer")
    return 2 * j, np.array([0xFF, 0xFF], dtype=np.uint8)
