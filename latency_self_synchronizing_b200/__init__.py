"""Self-synchronizing small-message all-reduce / all-gather on one B200.

N ranks are emulated inside one GPU as co-resident groups of CTAs of a
persistent sm_100a kernel. Each data block carries its own readiness evidence
(LL flag packing, LL128 lines, or a sentinel pre-fill), epoch-parity double
buffering removes the bottom barrier, and a fixed rank-order fp32 reduction
with one final bf16 rounding gives every rank the same bits. The compute path
lives in ``libsfc.so`` (C ABI declared in ``include/sfc.h``); this package is a
thin ctypes binding over it. Importing the package loads nothing: the library
is opened on first use and a missing library is an error, never a fallback.
"""

__all__ = ["lib", "Communicator", "Protocol", "Op", "Status", "SfcError"]


def __getattr__(name):
    if name in ("Communicator", "Protocol", "Op", "Status", "SfcError"):
        from . import api

        return getattr(api, name)
    if name == "lib":
        from . import _lib

        return _lib
    raise AttributeError(name)
