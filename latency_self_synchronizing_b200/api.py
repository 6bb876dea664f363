"""Python binding over libsfc: torch tensors and streams in, C ABI calls out.

Every step of the collective runs in the CUDA library; this module only
checks tensor metadata, collects device pointers and the current stream, and
turns status codes into exceptions.
"""

import ctypes as C
import enum

import torch

from . import _lib

__all__ = [
    "Status", "Protocol", "Op", "SfcError", "Communicator", "Plan", "pointer_table", "measure_floor",
    "algorithmic_bytes", "select_protocol_model", "default_cost_model", "status_string", "cost_estimate",
]


class Status(enum.IntEnum):
    OK = 0
    INVALID = 1
    CUDA = 2
    TIMEOUT = 3
    EPOCH = 4
    RESOURCES = 5
    SENTINEL_IN_INPUT = 6
    UNSUPPORTED = 7
    ABORTED = 8
    GUARD = 9


class Protocol(enum.IntEnum):
    AUTO = 0
    LL = 1
    LL128 = 2
    SENTINEL = 3
    BARRIER_ONESHOT = 4
    BARRIER_TWOSHOT = 5
    BARRIER_ONESHOT_DB = 6
    LL_TWOSHOT = 7
    SENTINEL_TWOSHOT = 8
    LL128_FAST = 9


class Op(enum.IntEnum):
    ALLREDUCE = 0
    ALLGATHER = 1


_NAMES = {"auto": Protocol.AUTO, "ll": Protocol.LL, "ll128": Protocol.LL128, "sentinel": Protocol.SENTINEL,
          "barrier_oneshot": Protocol.BARRIER_ONESHOT, "oneshot": Protocol.BARRIER_ONESHOT,
          "barrier_twoshot": Protocol.BARRIER_TWOSHOT, "twoshot": Protocol.BARRIER_TWOSHOT,
          "barrier_oneshot_db": Protocol.BARRIER_ONESHOT_DB, "oneshot_db": Protocol.BARRIER_ONESHOT_DB,
          "ll_twoshot": Protocol.LL_TWOSHOT, "sentinel_twoshot": Protocol.SENTINEL_TWOSHOT,
          "ll128_fast": Protocol.LL128_FAST}


def as_protocol(p):
    if isinstance(p, str):
        return _NAMES[p.lower()]
    return Protocol(int(p))


def as_op(o):
    if isinstance(o, str):
        return {"allreduce": Op.ALLREDUCE, "allgather": Op.ALLGATHER}[o.lower()]
    return Op(int(o))


class SfcError(RuntimeError):
    def __init__(self, status, what=""):
        self.status = Status(status)
        super().__init__(f"{what}: {status_string(status)} ({self.status.name})")


def status_string(s):
    return _lib.load().sfc_status_string(int(s)).decode()


def _check(rc, what):
    if rc != 0:
        raise SfcError(rc, what)


_raw_current_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream_handle(stream, device=None):
    """cudaStream_t of `stream`, or of the device's current stream."""
    if stream is not None:
        return C.c_void_p(stream.cuda_stream)
    if _raw_current_stream is not None and device is not None:
        return C.c_void_p(_raw_current_stream(device))
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dev_ptr(t, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def pointer_table(rows):
    """[[tensor per rank] per operation] -> int64 CUDA tensor of data pointers
    (every operand on one device, the table on that device too)."""
    ptrs = [_dev_ptr(t, "chain operand") for row in rows for t in row]
    dev = rows[0][0].device
    if any(t.device != dev for row in rows for t in row):
        raise ValueError(f"every chain operand must be on {dev}")
    return torch.tensor(ptrs, dtype=torch.int64, device=dev)


class Communicator:
    """N emulated ranks on the current CUDA device (one libsfc context)."""

    def __init__(self, nranks, max_bytes_per_rank, *, ctas_per_rank=0, timeout_us=0, debug_checks=False,
                 protocols=None, device_epochs=False):
        """device_epochs=True keeps the epoch sequence on the device: calls
        take no epoch, next_epoch reads 0, and calls can be captured in a
        CUDA graph and replayed (each replay continues the sequence)."""
        if not torch.cuda.is_available():
            raise RuntimeError("a CUDA device is required")
        self._lib = _lib.load()
        mask = 0
        if protocols is not None:
            for p in protocols:
                mask |= 1 << int(as_protocol(p))
        cfg = _lib.Config(int(ctas_per_rank), int(timeout_us), int(bool(debug_checks)), mask, int(bool(device_epochs)))
        handle = C.c_void_p()
        torch.cuda.init()
        _check(self._lib.sfc_init(C.byref(handle), int(nranks), int(max_bytes_per_rank), C.byref(cfg)), "sfc_init")
        self._ctx = handle
        self.nranks = int(nranks)
        self.max_bytes_per_rank = int(max_bytes_per_rank)
        self._device = torch.cuda.current_device()
        self._ptrs_in = (C.c_void_p * self.nranks)()
        self._ptrs_out = (C.c_void_p * self.nranks)()
        self._last = None  # (op, inputs, outputs, data pointers) of the last single call that passed the checks
        self._plans = []

    # ----------------------------------------------------------- lifecycle
    def close(self):
        for pl in getattr(self, "_plans", []):
            pl.close()  # plans go before their context
        self._plans = []
        if getattr(self, "_ctx", None):
            self._lib.sfc_destroy(self._ctx)
            self._ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    @property
    def next_epoch(self):
        return int(self._lib.sfc_next_epoch(self._ctx))

    def reset(self, stream=None):
        _check(self._lib.sfc_reset(self._ctx, _stream_handle(stream)), "sfc_reset")

    def status(self):
        """(Status, info) after synchronizing the last stream used."""
        info = C.c_uint32(0)
        rc = self._lib.sfc_get_status(self._ctx, C.byref(info))
        return Status(rc), int(info.value)

    def check_guards(self):
        """Status of the guard words around the scratch regions."""
        return Status(self._lib.sfc_check_guards(self._ctx))

    @property
    def launch_count(self):
        return int(self._lib.sfc_launch_count(self._ctx))

    # --------------------------------------------------------- collectives
    def _one(self, fn, op, inputs, outputs, protocol, epoch, stream):
        # per-call cost matters here (one launch per all-reduce): checks are
        # plain attribute reads, the pointer arrays are reused, the epoch is
        # left to the library (0 = next) and the stream read without a
        # Stream object. A call on the same tensor objects as the last one,
        # still at the same addresses and sizes (a decode loop on fixed
        # buffers), skips the metadata checks: they passed for these tensors.
        n = self.nranks
        last = self._last
        ptrs = None
        if last is not None and last[0] == op and len(inputs) == n and len(outputs) == n:
            li, lo, lp = last[1], last[2], last[3]
            if all(a is b for a, b in zip(inputs, li)) and all(a is b for a, b in zip(outputs, lo)):
                ptrs = [(t.data_ptr(), t.numel()) for t in inputs] + [(t.data_ptr(), t.numel()) for t in outputs]
                if ptrs != lp:
                    ptrs = None
        count = inputs[0].numel()
        if ptrs is None:
            self._last = None
            if len(inputs) != n or len(outputs) != n:
                raise ValueError(f"need {n} inputs and {n} outputs")
            want_out = count if op == Op.ALLREDUCE else n * count
            ins, outs = self._ptrs_in, self._ptrs_out
            bf16 = torch.bfloat16
            dev = self._device
            for r in range(n):
                a, b = inputs[r], outputs[r]
                if not (a.is_cuda and b.is_cuda and a.dtype is bf16 and b.dtype is bf16 and a.is_contiguous()
                        and b.is_contiguous()):
                    _dev_ptr(a, "input")
                    _dev_ptr(b, "output")
                if a.get_device() != dev or b.get_device() != dev:
                    raise ValueError(f"operands must be on cuda:{dev}, the communicator's device")
                if a.numel() != count:
                    raise ValueError("all inputs must have the same number of elements")
                if b.numel() != want_out:
                    raise ValueError(f"outputs must have {want_out} elements")
                ins[r] = a.data_ptr()
                outs[r] = b.data_ptr()
            self._last = (op, tuple(inputs), tuple(outputs),
                          [(t.data_ptr(), t.numel()) for t in inputs] + [(t.data_ptr(), t.numel()) for t in outputs])
        ins, outs = self._ptrs_in, self._ptrs_out
        proto = protocol if type(protocol) is int else int(as_protocol(protocol))
        e = 0 if epoch is None else int(epoch)
        rc = fn(self._ctx, ins, outs, count, 0, proto, e, _stream_handle(stream, self._device))
        if rc != 0:
            raise SfcError(rc, fn.__name__)

    def plan(self, inputs, outputs, op="allreduce", protocol="auto"):
        """A prepared single collective on fixed operands (sfc_plan_create):
        its launch() takes the next epoch and launches, nothing else."""
        n = self.nranks
        if len(inputs) != n or len(outputs) != n:
            raise ValueError(f"need {n} inputs and {n} outputs")
        o = as_op(op)
        count = inputs[0].numel()
        want_out = count if o == Op.ALLREDUCE else n * count
        for a, b in zip(inputs, outputs):
            _dev_ptr(a, "input")
            _dev_ptr(b, "output")
            if a.get_device() != self._device or b.get_device() != self._device:
                raise ValueError(f"operands must be on cuda:{self._device}, the communicator's device")
            if a.numel() != count or b.numel() != want_out:
                raise ValueError("operand sizes differ")
        ins = (C.c_void_p * n)(*[t.data_ptr() for t in inputs])
        outs = (C.c_void_p * n)(*[t.data_ptr() for t in outputs])
        h = C.c_void_p()
        _check(self._lib.sfc_plan_create(self._ctx, int(o), ins, outs, count, 0, int(as_protocol(protocol)),
                                         C.byref(h)), "sfc_plan_create")
        return Plan(self, h, (tuple(inputs), tuple(outputs)))

    def allreduce(self, inputs, outputs, protocol="auto", epoch=None, stream=None):
        """outputs[r] = rank-order fp32 sum of inputs, rounded once to bf16."""
        self._one(self._lib.sfc_allreduce, Op.ALLREDUCE, inputs, outputs, protocol, epoch, stream)

    def allgather(self, inputs, outputs, protocol="auto", epoch=None, stream=None):
        """outputs[r] = inputs[0] || ... || inputs[N-1]."""
        self._one(self._lib.sfc_allgather, Op.ALLGATHER, inputs, outputs, protocol, epoch, stream)

    def _device_tensor(self, t, dtypes, min_numel, exact, what):
        """Checks a tensor the kernel reads or writes directly: on this
        communicator's device (a host pointer would be dereferenced by the
        GPU), contiguous, of one of `dtypes`, with enough entries."""
        ok = (isinstance(t, torch.Tensor) and t.is_cuda and t.device.index == self._device and t.dtype in dtypes
              and t.is_contiguous() and (t.numel() == min_numel if exact else t.numel() >= min_numel))
        if not ok:
            raise ValueError(f"{what} must be a contiguous {'/'.join(str(d) for d in dtypes)} tensor on cuda:"
                             f"{self._device} with {'' if exact else 'at least '}{min_numel} entries")
        return C.c_void_p(t.data_ptr())

    def _timings_ptr(self, timings, k_ops):
        if timings is None:
            return None
        return self._device_tensor(timings, (torch.int64,), k_ops + 1, False, "timings")

    def _chain(self, fn, in_table, out_table, count, k_ops, protocol, epoch, skew_ns, timings, stream):
        n = self.nranks
        for name, t in (("in_table", in_table), ("out_table", out_table)):
            self._device_tensor(t, (torch.int64,), k_ops * n, True, name)
        skew_p = None
        if skew_ns is not None:
            skew_p = self._device_tensor(skew_ns, (torch.int32, torch.uint32), k_ops * n, True, "skew_ns")
        tim_p = self._timings_ptr(timings, k_ops)
        e = 0 if epoch is None else int(epoch)  # 0 = the next epoch
        _check(fn(self._ctx, int(k_ops), C.c_void_p(in_table.data_ptr()), C.c_void_p(out_table.data_ptr()),
                  int(count), 0, int(as_protocol(protocol)), e, skew_p, tim_p, _stream_handle(stream)),
               fn.__name__)

    def allreduce_chain(self, in_table, out_table, count, k_ops, protocol="auto", epoch=None, skew_ns=None,
                        timings=None, stream=None):
        """k_ops all-reduces in one persistent launch (pointer tables [k * N])."""
        self._chain(self._lib.sfc_allreduce_chain, in_table, out_table, count, k_ops, protocol, epoch, skew_ns,
                    timings, stream)

    def allgather_chain(self, in_table, out_table, count, k_ops, protocol="auto", epoch=None, skew_ns=None,
                        timings=None, stream=None):
        self._chain(self._lib.sfc_allgather_chain, in_table, out_table, count, k_ops, protocol, epoch, skew_ns,
                    timings, stream)

    def allreduce_chain_host(self, in_host, out_host, protocol="auto", epoch=None, timings=None, stream=None):
        """End to end from host memory: in_host / out_host are [k, N, count] bf16 CPU tensors."""
        for name, t in (("in_host", in_host), ("out_host", out_host)):
            if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous() or t.dim() != 3:
                raise ValueError(f"{name} must be a contiguous [k, N, count] bf16 CPU tensor")
        k, n, count = in_host.shape
        if n != self.nranks or tuple(out_host.shape) != (k, n, count):
            raise ValueError("shape mismatch")
        tim_p = self._timings_ptr(timings, k)
        e = 0 if epoch is None else int(epoch)  # 0 = the next epoch
        _check(self._lib.sfc_allreduce_chain_host(self._ctx, int(k), C.c_void_p(in_host.data_ptr()),
                                                  C.c_void_p(out_host.data_ptr()), int(count), 0,
                                                  int(as_protocol(protocol)), e, tim_p, _stream_handle(stream)),
               "sfc_allreduce_chain_host")

    def linear_allreduce(self, weights, xs, ys, epoch=None, stream=None):
        """Fused row-parallel linear + all-reduce for 1..8 decode tokens:
        ys[r] = sum over ranks of bf16(weights[q] @ xs[q]) (rank order, one
        rounding); weights[r] [hidden, kdim]; xs[r] [kdim] (one token) or
        [tokens, kdim]; ys[r] [hidden] or [tokens, hidden], matching xs."""
        n = self.nranks
        if not (len(weights) == len(xs) == len(ys) == n):
            raise ValueError(f"need {n} weights, inputs and outputs")
        hidden, kdim = weights[0].shape
        tokens = 1 if xs[0].dim() == 1 else int(xs[0].shape[0])
        for w, x_, y_ in zip(weights, xs, ys):
            if tuple(w.shape) != (hidden, kdim) or x_.numel() != tokens * kdim or y_.numel() != tokens * hidden:
                raise ValueError("shape mismatch")
        if any(t.get_device() != self._device for t in (*weights, *xs, *ys)):
            raise ValueError(f"operands must be on cuda:{self._device}, the communicator's device")
        W = (C.c_void_p * n)(*[_dev_ptr(w, "weight") for w in weights])
        X = (C.c_void_p * n)(*[_dev_ptr(t, "input") for t in xs])
        Y = (C.c_void_p * n)(*[_dev_ptr(t, "output") for t in ys])
        e = 0 if epoch is None else int(epoch)  # 0 = the next epoch
        _check(self._lib.sfc_linear_allreduce_tokens(self._ctx, W, X, Y, int(hidden), int(kdim), tokens, e,
                                                     _stream_handle(stream)), "sfc_linear_allreduce_tokens")

    def ll_view(self):
        v = _lib.LLView()
        _check(self._lib.sfc_get_ll_view(self._ctx, C.byref(v)), "sfc_get_ll_view")
        return v

    def reserve_epochs(self, k):
        first = C.c_uint32(0)
        _check(self._lib.sfc_reserve_epochs(self._ctx, int(k), C.byref(first)), "sfc_reserve_epochs")
        return int(first.value)

    # ------------------------------------------------------------- helpers
    def select_protocol(self, op, bytes_per_rank, nranks=None):
        n = self.nranks if nranks is None else int(nranks)
        return Protocol(self._lib.sfc_select_protocol(self._ctx, int(as_op(op)), int(bytes_per_rank), n))

    def set_cost_model(self, model):
        _check(self._lib.sfc_set_cost_model(self._ctx, C.byref(model)), "sfc_set_cost_model")

    def launch_shape(self, op, protocol, count):
        g, t = C.c_int(0), C.c_int(0)
        _check(self._lib.sfc_launch_shape(self._ctx, int(as_op(op)), int(as_protocol(protocol)), int(count),
                                          C.byref(g), C.byref(t)), "sfc_launch_shape")
        return g.value, t.value

    def scratch_slot(self, protocol, rank, parity, src):
        """(device pointer, bytes) of one receive slot, for inspection."""
        ptr, nb = C.c_void_p(), C.c_size_t()
        _check(self._lib.sfc_scratch_slot(self._ctx, int(as_protocol(protocol)), int(rank), int(parity),
                                          int(src), C.byref(ptr), C.byref(nb)), "sfc_scratch_slot")
        return ptr.value, nb.value

    def set_silent_rank(self, rank):
        _check(self._lib.sfc_set_silent_rank(self._ctx, int(rank)), "sfc_set_silent_rank")


def algorithmic_bytes(op, protocol, count, nranks):
    return float(_lib.load().sfc_algorithmic_bytes(int(as_op(op)), int(as_protocol(protocol)), int(count),
                                                   int(nranks)))


def default_cost_model():
    m = _lib.CostModel()
    _lib.load().sfc_default_cost_model(C.byref(m))
    return m


def cost_estimate(model, op, protocol, bytes_per_rank, nranks):
    return float(_lib.load().sfc_cost_estimate(C.byref(model), int(as_op(op)), int(as_protocol(protocol)),
                                               int(bytes_per_rank), int(nranks)))


def select_protocol_model(model, op, bytes_per_rank, nranks):
    return Protocol(_lib.load().sfc_select_protocol_model(C.byref(model), int(as_op(op)), int(bytes_per_rank),
                                                          int(nranks)))


class Plan:
    """A prepared collective of a Communicator (see Communicator.plan). It
    keeps its operand tensors alive; close() (or the communicator's close)
    releases it."""

    def __init__(self, comm, handle, keep):
        self._comm = comm
        self._h = handle
        self._keep = keep
        self._launch = comm._lib.sfc_plan_launch
        self._dev = comm._device
        comm._plans.append(self)

    def launch(self, stream=None):
        rc = self._launch(self._h, _stream_handle(stream, self._dev))
        if rc != 0:
            raise SfcError(rc, "sfc_plan_launch")

    def close(self):
        if self._h is not None and self._h.value:
            self._comm._lib.sfc_plan_destroy(self._h)
        self._h = None


def measure_floor(iters=500):
    """sfc_measure_floor as a dict (arrays as lists)."""
    r = _lib.FloorResult()
    _check(_lib.load().sfc_measure_floor(int(iters), C.byref(r)), "sfc_measure_floor")
    out = {}
    for f, _ in _lib.FloorResult._fields_:
        v = getattr(r, f)
        out[f] = list(v) if isinstance(v, C.Array) else v
    return out
