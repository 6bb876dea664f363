"""Helpers for the GPU parity tests: device buffers, pointer tables, readback."""
import numpy as np
import torch

from latency_self_synchronizing_b200 import api


def round8(n):
    return (n + 7) // 8 * 8


class Operands:
    """[K, N] operands of `count` elements each in one padded device buffer
    (row stride rounded to 8 elements so every operand is 16-byte aligned)."""

    def __init__(self, k, n, count, fill=None, device="cuda"):
        self.k, self.n, self.count = k, n, count
        self.stride = max(8, round8(count))
        self.buf = torch.zeros(k * n * self.stride, dtype=torch.int16, device=device)
        if fill is not None:
            host = np.zeros((k, n, self.stride), dtype=np.uint16)
            host[:, :, :count] = fill
            self.buf.copy_(torch.from_numpy(host.reshape(-1).view(np.int16)))
        base = self.buf.data_ptr()
        ptrs = [base + 2 * self.stride * (kk * n + r) for kk in range(k) for r in range(n)]
        self.table = torch.tensor(ptrs, dtype=torch.int64, device=device)
        self.ptrs = ptrs

    def bits(self):
        h = self.buf.cpu().numpy().view(np.uint16).reshape(self.k, self.n, self.stride)
        return h[:, :, : self.count].copy()

    def tensors(self, kk):
        """bf16 views of operation kk's N operands (for the one-op API)."""
        flat = self.buf.view(torch.bfloat16)
        return [flat[(kk * self.n + r) * self.stride:(kk * self.n + r) * self.stride + self.count]
                for r in range(self.n)]


def run_chain(comm, proto, x, op="allreduce", skew=None, timings=None):
    """Run one chain over inputs x [K, N, count] (uint16); return outputs."""
    k, n, count = x.shape
    ins = Operands(k, n, count, fill=x)
    out_count = count if op == "allreduce" else n * count
    outs = Operands(k, n, out_count)
    fn = comm.allreduce_chain if op == "allreduce" else comm.allgather_chain
    fn(ins.table, outs.table, count, k, protocol=proto, skew_ns=skew, timings=timings)
    torch.cuda.synchronize()
    st, info = comm.status()
    assert st == api.Status.OK, (st, hex(info))
    return outs.bits()


class _RawDevice:
    """A device byte range exposed through __cuda_array_interface__."""

    def __init__(self, ptr, nbytes):
        self.__cuda_array_interface__ = {"shape": (nbytes,), "typestr": "|u1", "data": (ptr, False),
                                         "version": 3}


def slot_bytes(comm, proto, rank, parity, src):
    """Host copy of one receive slot of the context's scratch."""
    ptr, nbytes = comm.scratch_slot(proto, rank, parity, src)
    torch.cuda.synchronize()
    return torch.as_tensor(_RawDevice(ptr, nbytes), device="cuda").cpu().numpy().copy()
