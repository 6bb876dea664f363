"""The public device API run from a user's own kernel.

A kernel built from a separate translation unit that includes only
include/sfc_ll_device.cuh ("Why Microseconds Matter in AI Infrastructure",
section "Communication is becoming part of GPU execution": low-latency send,
receive and reduce called from inside kernels) pushes its vectors with
ll_push and folds them with ll_allreduce_lane over a chain of epochs reserved
from a library context. Every output must equal the oracle's closed form bit
for bit, and the library's own calls must continue the epoch sequence
afterwards on the same scratch.
"""
import ctypes as C
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

from latency_self_synchronizing_b200 import api
from latency_self_synchronizing_b200.inputs import make_inputs
from oracle import reference
from _gpu_helpers import Operands

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

USER_SOURCE = r"""
#include <cuda_runtime.h>
#include "sfc_ll_device.cuh"

// 8 bf16 of row `x` from element 8 v; past `count` reads as +0
__device__ uint4 load_vec(const uint16_t* x, uint64_t v, uint64_t count) {
  if (8 * v + 8 <= count) return *reinterpret_cast<const uint4*>(x + 8 * v);
  uint32_t w[4] = {0u, 0u, 0u, 0u};
  for (int i = 0; i < 8; ++i)
    if (8 * v + i < count) w[i >> 1] |= static_cast<uint32_t>(x[8 * v + i]) << (16 * (i & 1));
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ void store_vec(uint16_t* y, uint64_t v, uint64_t count, uint4 val) {
  const uint32_t w[4] = {val.x, val.y, val.z, val.w};
  for (int i = 0; i < 8; ++i)
    if (8 * v + i < count) y[8 * v + i] = static_cast<uint16_t>(w[i >> 1] >> (16 * (i & 1)));
}

// rank = blockIdx.x / G; every rank's thread t of CTA k owns vectors
// k * blockDim + t + j * G * blockDim (the same every epoch)
template <int NR>
__global__ void user_chain(sfc_ll_view w, uint32_t first, int k_ops, const uint16_t* const* in,
                           uint16_t* const* out, uint64_t count, int G) {
  const int rank = blockIdx.x / G, k = blockIdx.x % G;
  const uint64_t nvec = (count + 7) / 8, stride = static_cast<uint64_t>(G) * blockDim.x;
  for (int op = 0; op < k_ops; ++op) {
    const uint32_t e = first + static_cast<uint32_t>(op);
    const uint16_t* x = in[op * NR + rank];
    uint16_t* y = out[op * NR + rank];
    for (uint64_t vb = static_cast<uint64_t>(k) * blockDim.x; vb < nvec; vb += stride) {
      const uint64_t v = vb + threadIdx.x;
      if (v < nvec) sfc_device::ll_push(w, rank, e, v, load_vec(x, v, count));
    }
    for (uint64_t vb = static_cast<uint64_t>(k) * blockDim.x; vb < nvec; vb += stride) {
      const uint64_t v = vb + threadIdx.x;
      const bool active = v < nvec;
      const uint4 own = active ? load_vec(x, v, count) : make_uint4(0u, 0u, 0u, 0u);
      uint4 r;
      if (!sfc_device::ll_allreduce_lane<NR>(w, rank, e, v, active, own, &r)) return;
      if (active) store_vec(y, v, count, r);
    }
  }
}

extern "C" int user_ll_chain(void* scratch, uint64_t slot_stride, int nranks, void* status, uint64_t timeout_ns,
                             uint32_t first, int k_ops, const void* in_table, const void* out_table, uint64_t count,
                             int G, int threads, void* stream) {
  sfc_ll_view w;
  w.scratch = static_cast<unsigned char*>(scratch);
  w.slot_stride = slot_stride;
  w.nranks = nranks;
  w.status = static_cast<int*>(status);
  w.timeout_ns = timeout_ns;
  const uint16_t* const* in = static_cast<const uint16_t* const*>(in_table);
  uint16_t* const* out = static_cast<uint16_t* const*>(const_cast<void*>(out_table));
  void* args[] = {&w, &first, &k_ops, &in, &out, &count, &G};
  const void* fn = nullptr;
  switch (nranks) {
    case 2: fn = reinterpret_cast<const void*>(&user_chain<2>); break;
    case 3: fn = reinterpret_cast<const void*>(&user_chain<3>); break;
    case 4: fn = reinterpret_cast<const void*>(&user_chain<4>); break;
    case 5: fn = reinterpret_cast<const void*>(&user_chain<5>); break;
    case 6: fn = reinterpret_cast<const void*>(&user_chain<6>); break;
    case 7: fn = reinterpret_cast<const void*>(&user_chain<7>); break;
    case 8: fn = reinterpret_cast<const void*>(&user_chain<8>); break;
    default: return -1;
  }
  // every rank waits on the others: all CTAs must be co-resident
  return static_cast<int>(cudaLaunchCooperativeKernel(fn, dim3(nranks * G), dim3(threads), args, 0,
                                                      static_cast<cudaStream_t>(stream)));
}
"""


@pytest.fixture(scope="module")
def user_lib(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.fail("nvcc is needed to build the user kernel")
    d = tmp_path_factory.mktemp("user_kernel")
    src = d / "user.cu"
    src.write_text(USER_SOURCE)
    so = d / "libuser.so"
    r = subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O3", "-shared",
                        "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(so)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    lib = C.CDLL(str(so))
    lib.user_ll_chain.restype = C.c_int
    lib.user_ll_chain.argtypes = [C.c_void_p, C.c_uint64, C.c_int, C.c_void_p, C.c_uint64, C.c_uint32, C.c_int,
                                  C.c_void_p, C.c_void_p, C.c_uint64, C.c_int, C.c_int, C.c_void_p]
    return lib


def _run_user_chain(lib, comm, x, G, threads):
    k, n, count = x.shape
    ins, outs = Operands(k, n, count, fill=x), Operands(k, n, count)
    view = comm.ll_view()
    first = comm.reserve_epochs(k)
    stream = torch.cuda.current_stream().cuda_stream
    rc = lib.user_ll_chain(view.scratch, view.slot_stride, view.nranks, view.status, view.timeout_ns, first, k,
                           ins.table.data_ptr(), outs.table.data_ptr(), count, G, threads, stream)
    assert rc == 0, f"cudaLaunchCooperativeKernel returned {rc}"
    torch.cuda.synchronize()
    st, info = comm.status()
    assert st == api.Status.OK, (st, hex(info))
    return outs.bits()


@pytest.mark.parametrize("n", [2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("count,G,threads", [(1, 1, 32), (1000, 1, 64), (4093, 2, 128), (20000, 3, 256)])
def test_user_kernel_chain_bit_exact(user_lib, n, count, G, threads):
    k = 6
    x = make_inputs(seed=700 + 10 * n + count % 97, k_ops=k, nranks=n, count=count)
    comm = api.Communicator(n, 2 * max(count, 8), protocols=["ll"])
    try:
        got = _run_user_chain(user_lib, comm, x, G, threads)
        for kk in range(k):
            want = reference.allreduce(x[kk])
            for r in range(n):
                np.testing.assert_array_equal(got[kk, r], want, err_msg=f"op {kk} rank {r}")
        # the library's own LL calls continue the sequence on the same slots
        y = make_inputs(seed=900 + n, k_ops=3, nranks=n, count=count)
        ins, outs = Operands(3, n, count, fill=y), Operands(3, n, count)
        comm.allreduce_chain(ins.table, outs.table, count, 3, protocol="ll")
        torch.cuda.synchronize()
        assert comm.status()[0] == api.Status.OK
        back = outs.bits()
        for kk in range(3):
            for r in range(n):
                np.testing.assert_array_equal(back[kk, r], reference.allreduce(y[kk]))
        # and the user kernel again, after the library's calls
        got = _run_user_chain(user_lib, comm, x[:2], G, threads)
        for kk in range(2):
            for r in range(n):
                np.testing.assert_array_equal(got[kk, r], reference.allreduce(x[kk]))
    finally:
        comm.close()
