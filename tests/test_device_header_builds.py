"""The public device API compiles in a user's own translation unit (no GPU
needed: nvcc cross-compiles for sm_100a). A kernel that only includes
include/sfc_ll_device.cuh pushes its vectors and folds them with the
library's layout; this checks the header stands alone with nothing but
include/ on the path, for every rank count the library supports."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

USER_KERNEL = r"""
#include "sfc_ll_device.cuh"

template <int NR>
__global__ void user_allreduce(sfc_ll_view w, int rank, uint32_t epoch, const uint4* in, uint4* out,
                               uint64_t nvec) {
  const uint64_t v = blockIdx.x * blockDim.x + threadIdx.x;
  const bool active = v < nvec;
  const uint4 own = active ? in[v] : make_uint4(0, 0, 0, 0);
  if (active) sfc_device::ll_push(w, rank, epoch, v, own);
  uint4 y;
  if (sfc_device::ll_allreduce_lane<NR>(w, rank, epoch, v, active, own, &y) && active) out[v] = y;
}

template __global__ void user_allreduce<2>(sfc_ll_view, int, uint32_t, const uint4*, uint4*, uint64_t);
template __global__ void user_allreduce<3>(sfc_ll_view, int, uint32_t, const uint4*, uint4*, uint64_t);
template __global__ void user_allreduce<4>(sfc_ll_view, int, uint32_t, const uint4*, uint4*, uint64_t);
template __global__ void user_allreduce<8>(sfc_ll_view, int, uint32_t, const uint4*, uint4*, uint64_t);
"""


def test_ll_device_header_compiles_in_a_user_kernel(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    src = tmp_path / "user.cu"
    src.write_text(USER_KERNEL)
    r = subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O3",
                        "-I", os.path.join(ROOT, "include"), "-c", str(src), "-o", str(tmp_path / "user.o")],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
