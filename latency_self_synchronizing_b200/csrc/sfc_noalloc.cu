// sfc_allreduce_noalloc: one LL all-reduce whose scratch lives in a
// file-scope device array instead of memory from cudaMalloc.
//
// Some callers cannot allocate device memory at the point where they need an
// all-reduce: code running inside a custom allocator or an out-of-memory
// handler, code that must not grow its footprint after start-up (a serving
// process that reserves all of HBM up front), or a host library that is not
// allowed to own allocations. This entry point serves them: the caller passes
// inputs and outputs, and everything else comes from a static array that every
// GPU loading this library holds until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "sfc.h"
#include "sfc_internal.h"

namespace {

constexpr int kMaxDevices = 64;
// Largest message: 4096 bf16 elements (8 KB) per rank, up to 8 ranks. The LL
// receive slots of both parities for 8 ranks need 2 * 8 * 7 slots of
// slot_bytes_gpu(LL, 4096, n) = 16 KB each.
constexpr uint64_t kNoAllocSlotBytes = 16384;
constexpr uint64_t kNoAllocSlots = 2ull * sfc::kMaxRanks * (sfc::kMaxRanks - 1);
constexpr uint64_t kNoAllocStatusBytes = 256;
constexpr uint64_t kNoAllocBytes = kNoAllocSlots * kNoAllocSlotBytes + kNoAllocStatusBytes;

// The scratch. In host code this name is a host-side stand-in, not a device
// address: the device address is obtained with cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocBytes];

void* g_addr[kMaxDevices] = {};
std::mutex g_mu;

// Per-device set-up: the symbol's device address on the current device.
sfc_status scratch_address(int dev, uint8_t** out) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      return SFC_ERR_CUDA;
    }
    g_addr[dev] = p;
  }
  *out = static_cast<uint8_t*>(g_addr[dev]);
  return SFC_OK;
}

}  // namespace

extern "C" sfc_status sfc_allreduce_noalloc(const void* const* in, void* const* out, int nranks, size_t count,
                                            void* stream) {
  using namespace sfc;
  if (in == nullptr || out == nullptr || nranks < kMinRanks || nranks > kMaxRanks) return SFC_ERR_INVALID;
  if (count > SFC_NOALLOC_MAX_COUNT) return SFC_ERR_INVALID;
  if (count == 0) return SFC_OK;
  const size_t bytes = count * 2;
  for (int r = 0; r < nranks; ++r) {
    if (in[r] == nullptr || out[r] == nullptr) return SFC_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(in[r]) | reinterpret_cast<uintptr_t>(out[r])) & 15u) return SFC_ERR_INVALID;
  }
  for (int a = 0; a < nranks; ++a)
    for (int b = 0; b < nranks; ++b) {
      const uintptr_t x = reinterpret_cast<uintptr_t>(in[a]), y = reinterpret_cast<uintptr_t>(out[b]);
      if (x < y + bytes && y < x + bytes) return SFC_ERR_INVALID;
      const uintptr_t z = reinterpret_cast<uintptr_t>(out[a]);
      if (a < b && z < y + bytes && y < z + bytes) return SFC_ERR_INVALID;
    }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    (void)cudaGetLastError();
    return SFC_ERR_CUDA;
  }
  uint8_t* base = nullptr;
  sfc_status s = scratch_address(dev, &base);
  if (s != SFC_OK) return s;

  const void* fn = kernel_for(nranks, kLL, kAllreduce);
  int occ = 0, sms = 0;
  if (fn == nullptr || cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, kThreads, 0) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return SFC_ERR_CUDA;
  }
  const uint64_t nvec = (count + 7) / 8;
  const int gmax = occ * sms / nranks;
  int G = static_cast<int>((nvec + kThreads - 1) / kThreads);
  if (G > gmax) G = gmax;
  if (G < 1) return SFC_ERR_RESOURCES;

  // Every call starts from a clean slate: LL flags of the previous call
  // (epoch 1 as well) and the status word are cleared on the stream first.
  const uint64_t slot = slot_bytes_gpu(kLL, count, nranks);
  const uint64_t used = 2ull * nranks * (nranks - 1) * slot;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* status = base + kNoAllocSlots * kNoAllocSlotBytes;
  if (cudaMemsetAsync(base, 0, used, st) != cudaSuccess ||
      cudaMemsetAsync(status, 0, kNoAllocStatusBytes, st) != cudaSuccess) {
    (void)cudaGetLastError();
    return SFC_ERR_CUDA;
  }
  KParams p{};
  for (int r = 0; r < nranks; ++r) {
    p.in_inline[r] = static_cast<const uint16_t*>(in[r]);
    p.out_inline[r] = static_cast<uint16_t*>(out[r]);
  }
  p.addr_mode = 0;
  p.count = count;
  p.k_ops = 1;
  p.G = G;
  p.first_epoch = 1;
  p.scratch = base;
  p.slot_stride = slot;
  p.scratch_bytes = used;
  p.status = reinterpret_cast<DevStatus*>(status);
  p.timeout_ns = 50ull * 1000 * 1000;
  p.silent_rank = -1;
  void* args[] = {&p};
  const cudaError_t e = cudaLaunchCooperativeKernel(fn, dim3(nranks * G), dim3(kThreads), args, 0, st);
  if (e == cudaErrorCooperativeLaunchTooLarge) {
    (void)cudaGetLastError();
    return SFC_ERR_RESOURCES;
  }
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return SFC_ERR_CUDA;
  }
  return SFC_OK;
}
