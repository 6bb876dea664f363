// sfc_allreduce_noalloc: one LL all-reduce whose scratch lives in a
// file-scope device array instead of memory from cudaMalloc, and
// sfc_noalloc_status, which reads the device status that array holds.
//
// Some callers cannot allocate device memory at the point where they need an
// all-reduce: code running inside a custom allocator or an out-of-memory
// handler, code that must not grow its footprint after start-up (a serving
// process that reserves all of HBM up front), or a host library that is not
// allowed to own allocations. This entry point serves them: the caller passes
// inputs and outputs, and everything else comes from a static array that every
// GPU loading this library holds until the process exits.
#include <cuda_runtime.h>

#include <cstdlib>
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
constexpr uint64_t kDefaultTimeoutNs = 50ull * 1000 * 1000;

// The scratch: LL slots, then the status block. In host code this name is a
// host-side stand-in, not a device address: the device address is obtained
// with cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocBytes];

// What the first call on a device looks up once, with that device current.
struct DeviceSetup {
  bool ready = false;
  uint8_t* base = nullptr;                     // device address of g_noalloc_scratch
  int occ_by_ranks[sfc::kMaxRanks + 1] = {};  // LL all-reduce CTAs per SM, per rank count
  int sms = 0;
};

DeviceSetup g_setup[kMaxDevices];
std::mutex g_mu;

// Read once per process: the wait bound (SFC_TIMEOUT_MS, as for contexts)
// and a rank that pushes nothing (SFC_NOALLOC_SILENT_RANK, for failure tests:
// its peers' waits run out and the status records the timeout).
uint64_t g_timeout_ns = 0;
int g_silent_rank = -2;  // -2 = not read yet

void read_environment() {
  if (g_silent_rank != -2) return;
  g_timeout_ns = kDefaultTimeoutNs;
  if (const char* t = std::getenv("SFC_TIMEOUT_MS")) {
    char* end = nullptr;
    const long ms = std::strtol(t, &end, 10);
    if (end != t && *end == '\0' && ms > 0 && ms <= 4000000) g_timeout_ns = static_cast<uint64_t>(ms) * 1000000ull;
  }
  g_silent_rank = -1;
  if (const char* s = std::getenv("SFC_NOALLOC_SILENT_RANK")) {
    char* end = nullptr;
    const long r = std::strtol(s, &end, 10);
    if (end != s && *end == '\0' && r >= 0 && r < sfc::kMaxRanks) g_silent_rank = static_cast<int>(r);
  }
}

// Per-device set-up on the current device: the array's device address (the
// lookup may load this library's device code and place the array in device
// memory), the SM count and the LL kernels' occupancy for every rank count.
sfc_status device_setup(const DeviceSetup** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    (void)cudaGetLastError();
    return SFC_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  read_environment();
  DeviceSetup& s = g_setup[dev];
  if (!s.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      return SFC_ERR_CUDA;
    }
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) {
      (void)cudaGetLastError();
      return SFC_ERR_CUDA;
    }
    for (int n = sfc::kMinRanks; n <= sfc::kMaxRanks; ++n) {
      const void* fn = sfc::kernel_for(n, sfc::kLL, sfc::kAllreduce);
      int occ = 0;
      if (fn == nullptr || cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, sfc::kThreads, 0) != cudaSuccess) {
        (void)cudaGetLastError();
        return SFC_ERR_CUDA;
      }
      s.occ_by_ranks[n] = occ;
    }
    s.base = static_cast<uint8_t*>(p);
    s.sms = sms;
    s.ready = true;
  }
  *out = &s;
  return SFC_OK;
}

}  // namespace

extern "C" sfc_status sfc_allreduce_noalloc(const void* const* in, void* const* out, int nranks, size_t count,
                                            void* stream) {
  using namespace sfc;
  if (count > SFC_NOALLOC_MAX_COUNT) return SFC_ERR_INVALID;
  const DeviceSetup* dv = nullptr;
  sfc_status s = device_setup(&dv);
  if (s != SFC_OK) return s;
  if (count == 0) return SFC_OK;  // set-up only
  if (in == nullptr || out == nullptr || nranks < kMinRanks || nranks > kMaxRanks) return SFC_ERR_INVALID;
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

  const uint64_t nvec = (count + 7) / 8;
  const int gmax = dv->occ_by_ranks[nranks] * dv->sms / nranks;
  int G = static_cast<int>((nvec + kThreads - 1) / kThreads);
  if (G > gmax) G = gmax;
  if (G < 1) return SFC_ERR_RESOURCES;

  // Every call starts the LL slots from a clean slate (the previous call used
  // epoch 1 as well), cleared on the stream first. The status block is not
  // cleared: an error stays recorded, and every later call exits at once,
  // until sfc_noalloc_status has read it.
  const uint64_t slot = slot_bytes_gpu(kLL, count, nranks);
  const uint64_t used = 2ull * nranks * (nranks - 1) * slot;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* base = dv->base;
  if (cudaMemsetAsync(base, 0, used, st) != cudaSuccess) {
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
  p.status = reinterpret_cast<DevStatus*>(base + kNoAllocSlots * kNoAllocSlotBytes);
  p.timeout_ns = g_timeout_ns;
  p.silent_rank = g_silent_rank < nranks ? g_silent_rank : -1;
  void* args[] = {&p};
  const cudaError_t e =
      cudaLaunchCooperativeKernel(kernel_for(nranks, kLL, kAllreduce), dim3(nranks * G), dim3(kThreads), args, 0, st);
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

extern "C" sfc_status sfc_noalloc_status(void* stream, uint32_t* info) {
  using namespace sfc;
  const DeviceSetup* dv = nullptr;
  sfc_status s = device_setup(&dv);
  if (s != SFC_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* status = dv->base + kNoAllocSlots * kNoAllocSlotBytes;
  DevStatus h{};
  // ordered after every earlier call on the stream; the host waits for it
  if (cudaMemcpyAsync(&h, status, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess) {
    (void)cudaGetLastError();
    return SFC_ERR_CUDA;
  }
  if (h.code != 0 || h.abort != 0) {
    if (cudaMemsetAsync(status, 0, sizeof(DevStatus), st) != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess) {
      (void)cudaGetLastError();
      return SFC_ERR_CUDA;
    }
  }
  if (info != nullptr) *info = h.info;
  if (h.code != 0) return static_cast<sfc_status>(h.code);
  return h.abort != 0 ? SFC_ERR_ABORTED : SFC_OK;
}
