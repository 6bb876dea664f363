// Latency floor microbenchmarks: the single-GPU analogue of the
// speed-of-light bound in "Why Microseconds Matter in AI Infrastructure",
// section "Defining the physical lower bound" (two L2 round trips plus one
// remote store, built on one 128-byte line).
//
//  * flag round trip: two CTAs on different SMs (each asks for more than half
//    of an SM's shared memory, so they cannot share one) ping-pong a 64-bit
//    flag with relaxed gpu-scope stores and polls; the initiator times each
//    round trip with clock64. Repeated for 16 responder SMs spread over the
//    GPU (both dies), so the median covers near and far pairs.
//  * L2 round trip: one thread chases a pointer chain through a small buffer
//    with L1-bypassing loads, so every load is one L2 hit.
// Every wait is bounded by a %globaltimer deadline.
#include <cuda_runtime.h>

#include <algorithm>
#include <vector>

#include "sfc.h"
#include "sfc_device.cuh"

namespace sfc {
namespace {

constexpr uint64_t kFloorTimeoutNs = 200ull * 1000 * 1000;  // 200 ms per trial
constexpr int kFloorSmem = 160 * 1024;

// Grid of one CTA per SM (each asks for more than half of an SM's shared
// memory). CTA 0 is the initiator, CTA `responder` answers, all others exit.
__global__ void flag_pingpong(uint64_t* flags, int iters, int responder, uint64_t* cycles, uint64_t* cal,
                              int* sms, int* err) {
  extern __shared__ uint8_t keep_apart[];
  if (threadIdx.x != 0) return;
  if (blockIdx.x != 0 && blockIdx.x != static_cast<unsigned>(responder)) return;
  keep_apart[0] = 0;
  uint64_t* a = flags;       // initiator -> responder
  uint64_t* b = flags + 32;  // responder -> initiator (another 256-byte block)
  sms[blockIdx.x == 0 ? 0 : 1] = static_cast<int>(smid());
  const uint64_t deadline = gtimer() + kFloorTimeoutNs;
  if (blockIdx.x == 0) {
    const uint64_t g0 = gtimer();
    const uint64_t c0 = clock64();
    for (int i = 1; i <= iters; ++i) {
      const uint64_t t0 = clock64();
      st_rlx_u64(a, static_cast<uint64_t>(i));
      uint32_t spins = 0;
      while (ld_rlx_u64(b) != static_cast<uint64_t>(i)) {
        if ((++spins & 255u) == 0 && gtimer() > deadline) {
          *err = 1;
          st_rlx_u64(a, ~0ull);  // release the responder
          return;
        }
      }
      cycles[i - 1] = clock64() - t0;
    }
    cal[0] = gtimer() - g0;
    cal[1] = clock64() - c0;
  } else {
    for (int i = 1; i <= iters; ++i) {
      uint32_t spins = 0;
      uint64_t v;
      while ((v = ld_rlx_u64(a)) != static_cast<uint64_t>(i)) {
        if (v == ~0ull) return;
        if ((++spins & 255u) == 0 && gtimer() > deadline) {
          *err = 1;
          return;
        }
      }
      st_rlx_u64(b, static_cast<uint64_t>(i));
    }
  }
}

__device__ __forceinline__ uint64_t ld_cg_u64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.global.cg.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// chain[i] holds the index of the next element; `steps` dependent loads.
__global__ void l2_chase(const uint64_t* chain, int n, int steps, uint64_t* out) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  uint64_t j = 0;
  for (int i = 0; i < n; ++i) j = ld_cg_u64(chain + j);  // warm: bring the chain into L2
  const uint64_t c0 = clock64();
  const uint64_t g0 = gtimer();
  for (int i = 0; i < steps; ++i) j = ld_cg_u64(chain + j);
  const uint64_t c1 = clock64();
  const uint64_t g1 = gtimer();
  out[0] = c1 - c0;
  out[1] = g1 - g0;
  out[2] = j;  // keep the chain live
}

__global__ void timer_step(uint64_t* out) {
  if (threadIdx.x != 0) return;
  uint64_t best = ~0ull;
  uint64_t prev = gtimer();
  for (int i = 0; i < 200000; ++i) {
    const uint64_t t = gtimer();
    if (t != prev) {
      best = min(best, t - prev);
      prev = t;
    }
  }
  out[0] = best;
}

double pct(std::vector<uint64_t> v, double q) {
  if (v.empty()) return 0.0;
  std::sort(v.begin(), v.end());
  size_t i = static_cast<size_t>(q * (v.size() - 1) + 0.5);
  return static_cast<double>(v[std::min(i, v.size() - 1)]);
}

}  // namespace
}  // namespace sfc

extern "C" sfc_status sfc_measure_floor(int iters, sfc_floor_result* out) {
  using namespace sfc;
  if (out == nullptr || iters < 16 || iters > (1 << 20)) return SFC_ERR_INVALID;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return SFC_ERR_CUDA;
  }
  int sm_count = 0;
  if (cudaDeviceGetAttribute(&sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sm_count < 2) {
    (void)cudaGetLastError();
    return SFC_ERR_CUDA;
  }
  // responders spread over the grid: pairs on the same and on different dies
  const int trials = std::min(16, sm_count - 1);
  const int chain_n = 4096;  // 32 KB pointer chain: L2 resident
  uint64_t* dflags = nullptr;
  uint64_t* dcycles = nullptr;
  uint64_t* dcal = nullptr;
  int* dsms = nullptr;
  int* derr = nullptr;
  uint64_t* dchain = nullptr;
  uint64_t* dout = nullptr;
  sfc_status st = SFC_OK;
  std::vector<uint64_t> rtts;
  std::vector<double> pair_p50;
  std::vector<uint64_t> hcal(2 * trials);
  int hsms[2] = {0, 0};
  int herr = 0;
  uint64_t chase[3] = {0, 0, 0};
  uint64_t step = 0;
  auto ok = [](cudaError_t e) {
    if (e != cudaSuccess) {
      (void)cudaGetLastError();
      return false;
    }
    return true;
  };
  do {
    if (!ok(cudaMalloc(&dflags, 64 * sizeof(uint64_t))) || !ok(cudaMalloc(&dcycles, sizeof(uint64_t) * iters)) ||
        !ok(cudaMalloc(&dcal, 2 * sizeof(uint64_t))) || !ok(cudaMalloc(&dsms, 2 * sizeof(int))) ||
        !ok(cudaMalloc(&derr, sizeof(int))) || !ok(cudaMalloc(&dchain, chain_n * sizeof(uint64_t))) ||
        !ok(cudaMalloc(&dout, 4 * sizeof(uint64_t)))) {
      st = SFC_ERR_CUDA;
      break;
    }
    if (!ok(cudaFuncSetAttribute(reinterpret_cast<const void*>(&flag_pingpong),
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kFloorSmem))) {
      st = SFC_ERR_CUDA;
      break;
    }
    std::vector<uint64_t> hcycles(iters);
    for (int t = 0; t < trials && st == SFC_OK; ++t) {
      int responder = 1 + static_cast<int>((static_cast<int64_t>(t) * (sm_count - 1)) / trials);
      if (responder >= sm_count) responder = sm_count - 1;
      if (!ok(cudaMemset(dflags, 0, 64 * sizeof(uint64_t))) || !ok(cudaMemset(derr, 0, sizeof(int)))) {
        st = SFC_ERR_CUDA;
        break;
      }
      void* args[] = {&dflags, &iters, &responder, &dcycles, &dcal, &dsms, &derr};
      if (!ok(cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(&flag_pingpong), dim3(sm_count), dim3(32),
                                          args, kFloorSmem, nullptr)) ||
          !ok(cudaDeviceSynchronize())) {
        st = SFC_ERR_CUDA;
        break;
      }
      if (!ok(cudaMemcpy(&herr, derr, sizeof(int), cudaMemcpyDeviceToHost)) ||
          !ok(cudaMemcpy(hcycles.data(), dcycles, sizeof(uint64_t) * iters, cudaMemcpyDeviceToHost)) ||
          !ok(cudaMemcpy(&hcal[2 * t], dcal, 2 * sizeof(uint64_t), cudaMemcpyDeviceToHost)) ||
          !ok(cudaMemcpy(hsms, dsms, 2 * sizeof(int), cudaMemcpyDeviceToHost))) {
        st = SFC_ERR_CUDA;
        break;
      }
      if (herr) {
        st = SFC_ERR_TIMEOUT;
        break;
      }
      // the first iterations warm the lines; keep the rest
      std::vector<uint64_t> kept(hcycles.begin() + std::min(iters / 8, 64), hcycles.end());
      pair_p50.push_back(pct(kept, 0.5));
      rtts.insert(rtts.end(), kept.begin(), kept.end());
    }
    if (st != SFC_OK) break;
    std::vector<uint64_t> hchain(chain_n);
    for (int i = 0; i < chain_n; ++i) hchain[i] = static_cast<uint64_t>((i + 97 * 16 + 1) % chain_n);
    if (!ok(cudaMemcpy(dchain, hchain.data(), chain_n * sizeof(uint64_t), cudaMemcpyHostToDevice))) {
      st = SFC_ERR_CUDA;
      break;
    }
    const int steps = 4096;
    l2_chase<<<1, 32>>>(dchain, chain_n, steps, dout);
    timer_step<<<1, 32>>>(dout + 3);
    if (!ok(cudaDeviceSynchronize()) || !ok(cudaMemcpy(chase, dout, 3 * sizeof(uint64_t), cudaMemcpyDeviceToHost)) ||
        !ok(cudaMemcpy(&step, dout + 3, sizeof(uint64_t), cudaMemcpyDeviceToHost))) {
      st = SFC_ERR_CUDA;
      break;
    }
    uint64_t cyc = 0, ns = 0;
    for (int t = 0; t < trials; ++t) {
      ns += hcal[2 * t];
      cyc += hcal[2 * t + 1];
    }
    const double ghz = ns ? static_cast<double>(cyc) / static_cast<double>(ns) : 1.0;
    out->sm_clock_ghz = ghz;
    out->flag_rtt_ns_p50 = pct(rtts, 0.50) / ghz;
    out->flag_rtt_ns_p99 = pct(rtts, 0.99) / ghz;
    out->flag_rtt_ns_min_pair = *std::min_element(pair_p50.begin(), pair_p50.end()) / ghz;
    out->flag_rtt_ns_max_pair = *std::max_element(pair_p50.begin(), pair_p50.end()) / ghz;
    out->pairs = static_cast<int>(pair_p50.size());
    out->l2_rtt_ns_p50 = static_cast<double>(chase[0]) / steps / ghz;
    out->globaltimer_step_ns = static_cast<double>(step);
    out->sm_a = hsms[0];
    out->sm_b = hsms[1];
  } while (false);
  cudaFree(dflags);
  cudaFree(dcycles);
  cudaFree(dcal);
  cudaFree(dsms);
  cudaFree(derr);
  cudaFree(dchain);
  cudaFree(dout);
  return st;
}
