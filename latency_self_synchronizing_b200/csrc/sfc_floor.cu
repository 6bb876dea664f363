// Latency floor microbenchmarks: the single-GPU analogue of the
// speed-of-light bound in "Why Microseconds Matter in AI Infrastructure",
// section "Defining the physical lower bound" (two L2 round trips plus one
// remote store, built on one 128-byte line).
//
//  * flag round trip: a launch of one CTA per SM (each asks for more than
//    half of an SM's shared memory, so no SM holds two); the CTA on SM a
//    (by %smid) stores a 64-bit flag with a relaxed gpu-scope store, the CTA
//    on SM b polls it and answers on a second flag, and a times each round
//    trip with clock64. Every other CTA exits. The SM set is fixed by %smid
//    (8 initiators and 8 responders spread evenly over the sorted ids, every
//    initiator with every responder) and each pair is measured at 8 flag
//    addresses: on B200 the L2 home of the flag moves one pair's round trip
//    by up to 0.6 us, more than the choice of SMs does, so the floor is the
//    median over all (pair, address) trials.
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
constexpr size_t kFlagArena = 32ull << 20;  // flag addresses spread over 32 MB

// Each CTA records its SM id: the set of ids the measuring launches can use.
__global__ void list_sms(int* ids) {
  extern __shared__ uint8_t keep_apart[];
  if (threadIdx.x != 0) return;
  keep_apart[0] = 0;
  ids[blockIdx.x] = static_cast<int>(smid());
}

// One CTA per SM. The CTA on SM `sa` initiates, the one on SM `sb` answers,
// all others exit. a: initiator -> responder flag, b: the answer.
__global__ void flag_pingpong(uint64_t* a, uint64_t* b, int iters, int sa, int sb, uint64_t* cycles, uint64_t* cal,
                              int* err) {
  extern __shared__ uint8_t keep_apart[];
  if (threadIdx.x != 0) return;
  const int me = static_cast<int>(smid());
  if (me != sa && me != sb) return;
  keep_apart[0] = 0;
  const uint64_t deadline = gtimer() + kFloorTimeoutNs;
  if (me == sa) {
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

double pctd(std::vector<double> v, double q) {
  if (v.empty()) return 0.0;
  std::sort(v.begin(), v.end());
  size_t i = static_cast<size_t>(q * (v.size() - 1) + 0.5);
  return v[std::min(i, v.size() - 1)];
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
  if (cudaDeviceGetAttribute(&sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      sm_count < 2 * SFC_FLOOR_SMS) {
    (void)cudaGetLastError();
    return SFC_ERR_CUDA;
  }
  const int chain_n = 4096;  // 32 KB pointer chain: L2 resident
  uint8_t* darena = nullptr;
  uint64_t* dcycles = nullptr;
  uint64_t* dcal = nullptr;
  int* dids = nullptr;
  int* derr = nullptr;
  uint64_t* dchain = nullptr;
  uint64_t* dout = nullptr;
  sfc_status st = SFC_OK;
  std::vector<double> trial_p50;  // one per (pair, location), cycles
  std::vector<std::vector<double>> by_loc(SFC_FLOOR_LOCATIONS);
  uint64_t cal_ns = 0, cal_cyc = 0;
  uint64_t chase[3] = {0, 0, 0};
  uint64_t step = 0;
  int sel[2 * SFC_FLOOR_SMS] = {};
  auto ok = [](cudaError_t e) {
    if (e != cudaSuccess) {
      (void)cudaGetLastError();
      return false;
    }
    return true;
  };
  do {
    if (!ok(cudaMalloc(&darena, kFlagArena)) || !ok(cudaMalloc(&dcycles, sizeof(uint64_t) * iters)) ||
        !ok(cudaMalloc(&dcal, 2 * sizeof(uint64_t))) || !ok(cudaMalloc(&dids, sizeof(int) * sm_count)) ||
        !ok(cudaMalloc(&derr, sizeof(int))) || !ok(cudaMalloc(&dchain, chain_n * sizeof(uint64_t))) ||
        !ok(cudaMalloc(&dout, 4 * sizeof(uint64_t)))) {
      st = SFC_ERR_CUDA;
      break;
    }
    if (!ok(cudaFuncSetAttribute(reinterpret_cast<const void*>(&flag_pingpong),
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kFloorSmem)) ||
        !ok(cudaFuncSetAttribute(reinterpret_cast<const void*>(&list_sms), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kFloorSmem))) {
      st = SFC_ERR_CUDA;
      break;
    }
    // the SM ids present, sorted; 16 of them spread evenly: initiators at
    // even positions, responders at odd ones
    {
      void* args[] = {&dids};
      std::vector<int> ids(sm_count);
      if (!ok(cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(&list_sms), dim3(sm_count), dim3(32), args,
                                          kFloorSmem, nullptr)) ||
          !ok(cudaDeviceSynchronize()) ||
          !ok(cudaMemcpy(ids.data(), dids, sizeof(int) * sm_count, cudaMemcpyDeviceToHost))) {
        st = SFC_ERR_CUDA;
        break;
      }
      std::sort(ids.begin(), ids.end());
      ids.erase(std::unique(ids.begin(), ids.end()), ids.end());
      if (static_cast<int>(ids.size()) < 2 * SFC_FLOOR_SMS) {
        st = SFC_ERR_RESOURCES;
        break;
      }
      const int m = static_cast<int>(ids.size());
      for (int k = 0; k < 2 * SFC_FLOOR_SMS; ++k)
        sel[k] = ids[static_cast<size_t>((static_cast<int64_t>(k) * (m - 1) + (2 * SFC_FLOOR_SMS - 1) / 2) /
                                         (2 * SFC_FLOOR_SMS - 1))];
    }
    std::vector<uint64_t> hcycles(iters);
    const int skip = std::min(iters / 8, 64);
    for (int loc = 0; loc < SFC_FLOOR_LOCATIONS && st == SFC_OK; ++loc) {
      // two flags 4 KB apart; locations 4 MB + 4 KB * loc apart
      uint64_t* fa = reinterpret_cast<uint64_t*>(darena + static_cast<size_t>(loc) * ((4u << 20) + (4u << 10)));
      uint64_t* fb = fa + 512;
      for (int i = 0; i < SFC_FLOOR_SMS && st == SFC_OK; ++i) {
        for (int j = 0; j < SFC_FLOOR_SMS && st == SFC_OK; ++j) {
          int sa = sel[2 * i], sb = sel[2 * j + 1];
          int herr = 0;
          uint64_t hcal[2] = {0, 0};
          void* args[] = {&fa, &fb, &iters, &sa, &sb, &dcycles, &dcal, &derr};
          if (!ok(cudaMemset(fa, 0, sizeof(uint64_t))) || !ok(cudaMemset(fb, 0, sizeof(uint64_t))) ||
              !ok(cudaMemset(derr, 0, sizeof(int))) ||
              !ok(cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(&flag_pingpong), dim3(sm_count), dim3(32),
                                              args, kFloorSmem, nullptr)) ||
              !ok(cudaDeviceSynchronize()) || !ok(cudaMemcpy(&herr, derr, sizeof(int), cudaMemcpyDeviceToHost)) ||
              !ok(cudaMemcpy(hcycles.data(), dcycles, sizeof(uint64_t) * iters, cudaMemcpyDeviceToHost)) ||
              !ok(cudaMemcpy(hcal, dcal, sizeof(hcal), cudaMemcpyDeviceToHost))) {
            st = SFC_ERR_CUDA;
            break;
          }
          if (herr) {
            st = SFC_ERR_TIMEOUT;
            break;
          }
          std::vector<uint64_t> kept(hcycles.begin() + skip, hcycles.end());
          const double p50 = pct(kept, 0.5);
          trial_p50.push_back(p50);
          by_loc[loc].push_back(p50);
          cal_ns += hcal[0];
          cal_cyc += hcal[1];
        }
      }
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
    const double ghz = cal_ns ? static_cast<double>(cal_cyc) / static_cast<double>(cal_ns) : 1.0;
    out->sm_clock_ghz = ghz;
    out->flag_rtt_ns_p50 = pctd(trial_p50, 0.50) / ghz;
    out->flag_rtt_ns_p10 = pctd(trial_p50, 0.10) / ghz;
    out->flag_rtt_ns_p90 = pctd(trial_p50, 0.90) / ghz;
    out->flag_rtt_ns_min_pair = *std::min_element(trial_p50.begin(), trial_p50.end()) / ghz;
    out->flag_rtt_ns_max_pair = *std::max_element(trial_p50.begin(), trial_p50.end()) / ghz;
    for (int loc = 0; loc < SFC_FLOOR_LOCATIONS; ++loc) out->flag_rtt_ns_by_location[loc] = pctd(by_loc[loc], 0.5) / ghz;
    for (int i = 0; i < SFC_FLOOR_SMS; ++i) {
      out->initiator_sm[i] = sel[2 * i];
      out->responder_sm[i] = sel[2 * i + 1];
    }
    out->pairs = static_cast<int>(trial_p50.size());
    out->l2_rtt_ns_p50 = static_cast<double>(chase[0]) / steps / ghz;
    out->globaltimer_step_ns = static_cast<double>(step);
  } while (false);
  cudaFree(darena);
  cudaFree(dcycles);
  cudaFree(dcal);
  cudaFree(dids);
  cudaFree(derr);
  cudaFree(dchain);
  cudaFree(dout);
  return st;
}
