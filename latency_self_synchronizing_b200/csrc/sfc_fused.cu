// Row-parallel linear layer fused with its all-reduce, for one decode token
// (the tensor-parallel decode pattern "SiFAR: Synchronization-Free All-Reduce
// for Low-Latency LLM Inference", introduction, and "Why Microseconds Matter
// in AI Infrastructure", section "Latency can matter more than bandwidth",
// describe: per layer a sharded matrix product, then an all-reduce of the
// activation). Built on the public device LL API (sfc_ll_device.cuh): the
// partial product leaves the registers that computed it as LL units, with no
// intermediate buffer and no second launch ("Why Microseconds Matter in AI
// Infrastructure", section "Communication is becoming part of GPU execution").
//
// Rank r's CTAs compute p_r = W_r x_r: each warp owns output vectors (8 rows)
// v = wg, wg + W, ... (W = warps per rank); for each it streams the 8 rows
// of W_r once (lanes take consecutive 16-byte column chunks, fp32 FMA),
// combines the lanes with a butterfly, rounds the 8 sums to bf16 and leaves
// the vector in lane i for its i-th vector. Then every lane pushes its vector
// to all peers and polls the peers' vectors for the same v (warp-collective,
// bounded), folds them in rank order and stores y_r. The GEMV is HBM-bound
// (weights are read once); no tensor cores.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sfc_device.cuh"
#include "sfc_ll_device.cuh"

namespace sfc {
namespace {

SFC_DEV float dot8(uint4 w, uint4 x, float acc) {
  acc = fmaf(bf_lo(w.x), bf_lo(x.x), acc);
  acc = fmaf(bf_hi(w.x), bf_hi(x.x), acc);
  acc = fmaf(bf_lo(w.y), bf_lo(x.y), acc);
  acc = fmaf(bf_hi(w.y), bf_hi(x.y), acc);
  acc = fmaf(bf_lo(w.z), bf_lo(x.z), acc);
  acc = fmaf(bf_hi(w.z), bf_hi(x.z), acc);
  acc = fmaf(bf_lo(w.w), bf_lo(x.w), acc);
  acc = fmaf(bf_hi(w.w), bf_hi(x.w), acc);
  return acc;
}

template <int NR>
__global__ void __launch_bounds__(kLinearThreads, NR >= 6 ? 1 : 2) linear_allreduce_kernel(const __grid_constant__ LinearParams p) {
  extern __shared__ uint4 xs[];  // x_r, kdim / 8 vectors
  const int r = blockIdx.x / p.G;
  const int k = blockIdx.x - r * p.G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t kvec = p.kdim / 8;
  const uint16_t* W = p.W[r];
  for (uint64_t i = threadIdx.x; i < kvec; i += blockDim.x) xs[i] = ld_nc_v4(p.x[r] + i * 8);
  __syncthreads();
  const uint64_t nvec = p.hidden / 8;
  const uint64_t wg = static_cast<uint64_t>(k) * (kLinearThreads / 32) + warp;
  const uint64_t ws = static_cast<uint64_t>(p.G) * (kLinearThreads / 32);
  for (uint64_t base = wg; base < nvec; base += ws * 32) {
    uint4 mine = make_uint4(0, 0, 0, 0);
    for (int i = 0; i < 32; ++i) {
      const uint64_t v = base + static_cast<uint64_t>(i) * ws;
      if (v >= nvec) break;  // warp-uniform
      float acc[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) acc[m] = 0.f;
      const uint16_t* rows = W + v * 8 * p.kdim;
#pragma unroll 2
      for (uint64_t c = lane; c < kvec; c += 32) {
        const uint4 xv = xs[c];
        uint4 wv[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) wv[m] = ld_nc_v4(rows + m * p.kdim + c * 8);
#pragma unroll
        for (int m = 0; m < 8; ++m) acc[m] = dot8(wv[m], xv, acc[m]);
      }
#pragma unroll
      for (int m = 0; m < 8; ++m) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc[m] += __shfl_xor_sync(kFull, acc[m], off);
      }
      if (lane == i)
        mine = make_uint4(pack_rn(acc[0], acc[1]), pack_rn(acc[2], acc[3]), pack_rn(acc[4], acc[5]),
                          pack_rn(acc[6], acc[7]));
    }
    const uint64_t v = base + static_cast<uint64_t>(lane) * ws;
    const bool act = v < nvec;
    if (act) sfc_device::ll_push(p.view, r, p.epoch, v, mine);
    uint4 out;
    if (!sfc_device::ll_allreduce_lane<NR>(p.view, r, p.epoch, v, act, mine, &out)) return;
    if (act) *reinterpret_cast<uint4*>(p.y[r] + v * 8) = out;
  }
}

struct LinearTable {
  const void* t[kMaxRanks + 1] = {};
  LinearTable() {
    t[2] = reinterpret_cast<const void*>(&linear_allreduce_kernel<2>);
    t[3] = reinterpret_cast<const void*>(&linear_allreduce_kernel<3>);
    t[4] = reinterpret_cast<const void*>(&linear_allreduce_kernel<4>);
    t[5] = reinterpret_cast<const void*>(&linear_allreduce_kernel<5>);
    t[6] = reinterpret_cast<const void*>(&linear_allreduce_kernel<6>);
    t[7] = reinterpret_cast<const void*>(&linear_allreduce_kernel<7>);
    t[8] = reinterpret_cast<const void*>(&linear_allreduce_kernel<8>);
  }
};

}  // namespace

const void* linear_kernel_for(int nranks) {
  static const LinearTable table;
  return (nranks >= kMinRanks && nranks <= kMaxRanks) ? table.t[nranks] : nullptr;
}

}  // namespace sfc
