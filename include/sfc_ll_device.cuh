/*
 * sfc_ll_device.cuh -- device-side LL API of libsfc, for CUDA kernels that
 * push and poll self-synchronizing LL units themselves ("Why Microseconds
 * Matter in AI Infrastructure", section "Communication is becoming part of
 * GPU execution": low-latency send, receive and reduction called directly
 * from inside kernels). Header only; include it in a .cu file compiled for
 * sm_100a. The view comes from sfc_get_ll_view, the epochs from
 * sfc_reserve_epochs (include/sfc.h).
 *
 * Layout (as the library's own LL kernels use it): an operation of `count`
 * bf16 per rank is cut into 16-byte vectors v = 0 .. ceil(count / 8) - 1;
 * vector v of rank src reaches rank dst as four 8-byte units {2 bf16, 32-bit
 * epoch}, written as two single-copy-atomic .v2.b64 stores at
 * sfc_ll_offset(v, 0) and sfc_ll_offset(v, 1) of dst's slot for src at parity
 * epoch & 1. A unit is valid when its epoch word equals the epoch.
 *
 * Rules the caller keeps (they are what makes the double buffer safe without
 * a barrier): every rank uses the same vector -> thread mapping for every
 * epoch; a thread pushes epoch e+1 only after its polls of epoch e returned;
 * epochs are used in sequence. The poll is warp-collective.
 */
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "sfc.h"

namespace sfc_device {

__device__ __forceinline__ uint64_t ll_offset(uint64_t v, int half) {
  // halves of 32 consecutive vectors lane-interleaved: 512 B + 512 B chunks
  return ((v >> 5) << 10) + (static_cast<uint64_t>(half) << 9) + ((v & 31) << 4);
}

__device__ __forceinline__ unsigned char* ll_slot(const sfc_ll_view& w, int recv, uint32_t epoch, int src) {
  const int j = src < recv ? src : src - 1;
  return w.scratch + static_cast<uint64_t>((recv * 2 + static_cast<int>(epoch & 1)) * (w.nranks - 1) + j) *
                         w.slot_stride;
}

__device__ __forceinline__ void st_v2u64(void* p, uint64_t a, uint64_t b) {
  asm volatile("st.relaxed.gpu.global.v2.b64 [%0], {%1, %2};" ::"l"(p), "l"(a), "l"(b) : "memory");
}
__device__ __forceinline__ void ld_v2u64(const void* p, uint64_t& a, uint64_t& b) {
  asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}

// Push vector v (8 bf16 as four 32-bit words) of rank `rank` to every peer.
__device__ __forceinline__ void ll_push(const sfc_ll_view& w, int rank, uint32_t epoch, uint64_t v, uint4 data) {
  const uint64_t ehi = static_cast<uint64_t>(epoch) << 32;
  for (int q = 0; q < w.nranks; ++q) {
    if (q == rank) continue;
    unsigned char* s = ll_slot(w, q, epoch, rank);
    st_v2u64(s + ll_offset(v, 0), ehi | data.x, ehi | data.y);
    st_v2u64(s + ll_offset(v, 1), ehi | data.z, ehi | data.w);
  }
}

// Warp-collective: every lane with `active` polls vector v from all peers
// (bounded by the view's timeout) and folds the N vectors in rank order in
// fp32 with one bf16 rounding; *out receives the result. Returns false if the
// wait ran out or the context was aborted (the timeout is recorded in the
// status block). NR = the number of ranks (compile-time).
template <int NR>
__device__ bool ll_allreduce_lane(const sfc_ll_view& w, int rank, uint32_t epoch, uint64_t v, bool active,
                                  uint4 own, uint4* out) {
  const uint64_t o0 = ll_offset(v, 0), o1 = ll_offset(v, 1);
  const unsigned char* base = ll_slot(w, rank, epoch, rank == 0 ? 1 : 0);
  uint32_t need = active ? ((1u << (NR - 1)) - 1u) : 0u;
  uint64_t a[NR - 1], b[NR - 1], c[NR - 1], d[NR - 1];
  uint64_t deadline = 0;
  uint32_t spins = 0;
  while (true) {
    const uint32_t cur = need;
#pragma unroll
    for (int j = 0; j < NR - 1; ++j)
      if (cur & (1u << j)) {
        const unsigned char* s = base + static_cast<uint64_t>(j) * w.slot_stride;
        ld_v2u64(s + o0, a[j], b[j]);
        ld_v2u64(s + o1, c[j], d[j]);
      }
#pragma unroll
    for (int j = 0; j < NR - 1; ++j)
      if ((cur & (1u << j)) && static_cast<uint32_t>(a[j] >> 32) == epoch &&
          static_cast<uint32_t>(b[j] >> 32) == epoch && static_cast<uint32_t>(c[j] >> 32) == epoch &&
          static_cast<uint32_t>(d[j] >> 32) == epoch)
        need &= ~(1u << j);
    if (!__any_sync(0xffffffffu, need != 0u)) break;
    if ((++spins & 31u) == 0u) {
      int stop = 0;
      if ((threadIdx.x & 31) == 0) {
        uint64_t now;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
        if (deadline == 0) deadline = now + w.timeout_ns;
        int ab;
        asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(ab) : "l"(w.status + 2) : "memory");
        if (ab) {
          stop = 1;
        } else if (now > deadline) {
          if (atomicCAS(w.status, 0, SFC_ERR_TIMEOUT) == 0) atomicExch(w.status + 1, 0xffffffffu);
          atomicExch(w.status + 2, 1);
          stop = 1;
        }
      }
      if (__shfl_sync(0xffffffffu, stop, 0)) return false;
    }
  }
  if (active) {
    float acc[8];
    bool first = true;
#pragma unroll
    for (int q = 0; q < NR; ++q) {
      const int jl = q < NR - 1 ? q : NR - 2, jh = q > 0 ? q - 1 : 0;
      // source q sits at j = q below the own rank and j = q - 1 above it;
      // both candidates use static indices so the arrays stay in registers
      const bool below = q < rank;
      uint32_t wd[4];
      wd[0] = static_cast<uint32_t>(below ? a[jl] : a[jh]);
      wd[1] = static_cast<uint32_t>(below ? b[jl] : b[jh]);
      wd[2] = static_cast<uint32_t>(below ? c[jl] : c[jh]);
      wd[3] = static_cast<uint32_t>(below ? d[jl] : d[jh]);
      if (q == rank) {
        wd[0] = own.x;
        wd[1] = own.y;
        wd[2] = own.z;
        wd[3] = own.w;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float lo = __uint_as_float(wd[i] << 16), hi = __uint_as_float(wd[i] & 0xffff0000u);
        acc[2 * i] = first ? lo : __fadd_rn(acc[2 * i], lo);
        acc[2 * i + 1] = first ? hi : __fadd_rn(acc[2 * i + 1], hi);
      }
      first = false;
    }
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
      o[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    *out = make_uint4(o[0], o[1], o[2], o[3]);
  }
  return true;
}

}  // namespace sfc_device
