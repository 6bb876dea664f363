// Device primitives: memory operations with explicit PTX memory-model
// semantics, bf16 packing, bounded waits and error recording.
//
// Memory-ordering choices (PTX ISA memory consistency model):
//  * Pushes and polls of the self-synchronizing protocols use .relaxed.gpu
//    accesses: coherent at GPU scope (served by L2, never a stale L1 line)
//    and free of data races with each other.
//  * An aligned 8-byte access is single-copy atomic; a vector access is a
//    set of element accesses of its element size. The LL unit (data word +
//    epoch word) is therefore moved as a .b64 element, so data and flag of a
//    unit are always observed together.
//  * LL128 and the barriers order data before a flag with a release pattern
//    (fence / st.release) and read it back with an acquire pattern.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "sfc_internal.h"

namespace sfc {

#define SFC_DEV __device__ __forceinline__

constexpr unsigned kFull = 0xffffffffu;

SFC_DEV uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

SFC_DEV uint32_t smid() {
  uint32_t s;
  asm volatile("mov.u32 %0, %%smid;" : "=r"(s));
  return s;
}

// ---- relaxed (gpu scope) accesses ----------------------------------------
SFC_DEV void st_rlx_v2u64(void* p, uint64_t a, uint64_t b) {
  asm volatile("st.relaxed.gpu.global.v2.b64 [%0], {%1, %2};" ::"l"(p), "l"(a), "l"(b) : "memory");
}
SFC_DEV void ld_rlx_v2u64(const void* p, uint64_t& a, uint64_t& b) {
  asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}
SFC_DEV void st_rlx_v4u32(void* p, uint4 v) {
  asm volatile("st.relaxed.gpu.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}
SFC_DEV uint4 ld_rlx_v4u32(const void* p) {
  uint4 v;
  asm volatile("ld.relaxed.gpu.global.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}
SFC_DEV void st_rlx_v2u32(void* p, uint2 v) {
  asm volatile("st.relaxed.gpu.global.v2.b32 [%0], {%1, %2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}
SFC_DEV uint2 ld_rlx_v2u32(const void* p) {
  uint2 v;
  asm volatile("ld.relaxed.gpu.global.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p) : "memory");
  return v;
}
SFC_DEV void st_rlx_u64(void* p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
SFC_DEV uint64_t ld_rlx_u64(const void* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
SFC_DEV int ld_rlx_s32(const void* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// Atomic exchange (relaxed, gpu scope): returns the old 8 bytes, leaves v.
SFC_DEV uint64_t atom_exch_u64(void* p, uint64_t v) {
  uint64_t old;
  asm volatile("atom.relaxed.gpu.global.exch.b64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
  return old;
}
// Device-epoch mode: the epoch this launch starts at. Written by the
// previous launch's last warp; the kernel boundary makes it visible.
SFC_DEV uint32_t device_epoch(const uint32_t* w) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(w) : "memory");
  return v;
}
// Lane 0 of every warp that finished its launch counts itself; the last of
// `warps` resets the counter and publishes the next epoch.
SFC_DEV void finish_device_epoch(uint32_t* epoch_dev, uint32_t* done, uint32_t warps, uint32_t next) {
  __threadfence();
  if (atomicAdd(done, 1u) == warps - 1) {
    atomicExch(done, 0u);
    atomicExch(epoch_dev, next);
  }
}
// ---- release / acquire -----------------------------------------------------
SFC_DEV void st_rel_u64(void* p, uint64_t v) {
  asm volatile("st.release.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
SFC_DEV uint64_t ld_acq_u64(const void* p) {
  uint64_t v;
  asm volatile("ld.acquire.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
SFC_DEV void fence_acq_rel() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
// Release fence: with a later strong write it forms a release pattern (every
// earlier access of the thread, and those ordered before it by a barrier, is
// visible to whoever observes that write through an acquire pattern). It
// waits for the thread's outstanding stores: about 0.5 us on B200.
SFC_DEV void fence_rel() { asm volatile("fence.release.gpu;" ::: "memory"); }
// Acquire fence: with an earlier strong read it forms an acquire pattern.
// It waits for no stores: measured as cheap as no fence on B200.
SFC_DEV void fence_acq() { asm volatile("fence.acquire.gpu;" ::: "memory"); }

// ---- read-only inputs (never written while a kernel runs) -----------------
SFC_DEV uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}
SFC_DEV uint2 ld_nc_v2(const void* p) {
  uint2 v;
  asm("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
SFC_DEV uint32_t ld_nc_u16(const void* p) {
  unsigned short v;
  asm("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}
// Bring the line holding p into L2 (no register result).
SFC_DEV void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

template <typename T>
SFC_DEV T ld_nc_ptr(const T* p) {
  uint64_t v;
  asm("ld.global.nc.u64 %0, [%1];" : "=l"(v) : "l"(p));
  return reinterpret_cast<T>(v);
}

// ---- element helpers ---------------------------------------------------------
// 8 bf16 starting at element e0 (e0 % 8 == 0) of a 16-byte aligned array of
// `count` elements; elements at or past `count` read as +0.
SFC_DEV uint4 load8(const uint16_t* base, uint64_t e0, uint64_t count) {
  if (e0 + 8 <= count) return ld_nc_v4(base + e0);
  uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (e0 + i < count) w[i >> 1] |= ld_nc_u16(base + e0 + i) << (16 * (i & 1));
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// 4 bf16 starting at element e0 (e0 % 4 == 0); past `count` reads as +0.
SFC_DEV uint2 load4(const uint16_t* base, uint64_t e0, uint64_t count) {
  if (e0 + 4 <= count) return ld_nc_v2(base + e0);
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (e0 + i < count) w[i >> 1] |= ld_nc_u16(base + e0 + i) << (16 * (i & 1));
  return make_uint2(w[0], w[1]);
}

SFC_DEV void store_elem(uint16_t* p, uint32_t h) { *p = static_cast<uint16_t>(h); }

// Store the first n (<= 8) bf16 of v at element offset e0 of `base`, but none
// at or past element `limit`. Vector stores when aligned, else per element.
SFC_DEV void store_n(uint16_t* base, uint64_t e0, uint4 v, int n, uint64_t limit) {
  uint64_t avail = limit > e0 ? limit - e0 : 0;
  int m = avail < static_cast<uint64_t>(n) ? static_cast<int>(avail) : n;
  uint16_t* p = base + e0;
  const uintptr_t a = reinterpret_cast<uintptr_t>(p);
  if (m == 8 && (a & 15) == 0) {
    *reinterpret_cast<uint4*>(p) = v;
    return;
  }
  if (m == 8 && (a & 7) == 0) {
    reinterpret_cast<uint2*>(p)[0] = make_uint2(v.x, v.y);
    reinterpret_cast<uint2*>(p)[1] = make_uint2(v.z, v.w);
    return;
  }
  if (m == 4 && (a & 7) == 0) {
    *reinterpret_cast<uint2*>(p) = make_uint2(v.x, v.y);
    return;
  }
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (i < m) store_elem(p + i, (w[i >> 1] >> (16 * (i & 1))) & 0xffffu);
}

// ---- bf16 arithmetic ----------------------------------------------------------
SFC_DEV float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
SFC_DEV float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
SFC_DEV uint32_t pack_rn(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // round to nearest even
  return *reinterpret_cast<uint32_t*>(&h);
}
SFC_DEV uint32_t word(const uint4& v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}
SFC_DEV bool has_sentinel(uint32_t w) {
  return (w & 0xffffu) == 0xffffu || (w >> 16) == 0xffffu;
}
SFC_DEV bool has_sentinel(const uint4& v) {
  return has_sentinel(v.x) || has_sentinel(v.y) || has_sentinel(v.z) || has_sentinel(v.w);
}

// Rank-order reduction of 8 elements: acc = x_0; acc += x_q for q = 1..N-1
// with fp32 round-to-nearest adds (no FMA contraction), one final bf16 RNE.
template <int N>
SFC_DEV uint4 reduce8(const uint4 (&x)[N]) {
  float acc[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] = bf_lo(word(x[0], i));
    acc[2 * i + 1] = bf_hi(word(x[0], i));
  }
#pragma unroll
  for (int q = 1; q < N; ++q) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] = __fadd_rn(acc[2 * i], bf_lo(word(x[q], i)));
      acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], bf_hi(word(x[q], i)));
    }
  }
  return make_uint4(pack_rn(acc[0], acc[1]), pack_rn(acc[2], acc[3]), pack_rn(acc[4], acc[5]),
                    pack_rn(acc[6], acc[7]));
}

// ---- errors and bounded waits ------------------------------------------------
SFC_DEV void record_error(const KParams& p, int code, uint32_t info) {
  if (atomicCAS(&p.status->code, 0, code) == 0) atomicExch(&p.status->info, info);
  atomicExch(&p.status->abort, 1);
}

SFC_DEV uint32_t err_info(int op, int rank, int src) {
  return (static_cast<uint32_t>(op) << 16) | (static_cast<uint32_t>(rank & 0xff) << 8) |
         static_cast<uint32_t>(src & 0xff);
}

// Per-warp wait bookkeeping for the poll loops. tick() is called once per
// poll iteration by every lane of the warp (the loops are warp-uniform);
// every 32nd iteration lane 0 reads the clock and the abort word. A wait
// ends with `true` (give up) when the context was aborted or the wait has
// lasted longer than timeout_ns; the latter is recorded as a timeout.
struct WarpWait {
  uint64_t deadline = 0;
  uint32_t spins = 0;
  SFC_DEV bool tick(const KParams& p, int op, int rank, int src) {
    if ((++spins & 31u) != 0u) return false;
    int stop = 0;
    if ((threadIdx.x & 31) == 0) {
      const uint64_t now = gtimer();
      if (deadline == 0) deadline = now + p.timeout_ns;
      if (ld_rlx_s32(&p.status->abort)) {
        stop = 1;
      } else if (now > deadline) {
        record_error(p, 3 /* SFC_ERR_TIMEOUT */, err_info(op, rank, src));
        stop = 1;
      }
    }
    return __shfl_sync(kFull, stop, 0) != 0;
  }
};

// Single-thread bounded wait step (barrier flag polls).
struct ThreadWait {
  uint64_t deadline = 0;
  uint32_t spins = 0;
  SFC_DEV bool tick(const KParams& p, int op, int rank, int src) {
    if ((++spins & 31u) != 0u) return false;
    const uint64_t now = gtimer();
    if (deadline == 0) deadline = now + p.timeout_ns;
    if (ld_rlx_s32(&p.status->abort)) return true;
    if (now > deadline) {
      record_error(p, 3 /* SFC_ERR_TIMEOUT */, err_info(op, rank, src));
      return true;
    }
    return false;
  }
};

// Bounded start skew: spin `ns` nanoseconds (at most the timeout).
SFC_DEV void spin_ns(uint64_t ns, uint64_t cap) {
  if (ns > cap) ns = cap;
  const uint64_t end = gtimer() + ns;
  while (gtimer() < end) {
  }
}

}  // namespace sfc
