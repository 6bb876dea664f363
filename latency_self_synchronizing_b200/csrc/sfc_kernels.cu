// Persistent collective kernels: N emulated ranks, G CTAs per rank, k_ops
// operations per launch.
//
// Rank r owns CTAs [r * G, (r + 1) * G). Every operation uses the same
// element -> (CTA, thread) mapping, so thread t of CTA k of every rank forms
// an independent self-synchronizing pipeline: it pushes its elements of
// operation e, then polls the same elements from every peer, and the peers'
// threads with the same index do the same. A writer reaches epoch e+2 only
// after the reader's epoch e+1 push arrived, which the reader issues only
// after it consumed epoch e. That is the double buffering of "Why
// Microseconds Matter in AI Infrastructure", section "Latency can matter more
// than bandwidth": receipt of data is the evidence that the other buffer can
// be reused, with no global barrier.
//
// Why no fence is needed between one operation's reads and the next one's
// pushes (a fence.acq_rel.gpu costs about 0.6 us on B200 even with nothing
// outstanding):
//  * LL and sentinel: the reader's next push is control dependent on the
//    poll accesses that returned epoch e's data (the poll loop exits on their
//    values), and the writer's e+2 store is control dependent on observing
//    that push. For the writer's e+2 store to be seen by (or, for the
//    sentinel's exchange, to precede) the reader's epoch-e access, the cycle
//    access(e) -> push(e+1) -> poll(e+1) -> store(e+2) -> access(e) through
//    dependencies and reads-from would have to exist, which the PTX memory
//    model's no-thin-air axiom excludes.
//  * Sentinel: the reset is the write half of the atomic exchange that reads
//    the data, so it is ordered with the data by atomicity, not by a fence.
//  * LL128: the writer's release fence between data and flags also orders
//    every earlier access of the thread (its reads of the previous
//    operation's lines included) before its next flags.
//
// Within an operation a warp polls all its sources at once (independent
// loads, one round trip per poll) and the warp decides with a vote whether
// to poll again, so lanes never diverge in the wait loop. Sources are taken
// in arrival order; the reduction runs in rank order 0..N-1 on registers
// ("flash-comm: Self-Synchronizing Collective Communication for LLM
// Decoding", abstract: transport order decoupled from reduction order).
#include <cuda_runtime.h>

#include "sfc_device.cuh"
#include "sfc_ll_device.cuh"

namespace sfc {

// ---------------------------------------------------------------- addressing
template <int N>
SFC_DEV const uint16_t* in_ptr(const KParams& p, int op, int r) {
  if (p.addr_mode == 0) return p.in_inline[r];
  if (p.addr_mode == 1) return ld_nc_ptr(&p.in_table[op * N + r]);
  return p.in_base + (static_cast<uint64_t>(op) * N + r) * p.in_stride;
}
template <int N>
SFC_DEV uint16_t* out_ptr(const KParams& p, int op, int r) {
  if (p.addr_mode == 0) return p.out_inline[r];
  if (p.addr_mode == 1) return ld_nc_ptr(&p.out_table[op * N + r]);
  return p.out_base + (static_cast<uint64_t>(op) * N + r) * p.out_stride;
}
// Receive slot of `recv` for data from `src` (src != recv) at `par`.
template <int N>
SFC_DEV uint8_t* slot_ptr(const KParams& p, int recv, int par, int src) {
  const int j = src < recv ? src : src - 1;
  return p.scratch + static_cast<uint64_t>((recv * 2 + par) * (N - 1) + j) * p.slot_stride;
}

// The next operation's input is brought into L2 while this one is in flight,
// standing in for a decode layer whose freshly produced activation sits in L2
// when its all-reduce starts; its values are read only after this operation
// completes. Each rank touches its own input: up to 8 of the thread's
// vectors (every small message; the head of a large one).
SFC_DEV void prefetch_next_input(const uint16_t* nx, uint64_t gtid, uint64_t gstride, uint64_t nvec) {
  if (nx == nullptr) return;
  int n = 0;
  for (uint64_t v = gtid; v < nvec && n < 8; v += gstride, ++n) prefetch_l2(nx + v * 8);
}

// Operand pointers of the current operation and the next input, read one
// operation ahead so that no table load sits on an operation's critical path.
struct Operands {
  const uint16_t* in;
  uint16_t* out;
  const uint16_t* in_next;  // null on the last operation
};

// Scratch access check. A build with -DSFC_DEBUG tests every scratch access
// against the protocol's region; one out of it records SFC_ERR_GUARD (detail =
// the offset from the region start) and is skipped, so the waits then end on
// the abort word instead of the access touching memory outside the region.
// Normal builds compile the check away.
SFC_DEV bool scratch_in_bounds(const KParams& p, const void* ptr, uint64_t bytes) {
  const uint8_t* a = static_cast<const uint8_t*>(ptr);
  if (a >= p.scratch && a + bytes <= p.scratch + p.scratch_bytes) return true;
  record_error(p, 9 /* SFC_ERR_GUARD */, static_cast<uint32_t>(a - p.scratch));
  return false;
}
#ifdef SFC_DEBUG
#define SFC_SCRATCH(p, ptr, bytes, ...)            \
  do {                                              \
    if (scratch_in_bounds(p, ptr, bytes)) {         \
      __VA_ARGS__;                                  \
    }                                               \
  } while (0)
#else
#define SFC_SCRATCH(p, ptr, bytes, ...) \
  do {                                  \
    __VA_ARGS__;                        \
  } while (0)
#endif

// Source rank of receive slot j of rank r (slots skip the own rank).
SFC_DEV int src_rank(int j, int r) { return j < r ? j : j + 1; }

// LL layout shared with the public device API (one definition).
SFC_DEV uint64_t ll_off(uint64_t v, int half) { return sfc_device::ll_offset(v, half); }

// LL poll + reduce of this thread's vectors, K at a time (all loads of a
// batch issued before any is examined). K = 1 is what the kernels use:
// batching several vectors per poll measured no faster on B200, since where a
// thread owns several vectors the path is bandwidth-bound already. Sources are
// indexed j = 0..N-2 (q = j or j + 1 around r) so that no register is spent
// on the own slot.
template <int N, int OP, int K>
SFC_DEV bool ll_poll(const KParams& p, int r, int op, uint32_t e, uint64_t gtid, uint64_t gstride,
                     const uint8_t* my, const uint16_t* in_r, uint16_t* out_r) {
  const uint64_t count = p.count;
  const uint64_t nvec = (count + 7) >> 3;
  const int lane = threadIdx.x & 31;
  for (uint64_t vb = gtid - lane; vb < nvec; vb += gstride * K) {
    uint64_t v[K];
    uint4 own[K];
    uint32_t need = 0;  // bit i * (N - 1) + j
#pragma unroll
    for (int i = 0; i < K; ++i) {
      v[i] = vb + lane + i * gstride;
      const bool act = v[i] < nvec;
      own[i] = act ? load8(in_r, v[i] * 8, count) : make_uint4(0, 0, 0, 0);
      if (act) need |= ((1u << (N - 1)) - 1u) << (i * (N - 1));
    }
    uint64_t a[K][N - 1], b[K][N - 1], c[K][N - 1], d[K][N - 1];
    WarpWait ww;
    while (true) {
      // issue every pending load before looking at any result, so one poll
      // costs one round trip whatever the number of sources and vectors
      const uint32_t cur = need;
#pragma unroll
      for (int i = 0; i < K; ++i) {
        const uint64_t o0 = ll_off(v[i], 0), o1 = ll_off(v[i], 1);
#pragma unroll
        for (int j = 0; j < N - 1; ++j) {
          if (cur & (1u << (i * (N - 1) + j))) {
            const uint8_t* s = my + static_cast<uint64_t>(j) * p.slot_stride;
            SFC_SCRATCH(p, s + o0, 16, ld_rlx_v2u64(s + o0, a[i][j], b[i][j]));
            SFC_SCRATCH(p, s + o1, 16, ld_rlx_v2u64(s + o1, c[i][j], d[i][j]));
          }
        }
      }
#pragma unroll
      for (int i = 0; i < K; ++i) {
#pragma unroll
        for (int j = 0; j < N - 1; ++j) {
          const uint32_t bit = 1u << (i * (N - 1) + j);
          if ((cur & bit) && static_cast<uint32_t>(a[i][j] >> 32) == e && static_cast<uint32_t>(b[i][j] >> 32) == e &&
              static_cast<uint32_t>(c[i][j] >> 32) == e && static_cast<uint32_t>(d[i][j] >> 32) == e)
            need &= ~bit;
        }
      }
      if (!__any_sync(kFull, need != 0u)) break;
      if (ww.tick(p, op, r, need ? src_rank((__ffs(need) - 1) % (N - 1), r) : -1)) return false;
    }
#pragma unroll
    for (int i = 0; i < K; ++i) {
      if (v[i] >= nvec) continue;
      uint4 x[N];
#pragma unroll
      for (int q = 0; q < N; ++q) {
        // source q sits at j = q (q < r) or j = q - 1 (q > r)
        const int jl = q < N - 1 ? q : N - 2, jh = q > 0 ? q - 1 : 0;
        const uint4 lo = make_uint4(static_cast<uint32_t>(a[i][jl]), static_cast<uint32_t>(b[i][jl]),
                                    static_cast<uint32_t>(c[i][jl]), static_cast<uint32_t>(d[i][jl]));
        const uint4 hi = make_uint4(static_cast<uint32_t>(a[i][jh]), static_cast<uint32_t>(b[i][jh]),
                                    static_cast<uint32_t>(c[i][jh]), static_cast<uint32_t>(d[i][jh]));
        x[q] = q == r ? own[i] : (q < r ? lo : hi);
      }
      if (OP == kAllreduce) {
        store_n(out_r, v[i] * 8, reduce8<N>(x), 8, count);
      } else {
#pragma unroll
        for (int q = 0; q < N; ++q) store_n(out_r, q * count + v[i] * 8, x[q], 8, q * count + count);
      }
    }
  }
  return true;
}

// ===================================================================== LL
// Unit = 8 bytes {2 bf16, epoch}; a 16-byte input vector v becomes units
// 4v..4v+3 stored as two .v2.b64 stores. Readiness: all four epoch words of
// the two loads equal e.
template <int N, int OP>
SFC_DEV bool ll_op(const KParams& p, int r, int op, uint32_t e, uint64_t gtid, uint64_t gstride,
                   const Operands& io) {
  const uint64_t count = p.count;
  const uint64_t nvec = (count + 7) >> 3;
  const int par = e & 1;
  const uint64_t ehi = static_cast<uint64_t>(e) << 32;
  const uint16_t* in_r = io.in;
  uint16_t* out_r = io.out;

  if (r != p.silent_rank) {
    for (uint64_t v = gtid; v < nvec; v += gstride) {
      const uint4 x = load8(in_r, v * 8, count);
      const uint64_t o0 = ll_off(v, 0), o1 = ll_off(v, 1);
#pragma unroll
      for (int q = 0; q < N; ++q) {
        if (q == r) continue;
        uint8_t* s = slot_ptr<N>(p, q, par, r);
        SFC_SCRATCH(p, s + o0, 16, st_rlx_v2u64(s + o0, ehi | x.x, ehi | x.y));
        SFC_SCRATCH(p, s + o1, 16, st_rlx_v2u64(s + o1, ehi | x.z, ehi | x.w));
      }
    }
  }
  prefetch_next_input(io.in_next, gtid, gstride, nvec);

  const uint8_t* my = slot_ptr<N>(p, r, par, r == 0 ? 1 : 0);  // slot j = 0
  return ll_poll<N, OP, 1>(p, r, op, e, gtid, gstride, my, in_r, out_r);
}

// ================================================================ sentinel
// Sentinel poll + reduce, K vectors at a time, sources indexed j = 0..N-2
// (as in the LL poll); two bits per (vector, source): its low and high 8-byte
// unit.
template <int N, int OP, int K, bool kLoadPoll>
SFC_DEV bool sentinel_poll(const KParams& p, int r, int op, uint64_t gtid, uint64_t gstride, uint8_t* my,
                           const uint16_t* in_r, uint16_t* out_r) {
  constexpr uint64_t kFill = ~0ull;
  const uint64_t count = p.count;
  const uint64_t nvec = (count + 7) >> 3;
  const int lane = threadIdx.x & 31;
  for (uint64_t vb = gtid - lane; vb < nvec; vb += gstride * K) {
    uint64_t v[K];
    uint4 own[K];
    uint32_t need = 0;  // bits 2 * (i * (N - 1) + j) and + 1
#pragma unroll
    for (int i = 0; i < K; ++i) {
      v[i] = vb + lane + i * gstride;
      const bool act = v[i] < nvec;
      own[i] = act ? load8(in_r, v[i] * 8, count) : make_uint4(0, 0, 0, 0);
      if (act) need |= ((1u << (2 * (N - 1))) - 1u) << (2 * i * (N - 1));
    }
    uint64_t a[K][N - 1], b[K][N - 1];  // accepted units are never exchanged again
    WarpWait ww;
    while (true) {
      // every pending exchange is issued before any result is examined
      const uint32_t cur = need;
#pragma unroll
      for (int i = 0; i < K; ++i) {
#pragma unroll
        for (int j = 0; j < N - 1; ++j) {
          const int u = 2 * (i * (N - 1) + j);
          uint8_t* s = my + static_cast<uint64_t>(j) * p.slot_stride + v[i] * 16;
          if (kLoadPoll) {
            if (cur & (3u << u)) {
              uint64_t ta = kFill, tb = kFill;
              SFC_SCRATCH(p, s, 16, ld_rlx_v2u64(s, ta, tb));
              if (cur & (1u << u)) a[i][j] = ta;
              if (cur & (2u << u)) b[i][j] = tb;
            }
          } else {
            if (cur & (1u << u)) SFC_SCRATCH(p, s, 8, a[i][j] = atom_exch_u64(s, kFill));
            if (cur & (2u << u)) SFC_SCRATCH(p, s + 8, 8, b[i][j] = atom_exch_u64(s + 8, kFill));
          }
        }
      }
#pragma unroll
      for (int i = 0; i < K; ++i) {
#pragma unroll
        for (int j = 0; j < N - 1; ++j) {
          const int u = 2 * (i * (N - 1) + j);
          if ((cur & (1u << u)) && a[i][j] != kFill) need &= ~(1u << u);
          if ((cur & (2u << u)) && b[i][j] != kFill) need &= ~(2u << u);
        }
      }
      if (!__any_sync(kFull, need != 0u)) break;
      if (ww.tick(p, op, r, need ? src_rank(((__ffs(need) - 1) / 2) % (N - 1), r) : -1)) return false;
    }
    if (kLoadPoll) {  // the vector is taken from every source: write the fill back
#pragma unroll
      for (int i = 0; i < K; ++i) {
        if (v[i] >= nvec) continue;
#pragma unroll
        for (int j = 0; j < N - 1; ++j) {
          uint8_t* s = my + static_cast<uint64_t>(j) * p.slot_stride + v[i] * 16;
          SFC_SCRATCH(p, s, 16, st_rlx_v2u64(s, kFill, kFill));
        }
      }
    }
#pragma unroll
    for (int i = 0; i < K; ++i) {
      if (v[i] >= nvec) continue;
      uint4 x[N];
#pragma unroll
      for (int q = 0; q < N; ++q) {
        const int jl = q < N - 1 ? q : N - 2, jh = q > 0 ? q - 1 : 0;
        const uint4 lo = make_uint4(static_cast<uint32_t>(a[i][jl]), static_cast<uint32_t>(a[i][jl] >> 32),
                                    static_cast<uint32_t>(b[i][jl]), static_cast<uint32_t>(b[i][jl] >> 32));
        const uint4 hi = make_uint4(static_cast<uint32_t>(a[i][jh]), static_cast<uint32_t>(a[i][jh] >> 32),
                                    static_cast<uint32_t>(b[i][jh]), static_cast<uint32_t>(b[i][jh] >> 32));
        x[q] = q == r ? own[i] : (q < r ? lo : hi);
      }
      if (OP == kAllreduce) {
        store_n(out_r, v[i] * 8, reduce8<N>(x), 8, count);
      } else {
#pragma unroll
        for (int q = 0; q < N; ++q) store_n(out_r, q * count + v[i] * 8, x[q], 8, q * count + count);
      }
    }
  }
  return true;
}



// Raw data into a slot pre-filled with 0xFFFF. The writer moves each 8 bytes
// as one single-copy-atomic .b64 element, so an 8-byte unit of the slot is
// either all fill or all data, and data never equals the fill (inputs never
// hold 0xFFFF elements). Two ways to take and reset the units:
//  * exchange (kLoadPoll = false, small messages): the reader polls each
//    8-byte unit with an atomic exchange against the fill: a result other
//    than the fill is the data, and the same atomic operation has already
//    written the fill back (the reset). One L2 atomic per unit and per poll
//    that still finds the fill; lowest latency.
//  * load + store (kLoadPoll = true, large messages): the reader polls with
//    16-byte relaxed loads, writes the fill back with a relaxed store once a
//    vector is complete, and ends the operation with an acquire fence and a
//    release fence. A writer reuses the slot two epochs later only after it
//    has seen this rank's next push (its poll followed by its own acquire
//    fence), so the release / acquire pair orders the resets before that
//    reuse. No atomics: at (N - 1) x bytes >= 384 KB the L2's atomic
//    throughput, not the round trip, bounds the exchange polls, and the
//    release fence (about 0.5 us) costs less than the atomics it saves.
template <int N, int OP, bool kLoadPoll>
SFC_DEV bool sentinel_op(const KParams& p, int r, int op, uint32_t e, uint64_t gtid, uint64_t gstride,
                         const Operands& io) {
  const uint64_t count = p.count;
  const uint64_t nvec = (count + 7) >> 3;
  const int par = e & 1;
  const uint16_t* in_r = io.in;
  uint16_t* out_r = io.out;

  if (r != p.silent_rank) {
    for (uint64_t v = gtid; v < nvec; v += gstride) {
      const uint4 x = load8(in_r, v * 8, count);
      // the receivers of a sentinel element may never see it arrive: record
      // the error; every wait then sees the abort word and exits
      if (p.debug && has_sentinel(x)) record_error(p, 6 /* SFC_ERR_SENTINEL_IN_INPUT */, err_info(op, r, r));
      const uint64_t lo = (static_cast<uint64_t>(x.y) << 32) | x.x;
      const uint64_t hi = (static_cast<uint64_t>(x.w) << 32) | x.z;
#pragma unroll
      for (int q = 0; q < N; ++q) {
        if (q == r) continue;
        uint8_t* s = slot_ptr<N>(p, q, par, r) + v * 16;
        SFC_SCRATCH(p, s, 16, st_rlx_v2u64(s, lo, hi));
      }
    }
  }
  prefetch_next_input(io.in_next, gtid, gstride, nvec);

  uint8_t* my = slot_ptr<N>(p, r, par, r == 0 ? 1 : 0);
  if (!kLoadPoll) return sentinel_poll<N, OP, 1, false>(p, r, op, gtid, gstride, my, in_r, out_r);
  const bool ok = sentinel_poll<N, OP, 1, true>(p, r, op, gtid, gstride, my, in_r, out_r);
  // acquire (after this operation's polls) + release (before the next
  // operation's pushes): a peer that sees the next push has seen the resets
  fence_acq();
  fence_rel();
  return ok;
}

// =================================================================== LL128
// A line = 120 data bytes (60 bf16) + 8-byte flag (= epoch). A warp moves 4
// lines: lane l serves line 4g + (l >> 3), sub-slot s = l & 7; lanes s < 7
// carry 16 data bytes at line offset 16 s, lane 7 carries the last 8 data
// bytes (offset 112) and the flag (offset 120). Writers store all data,
// __syncwarp + fence.release.gpu, then the flags (release pattern: the warp
// barrier orders the other lanes' data stores before the flag lane's fence);
// readers poll flags with relaxed loads, fence.acquire.gpu + __syncwarp
// (acquire pattern, handed to the other lanes by the barrier), then load the
// data. The acquire fence waits for no store and costs next to nothing on
// B200; the release fence waits for the data stores to complete, which is
// the one round trip LL128 pays that LL does not. Flags of up to B line
// groups are polled at once.
template <int N>
struct LL128Batch {
  static constexpr int B = N >= 16 ? 1 : 16 / N;  // B * N <= 16 flags in flight per lane
};

template <int N, int OP>
SFC_DEV bool ll128_op(const KParams& p, int r, int op, uint32_t e, uint64_t gtid, uint64_t gstride,
                      const Operands& io) {
  constexpr int B = LL128Batch<N>::B;
  const uint64_t count = p.count;
  const uint64_t nlines = (count + kLL128Elems - 1) / kLL128Elems;
  const uint64_t ngroups = (nlines + kLL128LinesPerWarp - 1) / kLL128LinesPerWarp;
  const int par = e & 1;
  const int lane = threadIdx.x & 31;
  const int sub = lane & 7;
  const uint64_t lsel = static_cast<uint64_t>(lane >> 3);
  const uint64_t wg = gtid >> 5, wstride = gstride >> 5;
  const uint16_t* in_r = io.in;
  uint16_t* out_r = io.out;
  const uint32_t peers = ((1u << N) - 1u) & ~(1u << r);

  if (r != p.silent_rank) {
    for (uint64_t g = wg; g < ngroups; g += wstride) {
      const uint64_t L = g * kLL128LinesPerWarp + lsel;
      if (L < nlines) {
        const uint64_t e0 = L * kLL128Elems + sub * 8;
        const uint2 lo = load4(in_r, e0, count);
        const uint2 hi = sub < 7 ? load4(in_r, e0 + 4, count) : make_uint2(0u, 0u);
#pragma unroll
        for (int q = 0; q < N; ++q) {
          if (q == r) continue;
          uint8_t* s = slot_ptr<N>(p, q, par, r) + L * kLL128Line + sub * 16;
          if (sub < 7)
            SFC_SCRATCH(p, s, 16, st_rlx_v4u32(s, make_uint4(lo.x, lo.y, hi.x, hi.y)));
          else
            SFC_SCRATCH(p, s, 8, st_rlx_v2u32(s, lo));
        }
      }
    }
    __syncwarp();
    fence_rel();
    for (uint64_t g = wg; g < ngroups; g += wstride) {
      const uint64_t L = g * kLL128LinesPerWarp + lsel;
      if (L < nlines && sub == 7) {
#pragma unroll
        for (int q = 0; q < N; ++q) {
          if (q == r) continue;
          uint8_t* fl = slot_ptr<N>(p, q, par, r) + L * kLL128Line + 120;
          SFC_SCRATCH(p, fl, 8, st_rlx_u64(fl, static_cast<uint64_t>(e)));
        }
      }
    }
  }
  if (io.in_next != nullptr) {
    const uint16_t* nx = io.in_next;
    int n = 0;
    for (uint64_t g = wg; g < ngroups && n < 8; g += wstride, ++n) {
      const uint64_t L = g * kLL128LinesPerWarp + lsel;
      const uint64_t e0 = L * kLL128Elems + sub * 8;
      if (L < nlines && e0 < count) prefetch_l2(nx + e0);
    }
  }

  const uint8_t* my = slot_ptr<N>(p, r, par, r == 0 ? 1 : 0);
  for (uint64_t g0 = wg; g0 < ngroups; g0 += wstride * B) {
    uint32_t need = 0;
    if (sub == 7) {
#pragma unroll
      for (int b = 0; b < B; ++b) {
        const uint64_t g = g0 + b * wstride;
        const uint64_t L = g * kLL128LinesPerWarp + lsel;
        if (g < ngroups && L < nlines) need |= peers << (b * N);
      }
    }
    WarpWait ww;
    while (true) {
      // all pending flags of the batch are loaded before any is compared
      const uint32_t cur = need;
      uint64_t f[B * N];
#pragma unroll
      for (int b = 0; b < B; ++b) {
        const uint64_t L = (g0 + b * wstride) * kLL128LinesPerWarp + lsel;
#pragma unroll
        for (int q = 0; q < N; ++q) {
          if (cur & (1u << (b * N + q))) {
            const int j = q < r ? q : q - 1;
            const uint8_t* fl = my + static_cast<uint64_t>(j) * p.slot_stride + L * kLL128Line + 120;
            SFC_SCRATCH(p, fl, 8, f[b * N + q] = ld_rlx_u64(fl));
          }
        }
      }
#pragma unroll
      for (int i = 0; i < B * N; ++i)
        if ((cur & (1u << i)) && f[i] == static_cast<uint64_t>(e)) need &= ~(1u << i);
      if (!__any_sync(kFull, need != 0u)) break;
      if (ww.tick(p, op, r, -1)) return false;
    }
    fence_acq();
    __syncwarp();
#pragma unroll 1
    for (int b = 0; b < B; ++b) {
      const uint64_t g = g0 + b * wstride;
      const uint64_t L = g * kLL128LinesPerWarp + lsel;
      if (g >= ngroups || L >= nlines) continue;
      const uint64_t e0 = L * kLL128Elems + sub * 8;
      const int n = sub < 7 ? 8 : 4;
      const uint2 olo = load4(in_r, e0, count);
      const uint2 ohi = sub < 7 ? load4(in_r, e0 + 4, count) : make_uint2(0u, 0u);
      const uint4 own = make_uint4(olo.x, olo.y, ohi.x, ohi.y);
      uint4 x[N];
#pragma unroll
      for (int q = 0; q < N; ++q) {
        if (q == r) {
          x[q] = own;
        } else {
          const int j = q < r ? q : q - 1;
          const uint8_t* s = my + static_cast<uint64_t>(j) * p.slot_stride + L * kLL128Line + sub * 16;
          if (sub < 7) {
            SFC_SCRATCH(p, s, 16, x[q] = ld_rlx_v4u32(s));
          } else {
            uint2 t = make_uint2(0, 0);
            SFC_SCRATCH(p, s, 8, t = ld_rlx_v2u32(s));
            x[q] = make_uint4(t.x, t.y, 0u, 0u);
          }
        }
      }
      if (OP == kAllreduce) {
        store_n(out_r, e0, reduce8<N>(x), n, count);
      } else {
#pragma unroll
        for (int q = 0; q < N; ++q) store_n(out_r, q * count + e0, x[q], n, q * count + count);
      }
    }
  }
  return true;
}

// ======================================================= self-sync twoshot
// Reduce-scatter then all-gather, each a self-synchronizing push (LL units or
// sentinel fill), no barrier. Shards are sv = ceil(nvec / N) vectors; thread
// position v (0 <= v < sv, the same for every rank) handles vector v of every
// shard: it pushes vector v of each peer's shard s to rank s, polls and
// reduces vector v of its own shard, pushes the result to every peer, then
// polls vector v of every other shard. Each push is control dependent on the
// polls before it, which orders slot reuse as in the oneshot protocols.
template <int N, bool kLLenc>
struct TwoshotSlots {
  // reduce-scatter slot of `recv` from `src` at `par`, then all-gather slots
  SFC_DEV static uint8_t* rs(const KParams& p, int recv, int par, int src) { return slot_ptr<N>(p, recv, par, src); }
  SFC_DEV static uint8_t* ag(const KParams& p, int recv, int par, int src) {
    return slot_ptr<N>(p, recv, par, src) + static_cast<uint64_t>(2 * N * (N - 1)) * p.slot_stride;
  }
};

// Store one 8-element vector into a slot position v, encoded.
template <bool kLLenc>
SFC_DEV void push_vec(const KParams& p, uint8_t* slot, uint64_t v, uint4 x, uint64_t ehi) {
  if (kLLenc) {
    uint8_t* s0 = slot + ll_off(v, 0);
    uint8_t* s1 = slot + ll_off(v, 1);
    SFC_SCRATCH(p, s0, 16, st_rlx_v2u64(s0, ehi | x.x, ehi | x.y));
    SFC_SCRATCH(p, s1, 16, st_rlx_v2u64(s1, ehi | x.z, ehi | x.w));
  } else {
    uint8_t* s = slot + v * 16;
    SFC_SCRATCH(p, s, 16,
                st_rlx_v2u64(s, (static_cast<uint64_t>(x.y) << 32) | x.x, (static_cast<uint64_t>(x.w) << 32) | x.z));
  }
}

// Poll position v of the slots of the sources in `need` (bit q) until every
// one is in; the received vectors land in x[q]. Warp-uniform; false = abort.
template <int N, bool kLLenc>
SFC_DEV bool poll_vecs(const KParams& p, uint8_t* base, uint64_t v, uint32_t e, uint32_t need, uint4 (&x)[N], int op,
                       int r) {
  // slot of source q: base + j(q) * slot_stride, j(q) = q < r ? q : q - 1
  constexpr uint64_t kFill = ~0ull;
  // LL: bit q = source q pending; sentinel: bits 2q, 2q+1 = its two units
  uint32_t pend = 0;
  if (kLLenc) {
    pend = need;
  } else {
#pragma unroll
    for (int q = 0; q < N; ++q)
      if (need & (1u << q)) pend |= 3u << (2 * q);
  }
  uint64_t a[N], b[N], c[N], d[N];
  WarpWait ww;
  while (true) {
    const uint32_t cur = pend;
#pragma unroll
    for (int q = 0; q < N; ++q) {
      uint8_t* sq = base + static_cast<uint64_t>(q < r ? q : q - 1) * p.slot_stride;
      if (kLLenc) {
        if (cur & (1u << q)) {
          SFC_SCRATCH(p, sq + ll_off(v, 0), 16, ld_rlx_v2u64(sq + ll_off(v, 0), a[q], b[q]));
          SFC_SCRATCH(p, sq + ll_off(v, 1), 16, ld_rlx_v2u64(sq + ll_off(v, 1), c[q], d[q]));
        }
      } else {
        if (cur & (1u << (2 * q))) SFC_SCRATCH(p, sq + v * 16, 8, a[q] = atom_exch_u64(sq + v * 16, kFill));
        if (cur & (2u << (2 * q))) SFC_SCRATCH(p, sq + v * 16 + 8, 8, b[q] = atom_exch_u64(sq + v * 16 + 8, kFill));
      }
    }
#pragma unroll
    for (int q = 0; q < N; ++q) {
      if (kLLenc) {
        if ((cur & (1u << q)) && static_cast<uint32_t>(a[q] >> 32) == e && static_cast<uint32_t>(b[q] >> 32) == e &&
            static_cast<uint32_t>(c[q] >> 32) == e && static_cast<uint32_t>(d[q] >> 32) == e)
          pend &= ~(1u << q);
      } else {
        if ((cur & (1u << (2 * q))) && a[q] != kFill) pend &= ~(1u << (2 * q));
        if ((cur & (2u << (2 * q))) && b[q] != kFill) pend &= ~(2u << (2 * q));
      }
    }
    if (!__any_sync(kFull, pend != 0u)) break;
    if (ww.tick(p, op, r, pend ? (kLLenc ? __ffs(pend) - 1 : (__ffs(pend) - 1) / 2) : -1)) return false;
  }
#pragma unroll
  for (int q = 0; q < N; ++q) {
    if (!(need & (1u << q))) continue;
    if (kLLenc)
      x[q] = make_uint4(static_cast<uint32_t>(a[q]), static_cast<uint32_t>(b[q]), static_cast<uint32_t>(c[q]),
                        static_cast<uint32_t>(d[q]));
    else
      x[q] = make_uint4(static_cast<uint32_t>(a[q]), static_cast<uint32_t>(a[q] >> 32), static_cast<uint32_t>(b[q]),
                        static_cast<uint32_t>(b[q] >> 32));
  }
  return true;
}

template <int N, bool kLLenc>
SFC_DEV bool selfsync_twoshot_op(const KParams& p, int r, int op, uint32_t e, uint64_t gtid, uint64_t gstride,
                                 const Operands& io) {
  using S = TwoshotSlots<N, kLLenc>;
  const uint64_t count = p.count;
  const uint64_t nvec = (count + 7) >> 3;
  const uint64_t sv = shard_vectors(count, N);
  const int par = e & 1;
  const uint64_t ehi = static_cast<uint64_t>(e) << 32;
  const int lane = threadIdx.x & 31;
  const uint16_t* in_r = io.in;
  uint16_t* out_r = io.out;
  const uint32_t peers = ((1u << N) - 1u) & ~(1u << r);

  // reduce-scatter push: vector v of shard s of my input goes to rank s
  if (r != p.silent_rank) {
    for (uint64_t v = gtid; v < sv; v += gstride) {
#pragma unroll
      for (int s = 0; s < N; ++s) {
        if (s == r) continue;
        const uint64_t vg = s * sv + v;
        if (vg < nvec) push_vec<kLLenc>(p, S::rs(p, s, par, r), v, load8(in_r, vg * 8, count), ehi);
      }
    }
  }
  if (io.in_next != nullptr) {
    int n = 0;
    for (uint64_t v = gtid; v < sv && n < 8; v += gstride) {
#pragma unroll
      for (int s = 0; s < N; ++s) {
        const uint64_t vg = s * sv + v;
        if (vg < nvec && n < 8) {
          prefetch_l2(io.in_next + vg * 8);
          ++n;
        }
      }
    }
  }

  // reduce-scatter poll + reduce, then all-gather push of the result
  {
    uint8_t* base = S::rs(p, r, par, r == 0 ? 1 : 0);
    for (uint64_t vb = gtid - lane; vb < sv; vb += gstride) {
      const uint64_t v = vb + lane;
      const uint64_t vg = r * sv + v;
      const bool act = v < sv && vg < nvec;
      uint4 x[N];
      if (!poll_vecs<N, kLLenc>(p, base, v, e, act ? peers : 0u, x, op, r)) return false;
      if (act) {
        const uint4 own = load8(in_r, vg * 8, count);
#pragma unroll
        for (int q = 0; q < N; ++q)
          if (q == r) x[q] = own;  // static indices keep x in registers
        const uint4 y = reduce8<N>(x);
        store_n(out_r, vg * 8, y, 8, count);
        if (r != p.silent_rank) {
#pragma unroll
          for (int q = 0; q < N; ++q)
            if (q != r) push_vec<kLLenc>(p, S::ag(p, q, par, r), v, y, ehi);
        }
      }
    }
  }

  // all-gather poll: vector v of every other shard
  {
    uint8_t* base = S::ag(p, r, par, r == 0 ? 1 : 0);
    for (uint64_t vb = gtid - lane; vb < sv; vb += gstride) {
      const uint64_t v = vb + lane;
      uint32_t need = 0;
      if (v < sv) {
#pragma unroll
        for (int q = 0; q < N; ++q)
          if (q != r && q * sv + v < nvec) need |= 1u << q;
      }
      uint4 x[N];
      if (!poll_vecs<N, kLLenc>(p, base, v, e, need, x, op, r)) return false;
#pragma unroll
      for (int q = 0; q < N; ++q)
        if (need & (1u << q)) store_n(out_r, (q * sv + v) * 8, x[q], 8, count);
    }
  }
  return true;
}

// ============================================================ LL128, one load
// The same line layout, moved the way the "LL128 atomic design" of "Why
// Microseconds Matter in AI Infrastructure" (section "Latency can matter more
// than bandwidth") is built: the 8 lanes of a line store their 16 bytes (lane
// 7: 8 data bytes + the flag) in one warp-wide store instruction, and a reader
// takes the whole line with one warp-wide load, accepting the data read in
// the same instruction as a matching flag. No fence on either side. The PTX
// memory model does not promise that a 128-byte line written by one warp
// instruction is observed whole; this protocol relies on B200 behaving so
// (writes and reads of one line are single L2 requests), which the skewed
// million-operation stress test checks bit for bit. Opt-in only: the
// selector never picks it by default.
template <int N, int OP>
SFC_DEV bool ll128_fast_op(const KParams& p, int r, int op, uint32_t e, uint64_t gtid, uint64_t gstride,
                           const Operands& io) {
  const uint64_t count = p.count;
  const uint64_t nlines = (count + kLL128Elems - 1) / kLL128Elems;
  const uint64_t ngroups = (nlines + kLL128LinesPerWarp - 1) / kLL128LinesPerWarp;
  const int par = e & 1;
  const int lane = threadIdx.x & 31;
  const int sub = lane & 7;
  const int lead = lane | 7;  // the flag lane of this lane's line
  const uint64_t lsel = static_cast<uint64_t>(lane >> 3);
  const uint64_t wg = gtid >> 5, wstride = gstride >> 5;
  const uint16_t* in_r = io.in;
  uint16_t* out_r = io.out;

  if (r != p.silent_rank) {
    for (uint64_t g = wg; g < ngroups; g += wstride) {
      const uint64_t L = g * kLL128LinesPerWarp + lsel;
      if (L < nlines) {
        const uint64_t e0 = L * kLL128Elems + sub * 8;
        const uint2 lo = load4(in_r, e0, count);
        const uint2 hi = sub < 7 ? load4(in_r, e0 + 4, count) : make_uint2(static_cast<uint32_t>(e), 0u);
        const uint64_t a = (static_cast<uint64_t>(lo.y) << 32) | lo.x;
        const uint64_t b = (static_cast<uint64_t>(hi.y) << 32) | hi.x;
#pragma unroll
        for (int q = 0; q < N; ++q) {
          if (q == r) continue;
          uint8_t* s = slot_ptr<N>(p, q, par, r) + L * kLL128Line + sub * 16;
          SFC_SCRATCH(p, s, 16, st_rlx_v2u64(s, a, b));
        }
      }
    }
  }
  if (io.in_next != nullptr) {
    int n = 0;
    for (uint64_t g = wg; g < ngroups && n < 8; g += wstride, ++n) {
      const uint64_t L = g * kLL128LinesPerWarp + lsel;
      const uint64_t e0 = L * kLL128Elems + sub * 8;
      if (L < nlines && e0 < count) prefetch_l2(io.in_next + e0);
    }
  }

  const uint8_t* my = slot_ptr<N>(p, r, par, r == 0 ? 1 : 0);
  for (uint64_t g = wg; g < ngroups; g += wstride) {
    const uint64_t L = g * kLL128LinesPerWarp + lsel;
    const bool has = L < nlines;
    uint32_t need = has ? ((1u << (N - 1)) - 1u) : 0u;  // bit j: source j pending for this line
    uint64_t a[N - 1], b[N - 1];
    WarpWait ww;
    while (true) {
      const uint32_t cur = need;
#pragma unroll
      for (int j = 0; j < N - 1; ++j)
        if (cur & (1u << j)) {
          const uint8_t* s = my + static_cast<uint64_t>(j) * p.slot_stride + L * kLL128Line + sub * 16;
          SFC_SCRATCH(p, s, 16, ld_rlx_v2u64(s, a[j], b[j]));
        }
      // the flag lane decides for its line; the other 7 lanes take its verdict
      uint32_t okbits = 0;
#pragma unroll
      for (int j = 0; j < N - 1; ++j)
        if ((cur & (1u << j)) && b[j] == static_cast<uint64_t>(e)) okbits |= 1u << j;
      okbits = __shfl_sync(kFull, okbits, lead);
      need &= ~okbits;
      if (!__any_sync(kFull, need != 0u)) break;
      if (ww.tick(p, op, r, -1)) return false;
    }
    if (!has) continue;
    const uint64_t e0 = L * kLL128Elems + sub * 8;
    const int n = sub < 7 ? 8 : 4;
    const uint2 olo = load4(in_r, e0, count);
    const uint2 ohi = sub < 7 ? load4(in_r, e0 + 4, count) : make_uint2(0u, 0u);
    uint4 x[N];
#pragma unroll
    for (int q = 0; q < N; ++q) {
      const int jl = q < N - 1 ? q : N - 2, jh = q > 0 ? q - 1 : 0;
      const bool below = q < r;
      const uint64_t va = below ? a[jl] : a[jh];
      const uint64_t vb = below ? b[jl] : b[jh];
      x[q] = make_uint4(static_cast<uint32_t>(va), static_cast<uint32_t>(va >> 32),
                        sub < 7 ? static_cast<uint32_t>(vb) : 0u, sub < 7 ? static_cast<uint32_t>(vb >> 32) : 0u);
      if (q == r) x[q] = make_uint4(olo.x, olo.y, ohi.x, ohi.y);
    }
    if (OP == kAllreduce) {
      store_n(out_r, e0, reduce8<N>(x), n, count);
    } else {
#pragma unroll
      for (int q = 0; q < N; ++q) store_n(out_r, q * count + e0, x[q], n, q * count + count);
    }
  }
  return true;
}

// ============================================================ barriers
// Per-CTA-index barrier: CTA k of rank r publishes (epoch << 2) | phase with
// a release store and waits until CTA k of every rank has published at least
// that (acquire loads by threads 0..N-1). CTA-uniform result.
template <int N>
SFC_DEV bool cta_barrier(const KParams& p, int r, int k, int op, uint64_t target) {
  __syncthreads();
  int bad = 0;
  if (threadIdx.x == 0 && r != p.silent_rank)
    st_rel_u64(&p.bar[static_cast<uint64_t>(r) * p.bar_stride + k], target);
  if (threadIdx.x < N) {
    const uint64_t* f = &p.bar[static_cast<uint64_t>(threadIdx.x) * p.bar_stride + k];
    ThreadWait tw;
    while (ld_acq_u64(f) < target) {
      if (tw.tick(p, op, r, threadIdx.x)) {
        bad = 1;
        break;
      }
    }
  }
  return __syncthreads_or(bad) == 0;
}

// Oneshot (pull): top barrier, read every rank's input, reduce in rank
// order (all-gather: copy), bottom barrier ("SiFAR: Synchronization-Free
// All-Reduce for Low-Latency LLM Inference", abstract). The dual-buffered
// variant drops the bottom barrier: the caller alternates two input buffers,
// which is SiFAR's co-design of communication and model execution.
// Oneshot result for vector v: the rank-order reduction, or the N copies.
template <int N, int OP>
SFC_DEV void oneshot_emit(uint16_t* out_r, uint64_t v, const uint4 (&x)[N], uint64_t count) {
  if (OP == kAllreduce) {
    store_n(out_r, v * 8, reduce8<N>(x), 8, count);
  } else {
#pragma unroll
    for (int q = 0; q < N; ++q) store_n(out_r, q * count + v * 8, x[q], 8, q * count + count);
  }
}

template <int N, int OP, bool kDualBuffered>
SFC_DEV bool oneshot_op(const KParams& p, int r, int k, int op, uint32_t e, uint64_t gtid, uint64_t gstride,
                        const Operands& io) {
  const uint64_t count = p.count;
  const uint64_t nvec = (count + 7) >> 3;
  const uint64_t eb = static_cast<uint64_t>(e) << 2;
  if (!cta_barrier<N>(p, r, k, op, eb | kPhaseTop)) return false;
  prefetch_next_input(io.in_next, gtid, gstride, nvec);
  uint16_t* out_r = io.out;
  const uint16_t* src[N];
#pragma unroll
  for (int q = 0; q < N; ++q) src[q] = in_ptr<N>(p, op, q);
  // U of the thread's vectors per step (U * N loads in flight before any
  // use) while U remain, then one at a time
  constexpr int U = N <= 2 ? 8 : (N <= 4 ? 4 : 3);
  uint64_t v = gtid;
  for (; v + (U - 1) * gstride < nvec; v += U * gstride) {
    uint4 x[U][N];
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int q = 0; q < N; ++q) x[u][q] = load8(src[q], (v + u * gstride) * 8, count);
#pragma unroll
    for (int u = 0; u < U; ++u) oneshot_emit<N, OP>(out_r, v + u * gstride, x[u], count);
  }
  for (; v < nvec; v += gstride) {
    uint4 x[N];
#pragma unroll
    for (int q = 0; q < N; ++q) x[q] = load8(src[q], v * 8, count);
    oneshot_emit<N, OP>(out_r, v, x, count);
  }
  // with dual-buffered inputs the next operation's top barrier already
  // orders every reuse of this operation's inputs: no bottom barrier
  if (kDualBuffered) return true;
  return cta_barrier<N>(p, r, k, op, eb | kPhaseBottom);
}

// Twoshot (pull): top barrier; reduce-scatter (rank r reduces shard r of
// every input into its reduction buffer and its output); middle barrier;
// all-gather (copy every other rank's reduced shard); bottom barrier. CTA k
// of each rank covers the same vector offsets inside every shard, so the
// per-CTA-index barriers order each producer before its consumers.
template <int N>
SFC_DEV bool twoshot_op(const KParams& p, int r, int k, int op, uint32_t e, uint64_t gtid, uint64_t gstride,
                        const Operands& io) {
  const uint64_t count = p.count;
  const uint64_t nvec = (count + 7) >> 3;
  const uint64_t sv = (nvec + N - 1) / N;  // vectors per shard
  const uint64_t eb = static_cast<uint64_t>(e) << 2;
  if (!cta_barrier<N>(p, r, k, op, eb | kPhaseTop)) return false;
  prefetch_next_input(io.in_next, gtid, gstride, nvec);
  uint16_t* out_r = io.out;
  {
    const uint16_t* src[N];
#pragma unroll
    for (int q = 0; q < N; ++q) src[q] = in_ptr<N>(p, op, q);
    const uint64_t lo = r * sv, hi = min(lo + sv, nvec);
    uint16_t* red = p.red + static_cast<uint64_t>(r) * p.red_stride;
    auto emit = [&](uint64_t v, const uint4(&x)[N]) {
      const uint4 y = reduce8<N>(x);
      *reinterpret_cast<uint4*>(red + (v - lo) * 8) = y;
      store_n(out_r, v * 8, y, 8, count);
    };
    constexpr int U = N <= 2 ? 8 : (N <= 4 ? 4 : 3);
    uint64_t v = lo + gtid;
    for (; v + (U - 1) * gstride < hi; v += U * gstride) {
      uint4 x[U][N];
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int q = 0; q < N; ++q) x[u][q] = load8(src[q], (v + u * gstride) * 8, count);
#pragma unroll
      for (int u = 0; u < U; ++u) emit(v + u * gstride, x[u]);
    }
    for (; v < hi; v += gstride) {
      uint4 x[N];
#pragma unroll
      for (int q = 0; q < N; ++q) x[q] = load8(src[q], v * 8, count);
      emit(v, x);
    }
  }
  if (!cta_barrier<N>(p, r, k, op, eb | kPhaseMid)) return false;
#pragma unroll 1
  for (int q = 0; q < N; ++q) {
    if (q == r) continue;
    const uint64_t lo = q * sv, hi = min(lo + sv, nvec);
    const uint16_t* red = p.red + static_cast<uint64_t>(q) * p.red_stride;
    // eight of the thread's vectors per step (all loads before any store)
    // while eight remain, then one at a time
    constexpr int kU = 8;
    uint64_t v = lo + gtid;
    for (; v + (kU - 1) * gstride < hi; v += kU * gstride) {
      uint4 y[kU];
#pragma unroll
      for (int i = 0; i < kU; ++i) y[i] = ld_rlx_v4u32(red + (v + i * gstride - lo) * 8);
#pragma unroll
      for (int i = 0; i < kU; ++i) store_n(out_r, (v + i * gstride) * 8, y[i], 8, count);
    }
    for (; v < hi; v += gstride) store_n(out_r, v * 8, ld_rlx_v4u32(red + (v - lo) * 8), 8, count);
  }
  return cta_barrier<N>(p, r, k, op, eb | kPhaseBottom);
}

// ============================================================== the kernel
// Two CTAs per SM (at most 128 registers a thread), except the self-sync
// twoshot kernels for four or more ranks, whose two poll phases keep more
// sources in flight: one CTA per SM, so they never spill.
template <int N, int PROTO>
struct MinBlocks {
  static constexpr int value = ((PROTO == kLLTwoshot || PROTO == kSentinelTwoshot) && N >= 4) ? 1 : 2;
};

template <int N, int PROTO, int OP>
__global__ void __launch_bounds__(kThreads, MinBlocks<N, PROTO>::value) sfc_kernel(const __grid_constant__ KParams p) {
  const int r = blockIdx.x / p.G;
  const int k = blockIdx.x - r * p.G;
  // the launch picks 128 or kThreads threads per CTA; every rank uses the same
  const uint64_t gtid = static_cast<uint64_t>(k) * blockDim.x + threadIdx.x;
  const uint64_t gstride = static_cast<uint64_t>(p.G) * blockDim.x;
  const int lane = threadIdx.x & 31;
  // poisoned context: do nothing. Single operations of a context skip this
  // load (one L2 round trip before the first push, about 6 % of a single
  // call's GPU time); their waits see the abort word at their first check.
  if (!p.skip_abort_prologue && ld_rlx_s32(&p.status->abort)) return;
  uint32_t first = p.first_epoch;
  if (p.epoch_dev != nullptr) {
    first = device_epoch(p.epoch_dev);
    if (first == 0 || static_cast<uint64_t>(first) + p.k_ops - 1 > 0xFFFFFFFFull) {
      if (threadIdx.x == 0) record_error(p, 4 /* SFC_ERR_EPOCH */, first);
      return;
    }
  }
  if (p.timings != nullptr && lane == 0)
    atomicMin(reinterpret_cast<unsigned long long*>(&p.timings[0]), static_cast<unsigned long long>(gtimer()));
  Operands io{in_ptr<N>(p, 0, r), out_ptr<N>(p, 0, r), nullptr};
  for (int op = 0; op < p.k_ops; ++op) {
    const uint32_t e = first + static_cast<uint32_t>(op);
    io.in_next = op + 1 < p.k_ops ? in_ptr<N>(p, op + 1, r) : nullptr;
    uint16_t* out_next = op + 1 < p.k_ops ? out_ptr<N>(p, op + 1, r) : nullptr;
    if (p.skew != nullptr) spin_ns(__ldg(&p.skew[op * N + r]), p.timeout_ns);
    bool ok;
    if (PROTO == kLL)
      ok = ll_op<N, OP>(p, r, op, e, gtid, gstride, io);
    else if (PROTO == kSentinel)
      ok = sentinel_op<N, OP, false>(p, r, op, e, gtid, gstride, io);
    else if (PROTO == kSentinelLoadPoll)
      ok = sentinel_op<N, OP, true>(p, r, op, e, gtid, gstride, io);
    else if (PROTO == kLL128)
      ok = ll128_op<N, OP>(p, r, op, e, gtid, gstride, io);
    else if (PROTO == kLL128Fast)
      ok = ll128_fast_op<N, OP>(p, r, op, e, gtid, gstride, io);
    else if (PROTO == kOneshot)
      ok = oneshot_op<N, OP, false>(p, r, k, op, e, gtid, gstride, io);
    else if (PROTO == kOneshotDB)
      ok = oneshot_op<N, OP, true>(p, r, k, op, e, gtid, gstride, io);
    else if (PROTO == kLLTwoshot)
      ok = selfsync_twoshot_op<N, true>(p, r, op, e, gtid, gstride, io);
    else if (PROTO == kSentinelTwoshot)
      ok = selfsync_twoshot_op<N, false>(p, r, op, e, gtid, gstride, io);
    else
      ok = twoshot_op<N>(p, r, k, op, e, gtid, gstride, io);
    if (!ok) return;
    io.in = io.in_next;
    io.out = out_next;
    if (p.timings != nullptr && lane == 0)
      atomicMax(reinterpret_cast<unsigned long long*>(&p.timings[1 + p.timing_first + op]),
                static_cast<unsigned long long>(gtimer()));
  }
  if (p.epoch_dev != nullptr && lane == 0)
    finish_device_epoch(p.epoch_dev, p.done_ctr, gridDim.x * (blockDim.x >> 5), first + p.k_ops);
}

// ============================================================ dispatch table
namespace {
template <int N>
struct Row {
  static void fill(const void* (&t)[kMaxRanks + 1][kNumProtocols][2]) {
    t[N][kLL][kAllreduce] = reinterpret_cast<const void*>(&sfc_kernel<N, kLL, kAllreduce>);
    t[N][kLL][kAllgather] = reinterpret_cast<const void*>(&sfc_kernel<N, kLL, kAllgather>);
    t[N][kLL128][kAllreduce] = reinterpret_cast<const void*>(&sfc_kernel<N, kLL128, kAllreduce>);
    t[N][kLL128][kAllgather] = reinterpret_cast<const void*>(&sfc_kernel<N, kLL128, kAllgather>);
    t[N][kSentinel][kAllreduce] = reinterpret_cast<const void*>(&sfc_kernel<N, kSentinel, kAllreduce>);
    t[N][kSentinel][kAllgather] = reinterpret_cast<const void*>(&sfc_kernel<N, kSentinel, kAllgather>);
    t[N][kOneshot][kAllreduce] = reinterpret_cast<const void*>(&sfc_kernel<N, kOneshot, kAllreduce>);
    t[N][kOneshot][kAllgather] = reinterpret_cast<const void*>(&sfc_kernel<N, kOneshot, kAllgather>);
    t[N][kTwoshot][kAllreduce] = reinterpret_cast<const void*>(&sfc_kernel<N, kTwoshot, kAllreduce>);
    t[N][kTwoshot][kAllgather] = nullptr;
    t[N][kOneshotDB][kAllreduce] = reinterpret_cast<const void*>(&sfc_kernel<N, kOneshotDB, kAllreduce>);
    t[N][kOneshotDB][kAllgather] = reinterpret_cast<const void*>(&sfc_kernel<N, kOneshotDB, kAllgather>);
    t[N][kLLTwoshot][kAllreduce] = reinterpret_cast<const void*>(&sfc_kernel<N, kLLTwoshot, kAllreduce>);
    t[N][kLLTwoshot][kAllgather] = nullptr;
    t[N][kSentinelTwoshot][kAllreduce] = reinterpret_cast<const void*>(&sfc_kernel<N, kSentinelTwoshot, kAllreduce>);
    t[N][kSentinelTwoshot][kAllgather] = nullptr;
    t[N][kLL128Fast][kAllreduce] = reinterpret_cast<const void*>(&sfc_kernel<N, kLL128Fast, kAllreduce>);
    t[N][kLL128Fast][kAllgather] = reinterpret_cast<const void*>(&sfc_kernel<N, kLL128Fast, kAllgather>);
  }
  static void fill_load_poll(const void* (&t)[kMaxRanks + 1][2]) {
    t[N][kAllreduce] = reinterpret_cast<const void*>(&sfc_kernel<N, kSentinelLoadPoll, kAllreduce>);
    t[N][kAllgather] = reinterpret_cast<const void*>(&sfc_kernel<N, kSentinelLoadPoll, kAllgather>);
  }
};

struct Table {
  const void* t[kMaxRanks + 1][kNumProtocols][2] = {};
  const void* load_poll[kMaxRanks + 1][2] = {};  // the sentinel's large-message kernels
  Table() {
    Row<2>::fill(t);
    Row<3>::fill(t);
    Row<4>::fill(t);
    Row<5>::fill(t);
    Row<6>::fill(t);
    Row<7>::fill(t);
    Row<8>::fill(t);
    Row<2>::fill_load_poll(load_poll);
    Row<3>::fill_load_poll(load_poll);
    Row<4>::fill_load_poll(load_poll);
    Row<5>::fill_load_poll(load_poll);
    Row<6>::fill_load_poll(load_poll);
    Row<7>::fill_load_poll(load_poll);
    Row<8>::fill_load_poll(load_poll);
  }
};
const Table& table() {
  static const Table t;
  return t;
}
}  // namespace

const void* kernel_for(int nranks, int protocol, int op) {
  if (nranks < kMinRanks || nranks > kMaxRanks || protocol < kLL || protocol >= kNumProtocols || op < 0 || op > 1)
    return nullptr;
  return table().t[nranks][protocol][op];
}

const void* launch_kernel_for(int nranks, int protocol, int op, uint64_t count) {
  if (protocol == kSentinel && sentinel_load_poll(nranks, count) && nranks >= kMinRanks && nranks <= kMaxRanks &&
      op >= 0 && op <= 1)
    return table().load_poll[nranks][op];
  return kernel_for(nranks, protocol, op);
}

uint64_t slot_bytes_gpu(int protocol, uint64_t count, int n) {
  const uint64_t nvec = (count + 7) / 8;
  switch (protocol) {
    case kLL:
      return ((nvec + kLLChunkVecs - 1) / kLLChunkVecs) * kLLChunkBytes;
    case kLL128:
    case kLL128Fast: {
      const uint64_t lines = (count + kLL128Elems - 1) / kLL128Elems;
      const uint64_t groups = (lines + kLL128LinesPerWarp - 1) / kLL128LinesPerWarp;
      return groups * kLL128LinesPerWarp * kLL128Line;
    }
    case kSentinel:
      return nvec * 16;
    case kLLTwoshot:
      return ((shard_vectors(count, n) + kLLChunkVecs - 1) / kLLChunkVecs) * kLLChunkBytes;
    case kSentinelTwoshot:
      return shard_vectors(count, n) * 16;
    default:
      return 0;
  }
}

}  // namespace sfc
