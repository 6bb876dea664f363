// Row-parallel linear layer fused with its all-reduce, for 1..8 decode tokens
// (the tensor-parallel decode pattern "SiFAR: Synchronization-Free All-Reduce
// for Low-Latency LLM Inference", introduction, and "Why Microseconds Matter
// in AI Infrastructure", section "Latency can matter more than bandwidth",
// describe: per layer a sharded matrix product, then an all-reduce of the
// activation). Built on the public device LL API (sfc_ll_device.cuh): each
// finished 8-row output vector leaves as LL units while the weights of the
// next ones are still streaming, with no intermediate buffer and no second
// launch ("Why Microseconds Matter in AI Infrastructure", section
// "Communication is becoming part of GPU execution").
//
// Rank r owns G CTAs; CTA k owns the contiguous output vectors [v0, v1) of
// p_r = W_r x_r (vector v = rows 8v .. 8v+7). The layer is bound by
// streaming W from HBM once; a single token is a matrix-vector product, so
// there is no tensor-core work. The CTA's 8 warps form 8 / ks groups of ks
// warps; a group takes one vector at a time and its warps split the columns
// into ks parts. A warp streams its 8 row segments with 16-byte loads
// (lanes on consecutive chunks, 16 loads in flight per lane), keeps 8 fp32
// dot products, and folds them across the warp in 9 shuffles (a transposing
// butterfly: 4, 2, 1 values exchanged, then two plain levels), leaving row m's
// sum in lanes 4m .. 4m+3. The last warp of a group to finish a vector adds
// the ks parts in part order, rounds to bf16 and pushes the vector to every
// peer. After the CTA's last vector, all its threads poll their vectors
// (rank-order fp32 fold, one bf16 rounding) and store y_r.
//
// Several tokens (a decode step's batch) share one pass over the weights: a
// kernel instance carries a token tile T (1, 2, 4 or 8), keeps 8 x T dot
// products per lane and pushes one vector per (token, 8 rows); token u's
// vector v is LL vector u * hidden / 8 + v, so the all-reduce covers
// tokens x hidden elements. Shapes in whole 16-row, 32-column tiles take the
// tensor-core kernels below instead for 2..8 tokens (16-row x 8-token MMA
// tiles, weight pieces of 16 or 32 bytes, one or two CTAs an SM).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sfc_device.cuh"
#include "sfc_ll_device.cuh"

namespace sfc {
namespace {

// streamed once: keep it out of L1
SFC_DEV uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// acc + w0 x0 + w1 x1 + ... + w7 x7, one fp32 FMA per element in element
// order, each taking its two bf16 operands as they are (sm_100's mixed
// bf16 x bf16 + f32 FMA: the same exact-product, single-rounding step as
// widening both to f32 first, without the widening instructions).
SFC_DEV float dot8(uint4 w, uint4 x, float acc) {
  asm("{\n\t.reg .b16 w0, w1, w2, w3, w4, w5, w6, w7, x0, x1, x2, x3, x4, x5, x6, x7;\n\t"
      "mov.b32 {w0, w1}, %1;\n\tmov.b32 {w2, w3}, %2;\n\tmov.b32 {w4, w5}, %3;\n\tmov.b32 {w6, w7}, %4;\n\t"
      "mov.b32 {x0, x1}, %5;\n\tmov.b32 {x2, x3}, %6;\n\tmov.b32 {x4, x5}, %7;\n\tmov.b32 {x6, x7}, %8;\n\t"
      "fma.rn.f32.bf16 %0, w0, x0, %0;\n\tfma.rn.f32.bf16 %0, w1, x1, %0;\n\t"
      "fma.rn.f32.bf16 %0, w2, x2, %0;\n\tfma.rn.f32.bf16 %0, w3, x3, %0;\n\t"
      "fma.rn.f32.bf16 %0, w4, x4, %0;\n\tfma.rn.f32.bf16 %0, w5, x5, %0;\n\t"
      "fma.rn.f32.bf16 %0, w6, x6, %0;\n\tfma.rn.f32.bf16 %0, w7, x7, %0;\n\t}"
      : "+f"(acc)
      : "r"(w.x), "r"(w.y), "r"(w.z), "r"(w.w), "r"(x.x), "r"(x.y), "r"(x.z), "r"(x.w));
  return acc;
}

// Warp fold of 8 per-lane partial sums: returns the sum over all 32 lanes of
// row m = 4 * bit4 + 2 * bit3 + bit2 of the lane index.
SFC_DEV float fold8(const float (&a)[8], int lane) {
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
  float h[4], q[2];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float send = b4 ? a[i] : a[i + 4];
    h[i] = (b4 ? a[i + 4] : a[i]) + __shfl_xor_sync(kFull, send, 16);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float send = b3 ? h[i] : h[i + 2];
    q[i] = (b3 ? h[i + 2] : h[i]) + __shfl_xor_sync(kFull, send, 8);
  }
  float s = (b2 ? q[1] : q[0]) + __shfl_xor_sync(kFull, b2 ? q[0] : q[1], 4);
  s += __shfl_xor_sync(kFull, s, 2);
  s += __shfl_xor_sync(kFull, s, 1);
  return s;
}

// Shared memory: x_r [T][kdim] | parts [per][ks][T][8] fp32 |
// own [per][T] (packed bf16) | counters [per]. T = token tile (1, 2, 4, 8);
// tokens past p.tokens are zero and never leave the CTA.
// (8 tokens keep 64 accumulators a lane: one CTA per SM, so nothing spills)
template <int NR, int T>
__global__ void __launch_bounds__(kLinearThreads, T >= 8 ? 1 : 2)
    linear_allreduce_kernel(const __grid_constant__ LinearParams p) {
  extern __shared__ __align__(16) unsigned char sm[];
  const int r = blockIdx.x / p.G;
  const int k = blockIdx.x - r * p.G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t kdim = p.kdim, kvec = kdim / 8, nvec = p.hidden / 8;
  const uint32_t per = p.per_cta, ks = p.ks, tokens = p.tokens;
  const uint32_t epoch = p.epoch_dev != nullptr ? device_epoch(p.epoch_dev) : p.epoch;
  if (epoch == 0 || epoch == 0xFFFFFFFFu) {  // device epochs ran out: sfc_reset first
    if (threadIdx.x == 0) {
      if (atomicCAS(p.view.status, 0, static_cast<int>(SFC_ERR_EPOCH)) == 0) atomicExch(p.view.status + 1, 0);
      atomicExch(p.view.status + 2, 1);
    }
    return;
  }
  const uint64_t v0 = static_cast<uint64_t>(k) * per;
  const uint64_t v1 = v0 + per < nvec ? v0 + per : nvec;
  const uint32_t owned = v0 < v1 ? static_cast<uint32_t>(v1 - v0) : 0u;

  uint4* xs = reinterpret_cast<uint4*>(sm);
  float* parts = reinterpret_cast<float*>(sm + kdim * 2 * T);
  uint4* ownv = reinterpret_cast<uint4*>(parts + static_cast<uint64_t>(per) * ks * T * 8);
  uint32_t* cnt = reinterpret_cast<uint32_t*>(ownv + static_cast<uint64_t>(per) * T);

  for (uint64_t i = threadIdx.x; i < kvec * T; i += blockDim.x) {
    const uint64_t tok = i / kvec;
    xs[i] = tok < tokens ? ld_nc_v4(p.x[r] + tok * kdim + (i - tok * kvec) * 8) : make_uint4(0, 0, 0, 0);
  }
  for (uint32_t i = threadIdx.x; i < per; i += blockDim.x) cnt[i] = 0;
  __syncthreads();

  const uint32_t groups = kLinearWarps / ks, g = warp / ks, h = warp % ks;
  const uint64_t c_lo = kvec * h / ks, c_hi = kvec * (h + 1) / ks;  // this warp's column chunks
  const uint16_t* W = p.W[r];
  for (uint32_t t = g; t < owned; t += groups) {
    const uint16_t* rows = W + (v0 + t) * 8 * kdim;
    float acc[T][8];
#pragma unroll
    for (int u = 0; u < T; ++u)
#pragma unroll
      for (int m = 0; m < 8; ++m) acc[u][m] = 0.f;
    // two chunks' loads in flight up to 4 tokens; at 8 tokens the 64
    // accumulators leave no room (measured: unrolling there is slower)
#pragma unroll(T <= 4 ? 2 : 1)
    for (uint64_t c = c_lo + lane; c < c_hi; c += 32) {
      uint4 wv[8];
#pragma unroll
      for (int m = 0; m < 8; ++m) wv[m] = ld_stream_v4(rows + m * kdim + c * 8);
#pragma unroll
      for (int u = 0; u < T; ++u) {
        const uint4 xv = xs[u * kvec + c];
#pragma unroll
        for (int m = 0; m < 8; ++m) acc[u][m] = dot8(wv[m], xv, acc[u][m]);
      }
    }
    float* pt = parts + (static_cast<uint64_t>(t) * ks + h) * T * 8;
#pragma unroll
    for (int u = 0; u < T; ++u) {
      const float s = fold8(acc[u], lane);
      if ((lane & 3) == 0) pt[u * 8 + (lane >> 2)] = s;
    }
    __threadfence_block();
    __syncwarp();
    if (lane == 0) {
      // the last of the group's ks warps completes the vector (all tokens)
      if (atomicAdd(&cnt[t], 1u) == ks - 1) {
        __threadfence_block();
        const volatile float* pv = parts + static_cast<uint64_t>(t) * ks * T * 8;
        for (uint32_t u = 0; u < tokens; ++u) {
          float y[8];
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            y[m] = pv[u * 8 + m];
            for (uint32_t j = 1; j < ks; ++j) y[m] += pv[(j * T + u) * 8 + m];
          }
          const uint4 own = make_uint4(pack_rn(y[0], y[1]), pack_rn(y[2], y[3]), pack_rn(y[4], y[5]),
                                       pack_rn(y[6], y[7]));
          ownv[t * T + u] = own;
          sfc_device::ll_push(p.view, r, epoch, u * nvec + v0 + t, own);
        }
      }
    }
  }
  __syncthreads();  // every vector of the CTA is pushed and its own part stored
  const uint32_t work = owned * tokens;
  for (uint32_t base = 0; base < work; base += kLinearThreads) {
    const uint32_t i = base + threadIdx.x;
    const bool act = i < work;
    const uint32_t u = act ? i / owned : 0, t = act ? i - u * owned : 0;
    const uint4 own = act ? ownv[t * T + u] : make_uint4(0, 0, 0, 0);
    uint4 out;
    if (!sfc_device::ll_allreduce_lane<NR>(p.view, r, epoch, u * nvec + v0 + t, act, own, &out)) return;
    if (act) *reinterpret_cast<uint4*>(p.y[r] + u * p.hidden + (v0 + t) * 8) = out;
  }
  if (p.epoch_dev != nullptr && lane == 0)
    finish_device_epoch(p.epoch_dev, p.done_ctr, gridDim.x * (blockDim.x >> 5), epoch + 1);
}

// ---------------------------------------------------------------------------
// 2..8 tokens on the tensor cores (mma.sync m16n8k16, bf16 in, fp32 out).
// The tile is 16 rows of W_r (two LL vectors) by 8 token columns (tokens past
// p.tokens are zero). The MMA's k order is a permutation both operands share,
// chosen so that every thread reads its weights as whole 16- or 32-byte
// pieces: thread (group g, quad q) takes W[row0 + g][k0 + P q .. P q + P-1]
// and W[row0 + g + 8][same], P = 8 or 16 columns, the block being 4P
// columns wide. Each 4 consecutive columns c .. c+3 of a thread's piece feed
// one MMA step: its A registers are (row g, c..c+1), (row g+8, c..c+1),
// (row g, c+2..c+3), (row g+8, c+2..c+3), which the instruction reads as
// the logical columns 2q, 2q+1 / 2q+8, 2q+9, and its B registers are
// x[token g] at the same physical columns under the same logical names. Over
// the four quads one step covers 16 distinct columns, so the steps compute
// W x exactly as a sum over the block's columns (fp32 accumulation, in the
// steps' order). The multiply-adds are far below the tensor pipe's rate; the
// weight stream bounds the layer, which is why the legacy warp-level
// instruction suffices here.
SFC_DEV void mma_16x8x16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 32 bytes of a weight row (the address 32-byte aligned), streamed once
SFC_DEV void ld_stream_v8(const void* p, uint32_t (&v)[8]) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "l"(p));
}

// One column block of a thread: its piece of rows g and g + 8 (kWide: 32
// bytes each, 64-column blocks; else 16 bytes, 32-column blocks).
template <bool kWide>
struct MmaBlock {
  static constexpr int kCols = kWide ? 64 : 32;  // columns per block
  static constexpr int kRegs = kWide ? 8 : 4;    // registers per row piece
  static constexpr int kRing = kWide ? 4 : 8;    // blocks in flight per thread: 256 bytes either way (x2 at one CTA an SM)
  SFC_DEV static void load(const uint16_t* src, uint32_t (&v)[kRegs]) {
    if constexpr (kWide) {
      ld_stream_v8(src, v);
    } else {
      const uint4 t = ld_stream_v4(src);
      v[0] = t.x, v[1] = t.y, v[2] = t.z, v[3] = t.w;
    }
  }
  // xp: x[token g] at the thread's first column of the block (shared memory)
  SFC_DEV static void mma(float (&d)[4], const uint32_t (&ra)[kRegs], const uint32_t (&rb)[kRegs],
                          const uint16_t* xp, bool tok_ok) {
#pragma unroll
    for (int h = 0; h < kRegs / 4; ++h) {
      const uint4 xv = tok_ok ? *reinterpret_cast<const uint4*>(xp + 8 * h) : make_uint4(0, 0, 0, 0);
      mma_16x8x16(d, ra[4 * h], rb[4 * h], ra[4 * h + 1], rb[4 * h + 1], xv.x, xv.y);
      mma_16x8x16(d, ra[4 * h + 2], rb[4 * h + 2], ra[4 * h + 3], rb[4 * h + 3], xv.z, xv.w);
    }
  }
};

// Shared memory: x_r [tokens][kdim] | parts [per][ks][16 rows][8 tokens]
// fp32 | own [per][2 vectors][8 tokens] (packed bf16) | counters [per]. A CTA
// owns the 16-row tiles [t0, t0 + per) of its rank; LL vector
// u * hidden / 8 + v carries rows 8v .. 8v+7 of token u. A warp keeps
// kRing blocks of loads in flight as a rolling ring (block i + kRing is
// requested as soon as block i's MMAs have read their registers); the first
// tile's ring is filled before the activation is waited for. (Measured on
// B200 and dropped: refilling the ring with the next tile's first blocks
// during a tile's last round, and x rows padded to shift the token rows'
// banks, each 0.5-2 % slower.) With 32-byte pieces a 32-column rest of the
// row (kdim % 64 == 32) is one 16-byte-piece block, taken by the tile's last
// part. kCtasPerSm = 1: one CTA an SM with a ring twice as deep (the same
// bytes in flight an SM), for activations so large that two CTAs' shared
// memory would leave the SM's unified L1 too little room for the loads in
// flight.
template <int NR, bool kWide, int kCtasPerSm>
__global__ void __launch_bounds__(kLinearThreads, kCtasPerSm) linear_mma_kernel(const __grid_constant__ LinearParams p) {
  using B = MmaBlock<kWide>;
  constexpr int kRing = B::kRing * (kCtasPerSm == 1 ? 2 : 1);
  extern __shared__ __align__(16) unsigned char sm[];
  const int r = blockIdx.x / p.G;
  const int kb = blockIdx.x - r * p.G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  const uint64_t kdim = p.kdim, nvec = p.hidden / 8, ntiles = p.hidden / 16;
  const uint32_t per = p.per_cta, ks = p.ks, tokens = p.tokens;
  const uint32_t epoch = p.epoch_dev != nullptr ? device_epoch(p.epoch_dev) : p.epoch;
  if (epoch == 0 || epoch == 0xFFFFFFFFu) {  // device epochs ran out: sfc_reset first
    if (threadIdx.x == 0) {
      if (atomicCAS(p.view.status, 0, static_cast<int>(SFC_ERR_EPOCH)) == 0) atomicExch(p.view.status + 1, 0);
      atomicExch(p.view.status + 2, 1);
    }
    return;
  }
  const uint64_t t0 = static_cast<uint64_t>(kb) * per;
  const uint64_t t1 = t0 + per < ntiles ? t0 + per : ntiles;
  const uint32_t owned = t0 < t1 ? static_cast<uint32_t>(t1 - t0) : 0u;

  uint16_t* xs = reinterpret_cast<uint16_t*>(sm);
  float* parts = reinterpret_cast<float*>(sm + ((tokens * kdim * 2 + 15) & ~15ull));
  uint4* ownv = reinterpret_cast<uint4*>(parts + static_cast<uint64_t>(per) * ks * 128);
  uint32_t* cnt = reinterpret_cast<uint32_t*>(ownv + static_cast<uint64_t>(per) * 16);

  // x_r into shared memory: every thread issues its 16-byte asynchronous
  // copies (no register round trip) before any is waited for, so the whole
  // activation is in flight at once
  {
    const uint32_t xb = static_cast<uint32_t>(__cvta_generic_to_shared(xs));
    const char* src = reinterpret_cast<const char*>(p.x[r]);
    const uint32_t bytes = static_cast<uint32_t>(tokens * kdim * 2);
#pragma unroll 1
    for (uint32_t o = threadIdx.x * 16; o < bytes; o += kLinearThreads * 16)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(xb + o), "l"(src + o) : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
  }

  const uint32_t groups = kLinearWarps / ks, grp = warp / ks, h = warp % ks;
  const uint64_t blocks = kdim / B::kCols;                                // whole blocks of a row
  const bool rest32 = kWide && (kdim & 63) != 0 && h == ks - 1;          // this part takes the 32-column rest
  const uint64_t s_lo = blocks * h / ks, s_hi = blocks * (h + 1) / ks;  // this warp's blocks
  const uint64_t ring_end = s_lo + (s_hi - s_lo) / kRing * kRing;        // blocks that go through the ring
  const bool ring = ring_end > s_lo;
  const uint16_t* W = p.W[r];
  const uint32_t col = q * (B::kCols / 4);  // the thread's first column in a block
  uint32_t a[kRing][B::kRegs], b[kRing][B::kRegs];
  bool filled = false;  // the ring holds the first tile's first kRing blocks
  if (ring && grp < owned) {
    const uint16_t* wg = W + ((t0 + grp) * 16 + g) * kdim + col;
#pragma unroll
    for (int i = 0; i < kRing; ++i) {
      B::load(wg + (s_lo + i) * B::kCols, a[i]);
      B::load(wg + 8 * kdim + (s_lo + i) * B::kCols, b[i]);
    }
    filled = true;
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  for (uint32_t i = threadIdx.x; i < per; i += blockDim.x) cnt[i] = 0;
  __syncthreads();

  const bool tok_ok = static_cast<uint32_t>(g) < tokens;
  const uint16_t* xrow = xs + (tok_ok ? g : 0) * kdim + col;
  for (uint32_t t = grp; t < owned; t += groups) {
    const uint16_t* wg = W + ((t0 + t) * 16 + g) * kdim + col;  // row g; row g + 8 is 8 kdim further
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    uint64_t s = s_lo;
    if (ring) {
      if (!filled) {
#pragma unroll
        for (int i = 0; i < kRing; ++i) {
          B::load(wg + (s_lo + i) * B::kCols, a[i]);
          B::load(wg + 8 * kdim + (s_lo + i) * B::kCols, b[i]);
        }
      }
      for (; s + kRing < ring_end; s += kRing) {
#pragma unroll
        for (int i = 0; i < kRing; ++i) {
          B::mma(d, a[i], b[i], xrow + (s + i) * B::kCols, tok_ok);
          B::load(wg + (s + kRing + i) * B::kCols, a[i]);
          B::load(wg + 8 * kdim + (s + kRing + i) * B::kCols, b[i]);
        }
      }
#pragma unroll
      for (int i = 0; i < kRing; ++i) {
        B::mma(d, a[i], b[i], xrow + (s + i) * B::kCols, tok_ok);
      }
      filled = false;
      s = ring_end;
    }
    for (; s < s_hi; ++s) {
      uint32_t a1[B::kRegs], b1[B::kRegs];
      B::load(wg + s * B::kCols, a1);
      B::load(wg + 8 * kdim + s * B::kCols, b1);
      B::mma(d, a1, b1, xrow + s * B::kCols, tok_ok);
    }
    if (rest32) {  // columns blocks * 64 .. + 31 as one 16-byte-piece block (thread columns 8q .. 8q+7)
      using R = MmaBlock<false>;
      const uint64_t c0 = blocks * 64 + 8 * q;
      const uint16_t* wt = W + ((t0 + t) * 16 + g) * kdim + c0;
      uint32_t a1[R::kRegs], b1[R::kRegs];
      R::load(wt, a1);
      R::load(wt + 8 * kdim, b1);
      R::mma(d, a1, b1, xs + (tok_ok ? g : 0) * kdim + c0, tok_ok);
    }
    // d0, d1: row g, tokens 2q, 2q+1; d2, d3: row g + 8, same tokens
    float* pt = parts + (static_cast<uint64_t>(t) * ks + h) * 128;
    pt[g * 8 + 2 * q] = d[0];
    pt[g * 8 + 2 * q + 1] = d[1];
    pt[(g + 8) * 8 + 2 * q] = d[2];
    pt[(g + 8) * 8 + 2 * q + 1] = d[3];
    __threadfence_block();
    __syncwarp();
    int last = 0;
    if (lane == 0) last = atomicAdd(&cnt[t], 1u) == ks - 1;
    if (__shfl_sync(kFull, last, 0)) {
      // the last of the tile's ks warps: lane 2u + half builds and pushes
      // token u's vector of rows 8 half .. 8 half + 7
      __threadfence_block();
      const uint32_t u = lane >> 1, half = lane & 1;
      if (u < tokens) {
        const volatile float* pv = parts + static_cast<uint64_t>(t) * ks * 128;
        float y[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const uint32_t row = half * 8 + m;
          y[m] = pv[row * 8 + u];
          for (uint32_t j = 1; j < ks; ++j) y[m] += pv[j * 128 + row * 8 + u];
        }
        const uint4 own = make_uint4(pack_rn(y[0], y[1]), pack_rn(y[2], y[3]), pack_rn(y[4], y[5]),
                                     pack_rn(y[6], y[7]));
        ownv[t * 16 + half * 8 + u] = own;
        sfc_device::ll_push(p.view, r, epoch, u * nvec + (t0 + t) * 2 + half, own);
      }
    }
  }
  __syncthreads();  // every vector of the CTA is pushed and its own part stored
  const uint32_t work = owned * 2 * tokens;
  for (uint32_t base = 0; base < work; base += kLinearThreads) {
    const uint32_t i = base + threadIdx.x;
    const bool act = i < work;
    // i = (u * owned + t) * 2 + half
    const uint32_t half = i & 1, ut = i >> 1;
    const uint32_t u = act ? ut / owned : 0, t = act ? ut - u * owned : 0;
    const uint64_t v = (t0 + t) * 2 + half;
    const uint4 own = act ? ownv[t * 16 + half * 8 + u] : make_uint4(0, 0, 0, 0);
    uint4 out;
    if (!sfc_device::ll_allreduce_lane<NR>(p.view, r, epoch, u * nvec + v, act, own, &out)) return;
    if (act) *reinterpret_cast<uint4*>(p.y[r] + u * p.hidden + v * 8) = out;
  }
  if (p.epoch_dev != nullptr && lane == 0)
    finish_device_epoch(p.epoch_dev, p.done_ctr, gridDim.x * (blockDim.x >> 5), epoch + 1);
}

template <int NR>
struct LinearRow {
  static const void* get(uint32_t variant) {
    switch (variant) {
      case kLinearMma16: return reinterpret_cast<const void*>(&linear_mma_kernel<NR, false, 2>);
      case kLinearMma32: return reinterpret_cast<const void*>(&linear_mma_kernel<NR, true, 2>);
      case kLinearMma16 + kLinearMmaOnePerSm:
        return reinterpret_cast<const void*>(&linear_mma_kernel<NR, false, 1>);
      case kLinearMma32 + kLinearMmaOnePerSm:
        return reinterpret_cast<const void*>(&linear_mma_kernel<NR, true, 1>);
      case 1: return reinterpret_cast<const void*>(&linear_allreduce_kernel<NR, 1>);
      case 2: return reinterpret_cast<const void*>(&linear_allreduce_kernel<NR, 2>);
      case 4: return reinterpret_cast<const void*>(&linear_allreduce_kernel<NR, 4>);
      case 8: return reinterpret_cast<const void*>(&linear_allreduce_kernel<NR, 8>);
      default: return nullptr;
    }
  }
};

}  // namespace

const void* linear_kernel_for(int nranks, uint32_t variant) {
  switch (nranks) {
    case 2: return LinearRow<2>::get(variant);
    case 3: return LinearRow<3>::get(variant);
    case 4: return LinearRow<4>::get(variant);
    case 5: return LinearRow<5>::get(variant);
    case 6: return LinearRow<6>::get(variant);
    case 7: return LinearRow<7>::get(variant);
    case 8: return LinearRow<8>::get(variant);
    default: return nullptr;
  }
}

}  // namespace sfc
