// Internal definitions shared by the host runtime and the kernels of libsfc.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "sfc.h"

namespace sfc {

constexpr int kThreads = 256;  // threads per CTA of the collective kernels (launch bound)
constexpr int kHostSegmentsMax = 8;    // host-buffer chains: launches whose copies overlap
constexpr int kHostSegmentMinOps = 16;  // fewest operations per such launch
constexpr int kSmallCtaThreads = 128;      // CTA size for small messages at 4+ ranks
constexpr uint64_t kSmallCtaMaxCount = 32768;  // bf16 per rank (64 KB) up to which it applies
constexpr int kMaxRanks = 8;
constexpr int kMinRanks = 2;

// protocol ids (match sfc_protocol)
enum : int {
  kLL = 1,
  kLL128 = 2,
  kSentinel = 3,
  kOneshot = 4,
  kTwoshot = 5,
  kOneshotDB = 6,
  kLLTwoshot = 7,
  kSentinelTwoshot = 8,
  kLL128Fast = 9,
  kNumProtocols = 10
};
// Internal kernel variant (not a protocol of the API): the sentinel protocol
// polled with loads and reset with stores, launched for large messages.
constexpr int kSentinelLoadPoll = 16;
// (N - 1) x bytes per rank from which the sentinel polls with loads: below
// it one atomic exchange per unit has the lower latency; above it the
// exchanges queue on the L2's atomic units (measured on B200: at 8 ranks
// x 128 KB p50 5.5 -> 3.5 us, p99 15 -> 4 us; at 4 ranks x 16 KB the
// exchange is 0.35 us faster). At 4 ranks x 128 KB, the point itself, the
// loads trade 4 % of p50 (2.18 -> 2.27 us) and 2 % of the mean for a 16 %
// lower p99 (3.1-3.2 -> 2.7 us).
constexpr uint64_t kSentinelLoadPollBytes = 384 * 1024;
inline bool sentinel_load_poll(int n, uint64_t count) {
  return static_cast<uint64_t>(n - 1) * count * 2 >= kSentinelLoadPollBytes;
}

// operations (match sfc_op)
enum : int { kAllreduce = 0, kAllgather = 1 };

// Barrier counter values are (epoch << 2) | phase, monotone over the whole
// epoch sequence, so any protocol mix keeps "flag >= target" meaningful.
enum : uint64_t { kPhaseTop = 1, kPhaseMid = 2, kPhaseBottom = 3 };

// LL128 geometry: a line is 120 data bytes (60 bf16) + an 8-byte flag word;
// a warp moves 4 lines (8 lanes x 16 bytes each) per step.
constexpr int kLL128Elems = 60;
constexpr int kLL128Line = 128;
constexpr int kLL128LinesPerWarp = 4;

// LL geometry: one 16-byte input vector (8 bf16) becomes four 8-byte units
// (2 bf16 + 32-bit epoch each), written as two 16-byte stores. The two halves
// of 32 consecutive vectors are laid out lane-interleaved (512 + 512 bytes)
// so that each warp-wide store covers whole 32-byte sectors.
constexpr int kLLChunkVecs = 32;
constexpr int kLLChunkBytes = 1024;

// Device status block (one per context).
struct DevStatus {
  int code;       // first sfc_status error recorded (0 = none)
  uint32_t info;  // detail: (op << 16) | (rank << 8) | source
  int abort;      // nonzero: every wait and every later kernel exits
  int pad;
};

// Kernel parameters (passed by value as a __grid_constant__).
struct KParams {
  // operand addressing: mode 0 = inline pointers (one operation),
  // 1 = device pointer tables [k * N + r], 2 = strided from a base.
  const uint16_t* in_inline[kMaxRanks];
  uint16_t* out_inline[kMaxRanks];
  const uint16_t* const* in_table;
  uint16_t* const* out_table;
  const uint16_t* in_base;
  uint16_t* out_base;
  uint64_t in_stride;   // elements between consecutive (k, r) inputs
  uint64_t out_stride;  // elements between consecutive (k, r) outputs
  int addr_mode;

  uint64_t count;       // elements per rank (all-gather: per shard)
  int k_ops;            // operations in this launch
  int G;                // CTAs per rank
  uint32_t first_epoch;

  uint8_t* scratch;     // protocol region; slot (recv, parity, j) at
                        // ((recv * 2 + parity) * (N - 1) + j) * slot_stride;
                        // the twoshot protocols keep their all-gather slots
                        // after the 2 * N * (N - 1) reduce-scatter slots
  uint64_t slot_stride; // bytes
  uint64_t scratch_bytes;  // size of the protocol region (debug builds check every access)
  uint64_t* bar;        // barrier counters [N][bar_stride]
  int bar_stride;
  uint16_t* red;        // twoshot reduced shards [N][red_stride]
  uint64_t red_stride;  // elements

  DevStatus* status;
  uint32_t* epoch_dev;  // device-epoch mode: the next epoch (read at start), else null
  uint32_t* done_ctr;   // device-epoch mode: warps finished (the last one advances epoch_dev)
  uint64_t* timings;    // [timing_first + k_ops + 1] or null
  uint32_t timing_first;  // completion of op k is stamped at timings[1 + timing_first + k]
  const uint32_t* skew; // [k_ops * N] ns or null
  uint64_t timeout_ns;
  int debug;
  int silent_rank;      // -1 = none
  int skip_abort_prologue;  // nonzero (single operations of a context): no abort-word load before the first push
};

// Fused row-parallel linear + LL all-reduce (one decode token).
struct LinearParams {
  const uint16_t* W[kMaxRanks];  // [hidden][kdim] row-major, per rank
  const uint16_t* x[kMaxRanks];  // [tokens][kdim], per rank
  uint16_t* y[kMaxRanks];        // [tokens][hidden], per rank
  uint64_t hidden;
  uint64_t kdim;
  uint32_t tokens;               // 1..8; the kernel's token tile T is the next power of two
  int G;                         // CTAs per rank
  uint32_t epoch;
  uint32_t per_cta;              // output vectors per CTA
  uint32_t* epoch_dev;           // device-epoch mode (as in KParams), else null
  uint32_t* done_ctr;
  uint32_t ks;                   // warps that split one vector's columns (1, 2, 4 or 8)
  sfc_ll_view view;
};
constexpr int kLinearThreads = 256;
constexpr int kLinearWarps = kLinearThreads / 32;
constexpr uint32_t kLinearMaxTokens = 8;
// token tile of the fused kernel for a token count: 1, 2, 4 or 8
inline uint32_t linear_token_tile(uint32_t tokens) { return tokens <= 1 ? 1 : tokens <= 2 ? 2 : tokens <= 4 ? 4 : 8; }
// dynamic shared memory of the fused kernel: x (T tokens), per-part sums,
// own vectors, counters
inline size_t linear_smem_bytes(uint64_t kdim, uint32_t T, uint32_t ks, uint32_t per_cta) {
  return kdim * 2 * T + 32ull * ks * T * per_cta + 16ull * T * per_cta + 4ull * per_cta;
}
// The tensor-core kernels (2..8 tokens, 16-row tiles) read each weight row
// as 16-byte pieces (32-column blocks) or as 32-byte pieces (64-column
// blocks; the weights 32-byte aligned).
constexpr uint32_t kLinearMma16 = 0;
constexpr uint32_t kLinearMma32 = 32;
// added to either: one CTA an SM with a ring twice as deep
constexpr uint32_t kLinearMmaOnePerSm = 64;
// shared memory per CTA above which two CTAs an SM give way to one
constexpr size_t kLinearOnePerSmSmemBytes = 96 * 1024;
// tensor-core kernel: x, per-part sums of 16 x 8, own vectors (2 x 8 per
// tile), counters
inline size_t linear_mma_smem_bytes(uint64_t kdim, uint32_t tokens, uint32_t ks, uint32_t per_tiles) {
  return ((tokens * kdim * 2 + 15) & ~15ull) + 512ull * ks * per_tiles + 256ull * per_tiles + 4ull * per_tiles;
}
// variant 1, 2, 4, 8: the CUDA-core kernel of that token tile;
// kLinearMma16 / kLinearMma32 (+ kLinearMmaOnePerSm): a tensor-core kernel
const void* linear_kernel_for(int nranks, uint32_t variant);

// Kernel entry for (nranks, protocol, op); null if not provided.
const void* kernel_for(int nranks, int protocol, int op);
// The kernel a launch of `count` elements per rank uses: kernel_for, or the
// sentinel's load-poll variant for large messages.
const void* launch_kernel_for(int nranks, int protocol, int op, uint64_t count);

// Encoded slot size (bytes) for `count` elements under the GPU layout (the
// twoshot protocols: for one shard of a `count`-element message).
uint64_t slot_bytes_gpu(int protocol, uint64_t count, int n);

// Vectors (8 elements) per shard of a `count`-element message over n ranks.
#ifdef __CUDACC__
__host__ __device__
#endif
inline uint64_t shard_vectors(uint64_t count, int n) { return ((count + 7) / 8 + n - 1) / n; }

}  // namespace sfc
