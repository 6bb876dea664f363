// Host runtime of libsfc: context, argument checks, epoch sequence, scratch
// provisioning, launch shape, cooperative launch, status, selector.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "sfc.h"
#include "sfc_cost_table.h"
#include "sfc_internal.h"

using namespace sfc;

struct sfc_ctx {
  int device = 0;
  int nranks = 0;
  size_t max_bytes = 0;
  uint64_t max_count = 0;
  sfc_config cfg{};
  int sm_count = 0;

  uint8_t* region[kNumProtocols] = {};  // per self-sync protocol scratch
  uint8_t* region_raw[kNumProtocols] = {};  // allocation: guard, region, guard
  uint64_t slot_stride[kNumProtocols] = {};
  uint64_t region_bytes[kNumProtocols] = {};
  uint64_t* bar = nullptr;
  int bar_stride = 0;
  uint16_t* red = nullptr;
  uint64_t red_stride = 0;
  DevStatus* dstatus = nullptr;
  DevStatus* hstatus = nullptr;  // page-locked mirror

  uint32_t next_epoch = 1;
  uint32_t* d_epoch = nullptr;   // device-epoch mode: {next epoch, finished warps} on the device
  uint32_t* h_epoch_init = nullptr;  // page-locked {1, 0}, copied over d_epoch by sfc_reset
  bool poisoned = false;
  int silent_rank = -1;
  cudaStream_t last_stream = nullptr;
  uint64_t launches = 0;
  sfc_cost_model model{};

  int occupancy[kNumProtocols][2][2][2] = {};  // blocks per SM, per (protocol, op, CTA size, kernel
                                               // variant), 0 = unknown
  int forced_protocol = 0;                // SFC_PROTOCOL: what AUTO resolves to (0 = the selector)
  int smem_optin = 0;                     // opt-in shared memory per block (bytes)
  int linear_occ[5] = {};                 // fused-linear CTAs per SM: token tile 1/2/4/8, tensor cores (0 = not queried)
  int linear_occ_one = 0;                 // the one-CTA-per-SM tensor-core kernels: set up (1) or not (0)

  // staging for the host-buffer entry point, and the copy streams and
  // events that overlap its copies with the chain segments
  uint16_t* stage_in = nullptr;
  uint16_t* stage_out = nullptr;
  size_t stage_bytes = 0;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t ev_start = nullptr;
  cudaEvent_t ev_in[kHostSegmentsMax] = {}, ev_run[kHostSegmentsMax] = {}, ev_out[kHostSegmentsMax] = {};
};

namespace {

constexpr uint32_t kDefaultTimeoutUs = 50000;
constexpr uint32_t kAllProtocolsMask = ((1u << kNumProtocols) - 1u) & ~1u;
constexpr int kBarStride = 1024;  // >= any CTAs-per-rank value
constexpr size_t kGuardBytes = 4096;
constexpr int kGuardByte = 0xA5;

bool cuda_ok(cudaError_t e) {
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  return true;
}

bool self_sync(int proto) {
  return proto == kLL || proto == kLL128 || proto == kSentinel || proto == kLLTwoshot || proto == kSentinelTwoshot ||
         proto == kLL128Fast;
}
bool twoshot_alg(int proto) { return proto == kTwoshot || proto == kLLTwoshot || proto == kSentinelTwoshot; }

bool provisioned(const sfc_ctx* c, int proto) {
  const uint32_t mask = c->cfg.protocol_mask ? c->cfg.protocol_mask : kAllProtocolsMask;
  return (mask >> proto) & 1u;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// [a, a + n) and [b, b + m) overlap?
bool overlap(const void* a, size_t n, const void* b, size_t m) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + m && y < x + n;
}

// Threads per CTA for a call. Small messages at 4+ ranks spread the same
// work over twice as many 128-thread CTAs (fewer polls in flight per SM):
// 5-13 % lower latency at 8 ranks and 8-64 KB, equal or better at 4 ranks,
// measured on B200 for LL, sentinel and the one-load LL128. Everything else
// keeps kThreads. A caller-fixed CTA count keeps kThreads too. (64-thread
// CTAs up to 16 KB measured slower at 4 ranks, 4 x 16 KB sentinel 1.70-1.73
// -> 1.79 us, and from 3 % faster to 25 % slower at 8 ranks: not used.)
int cta_threads(const sfc_ctx* c, int proto, uint64_t count) {
  const bool small_msg = c->nranks >= 4 && count <= kSmallCtaMaxCount && c->cfg.ctas_per_rank == 0;
  return small_msg && (proto == kLL || proto == kSentinel || proto == kLL128Fast) ? kSmallCtaThreads : kThreads;
}

int occupancy_of(sfc_ctx* c, int proto, int op, int threads, uint64_t count) {
  const void* fn = launch_kernel_for(c->nranks, proto, op, count);
  const int variant = fn != kernel_for(c->nranks, proto, op) ? 1 : 0;
  int& occ = c->occupancy[proto][op][threads == kThreads ? 0 : 1][variant];
  if (occ == 0) {
    int nb = 0;
    if (fn == nullptr || !cuda_ok(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, threads, 0)))
      return 0;
    occ = nb;
  }
  return occ;
}

// CTAs per rank for a call: enough threads for one unit of work each
// (an 8-element vector, or a 4-line LL128 group per warp), capped so that
// all N * G CTAs are co-resident.
int choose_G(sfc_ctx* c, int proto, int op, uint64_t count, int* gmax_out) {
  const int threads = cta_threads(c, proto, count);
  const int occ = occupancy_of(c, proto, op, threads, count);
  const int gmax = std::min(kBarStride, occ * c->sm_count / c->nranks);
  if (gmax_out) *gmax_out = gmax;
  if (gmax <= 0) return 0;
  if (c->cfg.ctas_per_rank > 0) return c->cfg.ctas_per_rank;
  const uint64_t nvec = (count + 7) / 8;
  uint64_t threads_needed;
  if (proto == kLL128 || proto == kLL128Fast) {
    const uint64_t lines = (count + kLL128Elems - 1) / kLL128Elems;
    threads_needed = (lines + kLL128LinesPerWarp - 1) / kLL128LinesPerWarp * 32;
  } else if (twoshot_alg(proto)) {
    threads_needed = shard_vectors(count, c->nranks);
  } else {
    threads_needed = nvec;
  }
  uint64_t g = (threads_needed + threads - 1) / threads;
  g = std::max<uint64_t>(1, std::min<uint64_t>(g, gmax));
  return static_cast<int>(g);
}

sfc_status check_common(sfc_ctx* c, sfc_op op, size_t count, sfc_dtype dtype, int proto, uint32_t first_epoch,
                        int k_ops) {
  if (c == nullptr || k_ops < 1) return SFC_ERR_INVALID;
  if (dtype != SFC_BF16) return SFC_ERR_UNSUPPORTED;
  if (op != SFC_OP_ALLREDUCE && op != SFC_OP_ALLGATHER) return SFC_ERR_INVALID;
  if (proto < kLL || proto >= kNumProtocols) return SFC_ERR_INVALID;
  if (op == SFC_OP_ALLGATHER && twoshot_alg(proto)) return SFC_ERR_UNSUPPORTED;
  if (!provisioned(c, proto)) return SFC_ERR_UNSUPPORTED;
  if (count > c->max_count) return SFC_ERR_INVALID;
  if (c->poisoned) return SFC_ERR_ABORTED;
  if (c->cfg.device_epochs) return first_epoch == 0 ? SFC_OK : SFC_ERR_EPOCH;  // the kernel checks the range
  // next_epoch is 0 once epoch 2^32 - 1 has been used: the sequence is spent
  // (an epoch of 0 would validate against zero-filled flags) until sfc_reset
  if (first_epoch == 0 || first_epoch != c->next_epoch) return SFC_ERR_EPOCH;
  if (static_cast<uint64_t>(first_epoch) + static_cast<uint64_t>(k_ops) - 1 > 0xFFFFFFFFull) return SFC_ERR_EPOCH;
  return SFC_OK;
}

void fill_common(sfc_ctx* c, KParams& p, int proto, uint64_t count, int k_ops, uint32_t first_epoch, int G) {
  p.count = count;
  p.k_ops = k_ops;
  p.G = G;
  p.first_epoch = first_epoch;
  p.scratch = self_sync(proto) ? c->region[proto] : nullptr;
  p.slot_stride = self_sync(proto) ? c->slot_stride[proto] : 0;
  p.scratch_bytes = self_sync(proto) ? c->region_bytes[proto] : 0;
  p.epoch_dev = c->cfg.device_epochs ? c->d_epoch : nullptr;
  p.done_ctr = c->cfg.device_epochs ? c->d_epoch + 1 : nullptr;
  p.bar = c->bar;
  p.bar_stride = c->bar_stride;
  p.red = c->red;
  p.red_stride = c->red_stride;
  p.status = c->dstatus;
  p.timeout_ns = static_cast<uint64_t>(c->cfg.timeout_us ? c->cfg.timeout_us : kDefaultTimeoutUs) * 1000ull;
  p.debug = c->cfg.debug_checks;
  p.silent_rank = c->silent_rank;
}

sfc_status launch(sfc_ctx* c, int proto, int op, KParams& p, cudaStream_t stream) {
  const void* fn = launch_kernel_for(c->nranks, proto, op, p.count);
  if (fn == nullptr) return SFC_ERR_UNSUPPORTED;
  int gmax = 0;
  (void)choose_G(c, proto, op, p.count, &gmax);
  if (p.G < 1 || p.G > gmax) return SFC_ERR_RESOURCES;
  void* args[] = {&p};
  const int threads = cta_threads(c, proto, p.count);
  cudaError_t e = cudaLaunchCooperativeKernel(fn, dim3(c->nranks * p.G), dim3(threads), args, 0, stream);
  if (e == cudaErrorCooperativeLaunchTooLarge) {
    (void)cudaGetLastError();
    return SFC_ERR_RESOURCES;
  }
  if (!cuda_ok(e)) return SFC_ERR_CUDA;
  c->launches++;
  c->last_stream = stream;
  return SFC_OK;
}

sfc_status prepare_timings(uint64_t* timings, int k_ops, cudaStream_t stream) {
  if (timings == nullptr) return SFC_OK;
  if (!cuda_ok(cudaMemsetAsync(timings, 0xFF, sizeof(uint64_t), stream))) return SFC_ERR_CUDA;
  if (!cuda_ok(cudaMemsetAsync(timings + 1, 0, sizeof(uint64_t) * k_ops, stream))) return SFC_ERR_CUDA;
  return SFC_OK;
}

// Epoch 0 is never a valid epoch; callers pass it for "the next one".
// (In device-epoch mode 0 stays 0: the kernel reads the epoch.)
uint32_t resolve_epoch(const sfc_ctx* c, uint32_t e) { return e == 0 && !c->cfg.device_epochs ? c->next_epoch : e; }

// Operand checks of a single operation (pointers, alignment, no overlap).
sfc_status check_operands(const sfc_ctx* c, sfc_op op, const void* const* in, void* const* out, size_t count) {
  const int N = c->nranks;
  const size_t in_bytes = count * 2;
  const size_t out_bytes = (op == SFC_OP_ALLGATHER ? N : 1) * count * 2;
  for (int r = 0; r < N; ++r) {
    if (in[r] == nullptr || out[r] == nullptr || !aligned16(in[r]) || !aligned16(out[r])) return SFC_ERR_INVALID;
  }
  for (int a = 0; a < N; ++a) {
    for (int b = 0; b < N; ++b) {
      if (overlap(in[a], in_bytes, out[b], out_bytes)) return SFC_ERR_INVALID;
      if (a < b && overlap(out[a], out_bytes, out[b], out_bytes)) return SFC_ERR_INVALID;
    }
  }
  return SFC_OK;
}

sfc_status one_op(sfc_ctx* c, sfc_op op, const void* const* in, void* const* out, size_t count, sfc_dtype dtype,
                  sfc_protocol protocol, uint32_t epoch, void* stream) {
  if (c == nullptr || in == nullptr || out == nullptr) return SFC_ERR_INVALID;
  epoch = resolve_epoch(c, epoch);
  if (count == 0) return (dtype == SFC_BF16) ? SFC_OK : SFC_ERR_UNSUPPORTED;
  int proto = protocol;
  if (proto == SFC_PROTO_AUTO) proto = sfc_select_protocol(c, op, count * 2, c->nranks);
  sfc_status s = check_common(c, op, count, dtype, proto, epoch, 1);
  if (s != SFC_OK) return s;
  s = check_operands(c, op, in, out, count);
  if (s != SFC_OK) return s;
  const int N = c->nranks;
  KParams p{};
  for (int r = 0; r < N; ++r) {
    p.in_inline[r] = static_cast<const uint16_t*>(in[r]);
    p.out_inline[r] = static_cast<uint16_t*>(out[r]);
  }
  p.addr_mode = 0;
  const int G = choose_G(c, proto, op, count, nullptr);
  fill_common(c, p, proto, count, 1, epoch, G);
  p.skip_abort_prologue = 1;
  s = launch(c, proto, op, p, static_cast<cudaStream_t>(stream));
  if (s == SFC_OK && !c->cfg.device_epochs) c->next_epoch = epoch + 1;
  return s;
}

sfc_status chain(sfc_ctx* c, sfc_op op, int k_ops, const void* const* in_table, void* const* out_table, size_t count,
                 sfc_dtype dtype, sfc_protocol protocol, uint32_t first_epoch, const uint32_t* skew_ns,
                 uint64_t* timings, void* stream) {
  if (c == nullptr || in_table == nullptr || out_table == nullptr) return SFC_ERR_INVALID;
  first_epoch = resolve_epoch(c, first_epoch);
  if (count == 0) return (dtype == SFC_BF16 && k_ops >= 1) ? SFC_OK : SFC_ERR_INVALID;
  int proto = protocol;
  if (proto == SFC_PROTO_AUTO) proto = sfc_select_protocol(c, op, count * 2, c->nranks);
  sfc_status s = check_common(c, op, count, dtype, proto, first_epoch, k_ops);
  if (s != SFC_OK) return s;
  if ((reinterpret_cast<uintptr_t>(in_table) | reinterpret_cast<uintptr_t>(out_table)) & 7u) return SFC_ERR_INVALID;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  s = prepare_timings(timings, k_ops, st);
  if (s != SFC_OK) return s;
  KParams p{};
  p.addr_mode = 1;
  p.in_table = reinterpret_cast<const uint16_t* const*>(in_table);
  p.out_table = reinterpret_cast<uint16_t* const*>(out_table);
  p.skew = skew_ns;
  p.timings = timings;
  const int G = choose_G(c, proto, op, count, nullptr);
  fill_common(c, p, proto, count, k_ops, first_epoch, G);
  s = launch(c, proto, op, p, st);
  if (s == SFC_OK && !c->cfg.device_epochs) c->next_epoch = first_epoch + static_cast<uint32_t>(k_ops);
  return s;
}

// Environment overrides, read once per context:
//   SFC_TIMEOUT_MS  bound on every device wait (ms, > 0), used when the
//                   config leaves timeout_us at 0;
//   SFC_PROTOCOL    the protocol AUTO resolves to (a name as in the Python
//                   binding, e.g. "sentinel", or its number), wherever that
//                   protocol is provisioned and supports the operation.
// Unparsable values are ignored.
void apply_env_overrides(sfc_ctx* c) {
  if (const char* t = std::getenv("SFC_TIMEOUT_MS")) {
    char* end = nullptr;
    const long ms = std::strtol(t, &end, 10);
    if (end != t && *end == '\0' && ms > 0 && ms <= 4000000 && c->cfg.timeout_us == 0)
      c->cfg.timeout_us = static_cast<uint32_t>(ms * 1000);
  }
  if (const char* pstr = std::getenv("SFC_PROTOCOL")) {
    static const char* const names[kNumProtocols] = {"auto",       "ll",          "ll128",
                                                     "sentinel",   "barrier_oneshot", "barrier_twoshot",
                                                     "barrier_oneshot_db", "ll_twoshot", "sentinel_twoshot",
                                                     "ll128_fast"};
    int f = 0;
    for (int i = 1; i < kNumProtocols; ++i)
      if (std::strcmp(pstr, names[i]) == 0) f = i;
    char* end = nullptr;
    const long v = std::strtol(pstr, &end, 10);
    if (f == 0 && end != pstr && *end == '\0' && v > 0 && v < kNumProtocols) f = static_cast<int>(v);
    c->forced_protocol = f;
  }
}

// Built-in latency model: the p50 latencies the message-size sweep measured
// on a B200 (sfc_cost_table.h); every protocol with a kernel is available.
void builtin_model(sfc_cost_model* m) {
  std::memset(m, 0, sizeof(*m));
  for (int op = 0; op < 2; ++op)
    for (int pr = 0; pr < SFC_NUM_PROTOCOLS; ++pr)
      for (int n = 0; n <= SFC_MAX_RANKS; ++n) {
        sfc_cost_entry& e = m->c[op][pr][n];
        bool measured = false;
        for (int i = 0; i < SFC_COST_BUCKETS; ++i) {
          e.table_us[i] = pr < kCostProtocols ? kMeasuredP50Us[op][pr][n][i] : -1.0;
          measured = measured || e.table_us[i] > 0;
        }
        // a protocol the sweep did not measure is never chosen by default, nor
        // is the opt-in one-load LL128
        const bool exists = pr >= kLL && pr != kLL128Fast && n >= kMinRanks &&
                            !(op == SFC_OP_ALLGATHER && twoshot_alg(pr));
        e.alpha_us = exists && measured ? 0.0 : -1.0;
        e.beta_us_per_byte = 0.0;
      }
}

}  // namespace

// ============================================================== public API
extern "C" {

const char* sfc_status_string(sfc_status s) {
  switch (s) {
    case SFC_OK: return "ok";
    case SFC_ERR_INVALID: return "invalid argument";
    case SFC_ERR_CUDA: return "CUDA runtime error";
    case SFC_ERR_TIMEOUT: return "device wait timed out";
    case SFC_ERR_EPOCH: return "epoch is not the next one";
    case SFC_ERR_RESOURCES: return "ranks' CTAs cannot all be co-resident";
    case SFC_ERR_SENTINEL_IN_INPUT: return "input contains the sentinel pattern";
    case SFC_ERR_UNSUPPORTED: return "unsupported protocol, operation or dtype";
    case SFC_ERR_ABORTED: return "context aborted by an earlier device error";
    case SFC_ERR_GUARD: return "a scratch guard word was overwritten";
  }
  return "unknown status";
}

double sfc_algorithmic_bytes(sfc_op op, sfc_protocol protocol, size_t count, int nranks) {
  if (nranks < kMinRanks || nranks > kMaxRanks || (op != 0 && op != 1)) return -1.0;
  const double n = nranks;
  const double s = 2.0 * static_cast<double>(count);
  const size_t shard = (count + nranks - 1) / nranks;  // elements per twoshot shard
  auto ll_enc = [](size_t c) { return 8.0 * static_cast<double>((c + 1) / 2); };
  switch (protocol) {
    case SFC_PROTO_LL:
    case SFC_PROTO_LL128:
    case SFC_PROTO_LL128_FAST:
    case SFC_PROTO_SENTINEL: {
      double enc = s;
      if (protocol == SFC_PROTO_LL) enc = ll_enc(count);
      if (protocol == SFC_PROTO_LL128 || protocol == SFC_PROTO_LL128_FAST)
        enc = 128.0 * static_cast<double>((count + kLL128Elems - 1) / kLL128Elems);
      const double reset = protocol == SFC_PROTO_SENTINEL ? (n - 1) * s : 0.0;
      const double written = op == SFC_OP_ALLREDUCE ? s : n * s;
      return n * (s + 2.0 * (n - 1) * enc + written + reset);
    }
    case SFC_PROTO_BARRIER_ONESHOT:
    case SFC_PROTO_BARRIER_ONESHOT_DB:
      return op == SFC_OP_ALLREDUCE ? n * (n * s + s) : n * (n * s + n * s);
    case SFC_PROTO_BARRIER_TWOSHOT:
      return op == SFC_OP_ALLREDUCE ? n * (s + s / n + s + s) : -1.0;
    case SFC_PROTO_LL_TWOSHOT:
    case SFC_PROTO_SENTINEL_TWOSHOT: {
      if (op != SFC_OP_ALLREDUCE) return -1.0;
      // read own input, push + poll (N-1) encoded shards in each of the two
      // phases, write the output; the sentinel also rewrites what it consumed
      const double sh = 2.0 * static_cast<double>(shard);
      const double enc = protocol == SFC_PROTO_LL_TWOSHOT ? ll_enc(shard) : sh;
      const double reset = protocol == SFC_PROTO_SENTINEL_TWOSHOT ? 2.0 * (n - 1) * sh : 0.0;
      return n * (s + 4.0 * (n - 1) * enc + s + reset);
    }
    default:
      return -1.0;
  }
}

void sfc_default_cost_model(sfc_cost_model* model) {
  if (model) builtin_model(model);
}

double sfc_cost_estimate(const sfc_cost_model* m, sfc_op op, sfc_protocol protocol, size_t bytes_per_rank,
                         int nranks) {
  if (m == nullptr || (op != 0 && op != 1) || protocol < SFC_PROTO_LL || protocol >= SFC_NUM_PROTOCOLS ||
      nranks < kMinRanks || nranks > kMaxRanks)
    return -1.0;
  const sfc_cost_entry& e = m->c[op][protocol][nranks];
  if (e.alpha_us < 0) return -1.0;
  const size_t count = bytes_per_rank / 2;
  const double bytes = sfc_algorithmic_bytes(op, protocol, count, nranks);
  if (bytes < 0) return -1.0;
  int first = -1, last = -1;
  for (int i = 0; i < SFC_COST_BUCKETS; ++i)
    if (e.table_us[i] > 0) {
      if (first < 0) first = i;
      last = i;
    }
  if (first < 0) return e.alpha_us + e.beta_us_per_byte * bytes;
  const double k = std::log2(static_cast<double>(bytes_per_rank > 0 ? bytes_per_rank : 1)) - SFC_COST_MIN_LOG2;
  if (k <= first) return e.table_us[first];
  if (k >= last) {
    const size_t ref = (static_cast<size_t>(1) << (SFC_COST_MIN_LOG2 + last)) / 2;
    const double ref_bytes = sfc_algorithmic_bytes(op, protocol, ref, nranks);
    return e.table_us[last] * (ref_bytes > 0 ? bytes / ref_bytes : 1.0);
  }
  int lo = static_cast<int>(std::floor(k));
  while (lo > first && !(e.table_us[lo] > 0)) --lo;
  int hi = static_cast<int>(std::ceil(k));
  while (hi < last && !(e.table_us[hi] > 0)) ++hi;
  if (hi == lo) return e.table_us[lo];
  return e.table_us[lo] + (e.table_us[hi] - e.table_us[lo]) * (k - lo) / (hi - lo);
}

sfc_protocol sfc_select_protocol_model(const sfc_cost_model* m, sfc_op op, size_t bytes_per_rank, int nranks) {
  static const int order[9] = {SFC_PROTO_SENTINEL,         SFC_PROTO_LL128,
                               SFC_PROTO_LL128_FAST,       SFC_PROTO_LL,
                               SFC_PROTO_SENTINEL_TWOSHOT, SFC_PROTO_LL_TWOSHOT,
                               SFC_PROTO_BARRIER_ONESHOT_DB, SFC_PROTO_BARRIER_ONESHOT,
                               SFC_PROTO_BARRIER_TWOSHOT};
  if (m == nullptr || nranks < kMinRanks || nranks > kMaxRanks || (op != 0 && op != 1)) return SFC_PROTO_AUTO;
  const size_t count = bytes_per_rank / 2;
  int best = SFC_PROTO_AUTO;
  double best_t = 0, best_b = 0;
  for (int i = 0; i < 9; ++i) {
    const int pr = order[i];
    const double t = sfc_cost_estimate(m, op, static_cast<sfc_protocol>(pr), bytes_per_rank, nranks);
    if (t < 0) continue;
    const double b = sfc_algorithmic_bytes(op, static_cast<sfc_protocol>(pr), count, nranks);
    if (best == SFC_PROTO_AUTO || t < best_t || (t == best_t && b < best_b)) {
      best = pr;
      best_t = t;
      best_b = b;
    }
  }
  return static_cast<sfc_protocol>(best);
}

sfc_protocol sfc_select_protocol(const sfc_ctx* c, sfc_op op, size_t bytes_per_rank, int nranks) {
  if (c == nullptr) return SFC_PROTO_AUTO;
  const int f = c->forced_protocol;
  if (f != 0 && provisioned(c, f) && !(op == SFC_OP_ALLGATHER && twoshot_alg(f))) return static_cast<sfc_protocol>(f);
  sfc_cost_model m = c->model;
  // protocols without scratch in this context are never chosen
  for (int pr = 1; pr < SFC_NUM_PROTOCOLS; ++pr)
    if (!provisioned(c, pr))
      for (int o = 0; o < 2; ++o)
        for (int n = 0; n <= SFC_MAX_RANKS; ++n) m.c[o][pr][n].alpha_us = -1.0;
  return sfc_select_protocol_model(&m, op, bytes_per_rank, nranks);
}

sfc_status sfc_set_cost_model(sfc_ctx* c, const sfc_cost_model* m) {
  if (c == nullptr || m == nullptr) return SFC_ERR_INVALID;
  c->model = *m;
  return SFC_OK;
}

sfc_status sfc_init(sfc_ctx** out, int nranks, size_t max_bytes_per_rank, const sfc_config* cfg) {
  if (out == nullptr) return SFC_ERR_INVALID;
  *out = nullptr;
  if (nranks < kMinRanks || nranks > kMaxRanks || max_bytes_per_rank == 0) return SFC_ERR_INVALID;
  if (cfg && (cfg->ctas_per_rank < 0 || cfg->ctas_per_rank > kBarStride)) return SFC_ERR_INVALID;
  if (cfg && (cfg->protocol_mask & ~kAllProtocolsMask)) return SFC_ERR_INVALID;
  sfc_ctx* c = new sfc_ctx();
  if (cfg) c->cfg = *cfg;
  apply_env_overrides(c);
  c->nranks = nranks;
  c->max_bytes = max_bytes_per_rank;
  c->max_count = max_bytes_per_rank / 2;
  builtin_model(&c->model);
  auto fail = [&](sfc_status s) {
    sfc_destroy(c);
    return s;
  };
  if (!cuda_ok(cudaGetDevice(&c->device))) return fail(SFC_ERR_CUDA);
  if (!cuda_ok(cudaDeviceGetAttribute(&c->sm_count, cudaDevAttrMultiProcessorCount, c->device)))
    return fail(SFC_ERR_CUDA);
  if (!cuda_ok(cudaDeviceGetAttribute(&c->smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, c->device)))
    return fail(SFC_ERR_CUDA);
  int coop = 0;
  if (!cuda_ok(cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, c->device)) || !coop)
    return fail(SFC_ERR_UNSUPPORTED);
  const uint64_t slots = static_cast<uint64_t>(nranks) * 2 * (nranks - 1);
  for (int pr : {kLL, kLL128, kSentinel, kLLTwoshot, kSentinelTwoshot, kLL128Fast}) {
    if (!provisioned(c, pr)) continue;
    const uint64_t sb = (slot_bytes_gpu(pr, c->max_count, nranks) + 255) / 256 * 256;
    c->slot_stride[pr] = sb;
    // twoshot: reduce-scatter slots, then as many all-gather slots
    c->region_bytes[pr] = sb * slots * (pr == kLLTwoshot || pr == kSentinelTwoshot ? 2 : 1);
    // guard words before and after the region catch any write out of it
    uint8_t* raw = nullptr;
    if (!cuda_ok(cudaMalloc(&raw, c->region_bytes[pr] + 2 * kGuardBytes))) return fail(SFC_ERR_CUDA);
    c->region_raw[pr] = raw;
    c->region[pr] = raw + kGuardBytes;
    if (!cuda_ok(cudaMemset(raw, kGuardByte, kGuardBytes)) ||
        !cuda_ok(cudaMemset(raw + kGuardBytes + c->region_bytes[pr], kGuardByte, kGuardBytes)))
      return fail(SFC_ERR_CUDA);
  }
  c->bar_stride = kBarStride;
  if (!cuda_ok(cudaMalloc(&c->bar, sizeof(uint64_t) * nranks * kBarStride))) return fail(SFC_ERR_CUDA);
  if (provisioned(c, kTwoshot)) {
    const uint64_t nvec = (c->max_count + 7) / 8;
    c->red_stride = ((nvec + nranks - 1) / nranks) * 8;
    if (!cuda_ok(cudaMalloc(&c->red, std::max<uint64_t>(16, 2 * c->red_stride * nranks) /* bytes */))) return fail(SFC_ERR_CUDA);
  }
  if (!cuda_ok(cudaMalloc(&c->dstatus, sizeof(DevStatus)))) return fail(SFC_ERR_CUDA);
  if (!cuda_ok(cudaMallocHost(&c->hstatus, sizeof(DevStatus)))) return fail(SFC_ERR_CUDA);
  if (!cuda_ok(cudaMalloc(&c->d_epoch, 2 * sizeof(uint32_t))) ||
      !cuda_ok(cudaMallocHost(&c->h_epoch_init, 2 * sizeof(uint32_t))))
    return fail(SFC_ERR_CUDA);
  c->h_epoch_init[0] = 1;
  c->h_epoch_init[1] = 0;
  sfc_status s = sfc_reset(c, nullptr);
  if (s != SFC_OK) return fail(s);
  if (!cuda_ok(cudaStreamSynchronize(nullptr))) return fail(SFC_ERR_CUDA);
  *out = c;
  return SFC_OK;
}

sfc_status sfc_destroy(sfc_ctx* c) {
  if (c == nullptr) return SFC_ERR_INVALID;
  (void)cudaDeviceSynchronize();
  for (int pr = 0; pr < kNumProtocols; ++pr) {
    if (c->region_raw[pr]) cudaFree(c->region_raw[pr]);
    c->region_raw[pr] = nullptr;
    c->region[pr] = nullptr;
  }
  if (c->bar) cudaFree(c->bar);
  if (c->red) cudaFree(c->red);
  if (c->dstatus) cudaFree(c->dstatus);
  if (c->hstatus) cudaFreeHost(c->hstatus);
  if (c->d_epoch) cudaFree(c->d_epoch);
  if (c->h_epoch_init) cudaFreeHost(c->h_epoch_init);
  if (c->stage_in) cudaFree(c->stage_in);
  if (c->stage_out) cudaFree(c->stage_out);
  if (c->h2d) cudaStreamDestroy(c->h2d);
  if (c->d2h) cudaStreamDestroy(c->d2h);
  if (c->ev_start) cudaEventDestroy(c->ev_start);
  for (int i = 0; i < kHostSegmentsMax; ++i)
    for (cudaEvent_t ev : {c->ev_in[i], c->ev_run[i], c->ev_out[i]})
      if (ev) cudaEventDestroy(ev);
  delete c;
  return SFC_OK;
}

sfc_status sfc_reset(sfc_ctx* c, void* stream) {
  if (c == nullptr) return SFC_ERR_INVALID;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int pr : {kLL, kLL128, kSentinel, kLLTwoshot, kSentinelTwoshot, kLL128Fast}) {
    if (c->region[pr] == nullptr) continue;
    const int fill = (pr == kSentinel || pr == kSentinelTwoshot) ? 0xFF : 0x00;
    if (!cuda_ok(cudaMemsetAsync(c->region[pr], fill, c->region_bytes[pr], st))) return SFC_ERR_CUDA;
  }
  if (!cuda_ok(cudaMemsetAsync(c->bar, 0, sizeof(uint64_t) * c->nranks * c->bar_stride, st))) return SFC_ERR_CUDA;
  if (!cuda_ok(cudaMemsetAsync(c->dstatus, 0, sizeof(DevStatus), st))) return SFC_ERR_CUDA;
  if (!cuda_ok(cudaMemcpyAsync(c->d_epoch, c->h_epoch_init, 2 * sizeof(uint32_t), cudaMemcpyHostToDevice, st)))
    return SFC_ERR_CUDA;
  c->next_epoch = 1;
  c->poisoned = false;
  c->last_stream = st;
  return SFC_OK;
}

sfc_status sfc_allreduce(sfc_ctx* c, const void* const* in, void* const* out, size_t count, sfc_dtype dtype,
                         sfc_protocol protocol, uint32_t epoch, void* stream) {
  return one_op(c, SFC_OP_ALLREDUCE, in, out, count, dtype, protocol, epoch, stream);
}

sfc_status sfc_allgather(sfc_ctx* c, const void* const* in, void* const* out, size_t count, sfc_dtype dtype,
                         sfc_protocol protocol, uint32_t epoch, void* stream) {
  return one_op(c, SFC_OP_ALLGATHER, in, out, count, dtype, protocol, epoch, stream);
}

// A prepared single operation: checks, protocol, kernel and launch shape
// fixed once; a launch only takes the next epoch and launches.
struct sfc_plan {
  sfc_ctx* c = nullptr;
  const void* fn = nullptr;
  int grid = 0;
  int block = 0;
  KParams p{};
};

sfc_status sfc_plan_create(sfc_ctx* c, sfc_op op, const void* const* in, void* const* out, size_t count,
                           sfc_dtype dtype, sfc_protocol protocol, sfc_plan** plan) {
  if (plan == nullptr) return SFC_ERR_INVALID;
  *plan = nullptr;
  if (c == nullptr || in == nullptr || out == nullptr || count == 0) return SFC_ERR_INVALID;
  int proto = protocol;
  if (proto == SFC_PROTO_AUTO) proto = sfc_select_protocol(c, op, count * 2, c->nranks);
  sfc_status s = check_common(c, op, count, dtype, proto, c->cfg.device_epochs ? 0 : c->next_epoch, 1);
  if (s != SFC_OK) return s;
  s = check_operands(c, op, in, out, count);
  if (s != SFC_OK) return s;
  const void* fn = launch_kernel_for(c->nranks, proto, op, count);
  if (fn == nullptr) return SFC_ERR_UNSUPPORTED;
  int gmax = 0;
  const int G = choose_G(c, proto, op, count, &gmax);
  if (G < 1 || G > gmax) return SFC_ERR_RESOURCES;
  sfc_plan* pl = new (std::nothrow) sfc_plan();
  if (pl == nullptr) return SFC_ERR_RESOURCES;
  pl->c = c;
  pl->fn = fn;
  pl->grid = c->nranks * G;
  pl->block = cta_threads(c, proto, count);
  for (int r = 0; r < c->nranks; ++r) {
    pl->p.in_inline[r] = static_cast<const uint16_t*>(in[r]);
    pl->p.out_inline[r] = static_cast<uint16_t*>(out[r]);
  }
  pl->p.addr_mode = 0;
  fill_common(c, pl->p, proto, count, 1, 0, G);
  pl->p.skip_abort_prologue = 1;
  *plan = pl;
  return SFC_OK;
}

sfc_status sfc_plan_launch(sfc_plan* pl, void* stream) {
  if (pl == nullptr) return SFC_ERR_INVALID;
  sfc_ctx* c = pl->c;
  if (c->poisoned) return SFC_ERR_ABORTED;
  uint32_t e = 0;
  if (!c->cfg.device_epochs) {
    e = c->next_epoch;
    if (e == 0) return SFC_ERR_EPOCH;  // the sequence is spent: sfc_reset first
  }
  pl->p.first_epoch = e;
  pl->p.silent_rank = c->silent_rank;
  void* args[] = {&pl->p};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t err = cudaLaunchCooperativeKernel(pl->fn, dim3(pl->grid), dim3(pl->block), args, 0, st);
  if (err == cudaErrorCooperativeLaunchTooLarge) {
    (void)cudaGetLastError();
    return SFC_ERR_RESOURCES;
  }
  if (!cuda_ok(err)) return SFC_ERR_CUDA;
  c->launches++;
  c->last_stream = st;
  if (!c->cfg.device_epochs) c->next_epoch = e + 1;
  return SFC_OK;
}

sfc_status sfc_plan_destroy(sfc_plan* pl) {
  delete pl;
  return SFC_OK;
}

sfc_status sfc_allreduce_chain(sfc_ctx* c, int k_ops, const void* const* in_table, void* const* out_table,
                               size_t count, sfc_dtype dtype, sfc_protocol protocol, uint32_t first_epoch,
                               const uint32_t* skew_ns, uint64_t* timings, void* stream) {
  return chain(c, SFC_OP_ALLREDUCE, k_ops, in_table, out_table, count, dtype, protocol, first_epoch, skew_ns,
               timings, stream);
}

sfc_status sfc_allgather_chain(sfc_ctx* c, int k_ops, const void* const* in_table, void* const* out_table,
                               size_t count, sfc_dtype dtype, sfc_protocol protocol, uint32_t first_epoch,
                               const uint32_t* skew_ns, uint64_t* timings, void* stream) {
  return chain(c, SFC_OP_ALLGATHER, k_ops, in_table, out_table, count, dtype, protocol, first_epoch, skew_ns,
               timings, stream);
}

sfc_status sfc_allreduce_chain_host(sfc_ctx* c, int k_ops, const void* in_host, void* out_host, size_t count,
                                    sfc_dtype dtype, sfc_protocol protocol, uint32_t first_epoch, uint64_t* timings,
                                    void* stream) {
  if (c == nullptr || in_host == nullptr || out_host == nullptr || k_ops < 1) return SFC_ERR_INVALID;
  first_epoch = resolve_epoch(c, first_epoch);
  if (count == 0) return dtype == SFC_BF16 ? SFC_OK : SFC_ERR_UNSUPPORTED;
  int proto = protocol;
  if (proto == SFC_PROTO_AUTO) proto = sfc_select_protocol(c, SFC_OP_ALLREDUCE, count * 2, c->nranks);
  sfc_status s = check_common(c, SFC_OP_ALLREDUCE, count, dtype, proto, first_epoch, k_ops);
  if (s != SFC_OK) return s;
  const uint64_t stride = (count + 7) / 8 * 8;  // keep every operand 16-byte aligned
  const size_t need = static_cast<size_t>(k_ops) * c->nranks * stride * 2;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (need > c->stage_bytes) {
    if (c->stage_in || c->stage_out) {
      // every earlier copy was joined into the caller's stream it was issued on
      if (!cuda_ok(cudaDeviceSynchronize())) return SFC_ERR_CUDA;
      cudaFree(c->stage_in);
      cudaFree(c->stage_out);
      c->stage_in = c->stage_out = nullptr;
      c->stage_bytes = 0;
    }
    if (!cuda_ok(cudaMalloc(&c->stage_in, need)) || !cuda_ok(cudaMalloc(&c->stage_out, need))) return SFC_ERR_CUDA;
    c->stage_bytes = need;
  }
  if (c->h2d == nullptr) {
    if (!cuda_ok(cudaStreamCreateWithFlags(&c->h2d, cudaStreamNonBlocking)) ||
        !cuda_ok(cudaStreamCreateWithFlags(&c->d2h, cudaStreamNonBlocking)) ||
        !cuda_ok(cudaEventCreateWithFlags(&c->ev_start, cudaEventDisableTiming)))
      return SFC_ERR_CUDA;
    for (int i = 0; i < kHostSegmentsMax; ++i)
      if (!cuda_ok(cudaEventCreateWithFlags(&c->ev_in[i], cudaEventDisableTiming)) ||
          !cuda_ok(cudaEventCreateWithFlags(&c->ev_run[i], cudaEventDisableTiming)) ||
          !cuda_ok(cudaEventCreateWithFlags(&c->ev_out[i], cudaEventDisableTiming)))
        return SFC_ERR_CUDA;
  }
  s = prepare_timings(timings, k_ops, st);
  if (s != SFC_OK) return s;
  const int G = choose_G(c, proto, SFC_OP_ALLREDUCE, count, nullptr);
  // The chain runs as `nseg` consecutive launches of consecutive operations.
  // All input copies are queued first on the h2d stream (a cooperative
  // launch can hold the host until the device starts it, so queuing them
  // between launches would delay them); segment j waits only for its own
  // inputs, and its outputs are copied out on the d2h stream while segment
  // j+1 runs. The caller's stream finally waits for the last output copy, so
  // the call is ordered on `stream` like any other.
  const int nseg = std::max(1, std::min(kHostSegmentsMax, k_ops / kHostSegmentMinOps));
  const size_t row_dev = stride * 2, row_host = count * 2;
  auto seg_rows = [&](int j, size_t* row0, size_t* rows) {
    const int64_t a = static_cast<int64_t>(k_ops) * j / nseg, b = static_cast<int64_t>(k_ops) * (j + 1) / nseg;
    *row0 = static_cast<size_t>(a) * c->nranks;
    *rows = static_cast<size_t>(b - a) * c->nranks;
    return static_cast<int>(a);
  };
  // one flat copy when host and device rows have the same pitch
  auto copy = [&](void* dst, size_t dpitch, const void* src, size_t spitch, size_t rows, cudaMemcpyKind kind,
                  cudaStream_t cs) {
    if (dpitch == spitch) return cuda_ok(cudaMemcpyAsync(dst, src, rows * row_host, kind, cs));
    return cuda_ok(cudaMemcpy2DAsync(dst, dpitch, src, spitch, row_host, rows, kind, cs));
  };
  if (!cuda_ok(cudaEventRecord(c->ev_start, st)) || !cuda_ok(cudaStreamWaitEvent(c->h2d, c->ev_start, 0)))
    return SFC_ERR_CUDA;
  for (int j = 0; j < nseg; ++j) {
    size_t row0, rows;
    (void)seg_rows(j, &row0, &rows);
    if (!copy(c->stage_in + row0 * stride, row_dev, static_cast<const uint8_t*>(in_host) + row0 * row_host, row_host,
              rows, cudaMemcpyHostToDevice, c->h2d) ||
        !cuda_ok(cudaEventRecord(c->ev_in[j], c->h2d)))
      return SFC_ERR_CUDA;
  }
  for (int j = 0; j < nseg; ++j) {
    size_t row0, rows;
    const int a = seg_rows(j, &row0, &rows);
    const int kj = static_cast<int>(rows / c->nranks);
    if (!cuda_ok(cudaStreamWaitEvent(st, c->ev_in[j], 0))) return SFC_ERR_CUDA;
    KParams p{};
    p.addr_mode = 2;
    p.in_base = c->stage_in + row0 * stride;
    p.out_base = c->stage_out + row0 * stride;
    p.in_stride = stride;
    p.out_stride = stride;
    p.timings = timings;
    p.timing_first = static_cast<uint32_t>(a);
    fill_common(c, p, proto, count, kj, first_epoch + static_cast<uint32_t>(a), G);
    s = launch(c, proto, SFC_OP_ALLREDUCE, p, st);
    if (s != SFC_OK) return s;
    if (!c->cfg.device_epochs) c->next_epoch = first_epoch + static_cast<uint32_t>(a + kj);
    if (!cuda_ok(cudaEventRecord(c->ev_run[j], st)) || !cuda_ok(cudaStreamWaitEvent(c->d2h, c->ev_run[j], 0)) ||
        !copy(static_cast<uint8_t*>(out_host) + row0 * row_host, row_host, c->stage_out + row0 * stride, row_dev,
              rows, cudaMemcpyDeviceToHost, c->d2h) ||
        !cuda_ok(cudaEventRecord(c->ev_out[j], c->d2h)))
      return SFC_ERR_CUDA;
  }
  if (!cuda_ok(cudaStreamWaitEvent(st, c->ev_out[nseg - 1], 0))) return SFC_ERR_CUDA;
  return SFC_OK;
}

sfc_status sfc_get_status(sfc_ctx* c, uint32_t* info) {
  if (c == nullptr) return SFC_ERR_INVALID;
  if (!cuda_ok(cudaMemcpyAsync(c->hstatus, c->dstatus, sizeof(DevStatus), cudaMemcpyDeviceToHost, c->last_stream)))
    return SFC_ERR_CUDA;
  if (!cuda_ok(cudaStreamSynchronize(c->last_stream))) return SFC_ERR_CUDA;
  if (info) *info = c->hstatus->info;
  const int code = c->hstatus->code;
  if (code != 0 || c->hstatus->abort) c->poisoned = true;
  if (code == 0 && c->hstatus->abort) return SFC_ERR_ABORTED;
  return static_cast<sfc_status>(code);
}

uint32_t sfc_next_epoch(const sfc_ctx* c) { return c && !c->cfg.device_epochs ? c->next_epoch : 0; }

sfc_status sfc_launch_shape(sfc_ctx* c, sfc_op op, sfc_protocol protocol, size_t count, int* ctas_per_rank,
                            int* threads_per_cta) {
  if (c == nullptr || (op != 0 && op != 1)) return SFC_ERR_INVALID;
  int proto = protocol;
  if (proto == SFC_PROTO_AUTO) proto = sfc_select_protocol(c, op, count * 2, c->nranks);
  if (proto < kLL || proto >= kNumProtocols) return SFC_ERR_INVALID;
  if (kernel_for(c->nranks, proto, op) == nullptr) return SFC_ERR_UNSUPPORTED;
  const int G = choose_G(c, proto, op, count, nullptr);
  if (G <= 0) return SFC_ERR_RESOURCES;
  if (ctas_per_rank) *ctas_per_rank = G;
  if (threads_per_cta) *threads_per_cta = cta_threads(c, proto, count);
  return SFC_OK;
}

sfc_status sfc_scratch_slot(sfc_ctx* c, sfc_protocol protocol, int rank, int parity, int src, void** ptr,
                            size_t* bytes) {
  if (c == nullptr || ptr == nullptr) return SFC_ERR_INVALID;
  const int pr = protocol;
  if (!self_sync(pr) || c->region[pr] == nullptr) return SFC_ERR_UNSUPPORTED;
  const bool two = pr == kLLTwoshot || pr == kSentinelTwoshot;
  if (rank < 0 || rank >= c->nranks || src < 0 || src >= c->nranks || src == rank || parity < 0 ||
      parity > (two ? 3 : 1))
    return SFC_ERR_INVALID;
  const int j = src < rank ? src : src - 1;
  uint64_t idx = static_cast<uint64_t>((rank * 2 + (parity & 1)) * (c->nranks - 1) + j);
  if (parity >= 2) idx += static_cast<uint64_t>(2 * c->nranks * (c->nranks - 1));  // all-gather slots
  *ptr = c->region[pr] + idx * c->slot_stride[pr];
  if (bytes) *bytes = c->slot_stride[pr];
  return SFC_OK;
}

sfc_status sfc_set_silent_rank(sfc_ctx* c, int silent_rank) {
  if (c == nullptr || silent_rank < -1 || silent_rank >= c->nranks) return SFC_ERR_INVALID;
  c->silent_rank = silent_rank;
  return SFC_OK;
}

uint64_t sfc_launch_count(const sfc_ctx* c) { return c ? c->launches : 0; }

sfc_status sfc_get_ll_view(sfc_ctx* c, sfc_ll_view* view) {
  if (c == nullptr || view == nullptr) return SFC_ERR_INVALID;
  if (c->region[kLL] == nullptr) return SFC_ERR_UNSUPPORTED;
  view->scratch = c->region[kLL];
  view->slot_stride = c->slot_stride[kLL];
  view->nranks = c->nranks;
  view->status = reinterpret_cast<int*>(c->dstatus);
  view->timeout_ns = static_cast<uint64_t>(c->cfg.timeout_us ? c->cfg.timeout_us : kDefaultTimeoutUs) * 1000ull;
  return SFC_OK;
}

sfc_status sfc_reserve_epochs(sfc_ctx* c, uint32_t k, uint32_t* first) {
  if (c == nullptr || first == nullptr || k == 0) return SFC_ERR_INVALID;
  if (c->cfg.device_epochs) return SFC_ERR_UNSUPPORTED;  // the host does not know the epoch
  if (c->poisoned) return SFC_ERR_ABORTED;
  if (c->next_epoch == 0 || static_cast<uint64_t>(c->next_epoch) + k - 1 > 0xFFFFFFFFull) return SFC_ERR_EPOCH;
  *first = c->next_epoch;
  c->next_epoch += k;
  return SFC_OK;
}

sfc_status sfc_linear_allreduce(sfc_ctx* c, const void* const* W, const void* const* x, void* const* y,
                                size_t hidden, size_t kdim, uint32_t epoch, void* stream) {
  return sfc_linear_allreduce_tokens(c, W, x, y, hidden, kdim, 1, epoch, stream);
}

sfc_status sfc_linear_allreduce_tokens(sfc_ctx* c, const void* const* W, const void* const* x, void* const* y,
                                       size_t hidden, size_t kdim, uint32_t tokens, uint32_t epoch, void* stream) {
  if (c == nullptr || W == nullptr || x == nullptr || y == nullptr) return SFC_ERR_INVALID;
  if (tokens < 1 || tokens > sfc::kLinearMaxTokens) return SFC_ERR_INVALID;
  // 2+ tokens on shapes of whole 16-row, 32-column tiles run on the tensor
  // cores (16-row x 8-token tiles); one token, or other shapes, on the CUDA
  // cores (token tile T)
  const bool mma = tokens >= 2 && hidden % 16 == 0 && kdim % 32 == 0;
  const uint32_t T = mma ? kLinearMma16 : sfc::linear_token_tile(tokens);
  if (hidden == 0 || hidden % 8 || hidden * tokens > c->max_count || kdim == 0 || kdim % 8 ||
      kdim * (mma ? tokens : T) > 49152)
    return SFC_ERR_INVALID;
  if (c->region[kLL] == nullptr) return SFC_ERR_UNSUPPORTED;
  if (c->poisoned) return SFC_ERR_ABORTED;
  epoch = resolve_epoch(c, epoch);
  if (c->cfg.device_epochs ? epoch != 0 : (epoch == 0 || epoch != c->next_epoch)) return SFC_ERR_EPOCH;
  const int N = c->nranks;
  sfc::LinearParams p{};
  p.epoch_dev = c->cfg.device_epochs ? c->d_epoch : nullptr;
  p.done_ctr = c->cfg.device_epochs ? c->d_epoch + 1 : nullptr;
  for (int r = 0; r < N; ++r) {
    if (!W[r] || !x[r] || !y[r] || !aligned16(W[r]) || !aligned16(x[r]) || !aligned16(y[r])) return SFC_ERR_INVALID;
    p.W[r] = static_cast<const uint16_t*>(W[r]);
    p.x[r] = static_cast<const uint16_t*>(x[r]);
    p.y[r] = static_cast<uint16_t*>(y[r]);
  }
  const size_t xb = tokens * kdim * 2, yb = tokens * hidden * 2;
  for (int a = 0; a < N; ++a)
    for (int b = 0; b < N; ++b)
      if (overlap(y[a], yb, x[b], xb) || overlap(y[a], yb, W[b], hidden * kdim * 2) ||
          (a < b && overlap(y[a], yb, y[b], yb)))
        return SFC_ERR_INVALID;
  // The tensor-core kernels: 32-byte weight pieces where ks >= 2 warps share
  // a tile (measured on B200: 0.92-0.97 of the weight stream there against
  // 0.75-0.87 with 16-byte pieces), 16-byte pieces where every warp owns
  // whole tiles (2-5 % faster there). 32-byte loads need every W_r 32-byte
  // aligned; otherwise the 16-byte pieces serve every shape.
  bool w32_ok = mma;
  for (int r = 0; r < N && w32_ok; ++r) w32_ok = (reinterpret_cast<uintptr_t>(W[r]) & 31u) == 0;
  // as many CTAs per rank as fit (two per SM), each rank's output units
  // (8-row vectors, or 16-row tiles on the tensor cores) split evenly over
  // its CTAs; ks warps share a unit when that evens out the 8 warps' work
  // (every part keeps at least 1024 columns)
  const uint64_t units = mma ? hidden / 16 : hidden / 8;  // 16-row tiles or 8-row vectors
  const uint64_t kparts = kdim / 1024;  // most column parts a unit may split into
  const int ti = mma ? 4 : T == 1 ? 0 : T == 2 ? 1 : T == 4 ? 2 : 3;
  int occ = c->linear_occ[ti];
  if (occ == 0) {
    occ = 2;
    const uint32_t kernels[2] = {T, kLinearMma32};  // both tensor-core kernels share the cache entry
    for (int k = 0; k < (mma ? 2 : 1); ++k) {
      const void* f = linear_kernel_for(N, kernels[k]);
      int o = 0;
      if (f == nullptr) return SFC_ERR_UNSUPPORTED;
      if (!cuda_ok(cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, c->smem_optin)))
        return SFC_ERR_CUDA;
      if (!cuda_ok(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, f, kLinearThreads, 0)) || o < 1)
        return SFC_ERR_RESOURCES;
      occ = std::min(occ, o);
    }
    c->linear_occ[ti] = occ;
  }
  int G = 0;
  uint32_t per = 0, ks = 1;
  bool wide = false;
  size_t smem = 0;
  // G, per, ks, piece width and shared memory from G0 CTAs per rank down
  // until the CTAs fit (both CTAs of an SM when two share one)
  auto fit = [&](int G0) {
    for (G = G0; G >= 1; --G) {
      per = static_cast<uint32_t>((units + G - 1) / G);
      double best = -1.0;
      for (uint32_t cand = 1; cand <= 8; cand *= 2) {
        if (cand > 1 && kparts < cand) break;
        const uint32_t groups = 8 / cand, rounds = (per + groups - 1) / groups;
        const double eff = static_cast<double>(per) / (static_cast<double>(rounds) * groups);
        if (eff > best + 1e-9) {
          best = eff;
          ks = cand;
        }
      }
      wide = w32_ok && ks >= 2;
      smem = mma ? sfc::linear_mma_smem_bytes(kdim, tokens, ks, per) : sfc::linear_smem_bytes(kdim, T, ks, per);
      if (smem <= static_cast<size_t>(c->smem_optin) &&
          (G * N <= c->sm_count || 2 * (smem + 1024) <= static_cast<size_t>(c->smem_optin) + 1024))
        return true;
    }
    return false;
  };
  if (!fit(occ * c->sm_count / N)) return SFC_ERR_RESOURCES;
  // Two CTAs an SM whose shared memory passes 2 x 96 KB leave the SM's
  // unified L1 too little room for the weight loads in flight; where the SMs
  // divide evenly among the ranks, one CTA an SM with a ring twice as deep
  // keeps the same bytes in flight and holds x once (measured on B200,
  // 2 x 8192 x 6144 x 8 tokens: 51.6 -> 34.9 us; at 56-86 KB of x, one CTA an
  // SM was 4-12 % slower, so it stays off there).
  bool one_per_sm = false;
  if (mma && c->sm_count % N == 0 && smem > kLinearOnePerSmSmemBytes) {
    if (c->linear_occ_one == 0) {
      for (const uint32_t v : {kLinearMma16 + kLinearMmaOnePerSm, kLinearMma32 + kLinearMmaOnePerSm}) {
        const void* f = linear_kernel_for(N, v);
        int o = 0;
        if (f == nullptr) return SFC_ERR_UNSUPPORTED;
        if (!cuda_ok(cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, c->smem_optin)))
          return SFC_ERR_CUDA;
        if (!cuda_ok(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, f, kLinearThreads, 0)) || o < 1)
          return SFC_ERR_RESOURCES;
      }
      c->linear_occ_one = 1;
    }
    one_per_sm = true;
    if (!fit(c->sm_count / N)) return SFC_ERR_RESOURCES;
  }
  const void* fn = linear_kernel_for(N, (wide ? kLinearMma32 : T) + (one_per_sm ? kLinearMmaOnePerSm : 0u));
  p.per_cta = per;
  p.ks = ks;
  p.hidden = hidden;
  p.kdim = kdim;
  p.tokens = tokens;
  p.G = G;
  p.epoch = epoch;
  sfc_status s = sfc_get_ll_view(c, &p.view);
  if (s != SFC_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* args[] = {&p};
  cudaError_t e = cudaLaunchCooperativeKernel(fn, dim3(N * G), dim3(kLinearThreads), args, smem, st);
  if (e == cudaErrorCooperativeLaunchTooLarge) {
    (void)cudaGetLastError();
    return SFC_ERR_RESOURCES;
  }
  if (!cuda_ok(e)) return SFC_ERR_CUDA;
  c->launches++;
  c->last_stream = st;
  if (!c->cfg.device_epochs) c->next_epoch = epoch + 1;
  return SFC_OK;
}

sfc_status sfc_check_guards(sfc_ctx* c) {
  if (c == nullptr) return SFC_ERR_INVALID;
  if (!cuda_ok(cudaStreamSynchronize(c->last_stream))) return SFC_ERR_CUDA;
  std::vector<uint8_t> h(kGuardBytes);
  for (int pr = 0; pr < kNumProtocols; ++pr) {
    if (c->region_raw[pr] == nullptr) continue;
    for (uint8_t* g : {c->region_raw[pr], c->region[pr] + c->region_bytes[pr]}) {
      if (!cuda_ok(cudaMemcpy(h.data(), g, kGuardBytes, cudaMemcpyDeviceToHost))) return SFC_ERR_CUDA;
      for (uint8_t b : h)
        if (b != kGuardByte) return SFC_ERR_GUARD;
    }
  }
  return SFC_OK;
}

}  // extern "C"
