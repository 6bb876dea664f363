/*
 * sfc.h -- C ABI of libsfc: self-synchronizing small-message all-reduce and
 * all-gather with N ranks emulated inside one B200.
 *
 * What is computed ("flash-comm: Self-Synchronizing Collective Communication
 * for LLM Decoding", abstract): an all-reduce in which every data block
 * carries its own readiness evidence, so a receiver validates exactly the
 * blocks it needs and no separate barrier is run; the reduction order is
 * fixed (rank 0, 1, ..., N-1, fp32 accumulation, one rounding to bf16) and
 * independent of the order in which blocks arrive, so every rank gets the
 * same bits; the same mechanism gives a standalone all-gather.
 *
 * Readiness encodings ("Why Microseconds Matter in AI Infrastructure",
 * section "Latency can matter more than bandwidth"):
 *   LL       -- data and flag in one atomic store: each 8-byte unit holds two
 *               bf16 elements and the 32-bit epoch.
 *   LL128    -- a 128-byte line of 120 data bytes and an 8-byte epoch flag.
 *   SENTINEL -- raw data into a receive buffer pre-filled with the negative
 *               NaN 0xFFFF, polled until it changes, then reset.
 * Double buffering by epoch parity (same section) replaces the bottom barrier.
 * The explicit-barrier oneshot / twoshot algorithms ("SiFAR:
 * Synchronization-Free All-Reduce for Low-Latency LLM Inference", abstract)
 * are provided in the same kernel framework as the comparison baseline.
 *
 * Emulation: rank r is a group of co-resident CTAs of one persistent
 * cooperative kernel; "sending to rank p" is a store into rank p's scratch in
 * this GPU's HBM. No data crosses a GPU boundary.
 *
 * Conventions shared by every call:
 *   - Pointers named "device" are CUDA device pointers on the context's
 *     device; pointers named "host" are host pointers. Tensor data is bf16
 *     (raw 16-bit patterns), element counts are per rank.
 *   - in[r] / out[r] are owned by the caller, 16-byte aligned, and must not
 *     overlap each other (no in-place). The library never reads an input
 *     after the call's kernel has finished and never writes an input.
 *   - Epochs: 32-bit, start at 1 after sfc_init / sfc_reset; every
 *     operation consumes one, and a call must pass exactly the next one
 *     (sfc_next_epoch), else SFC_ERR_EPOCH; 0, never an epoch itself,
 *     stands for the next one. All-reduce and all-gather share the
 *     sequence. Parity = epoch & 1 selects the scratch buffer. Once epoch
 *     2^32 - 1 has been used the sequence is spent: sfc_next_epoch returns 0
 *     and every call returns SFC_ERR_EPOCH until sfc_reset.
 *   - Device epochs (sfc_config.device_epochs): the next epoch is a word in
 *     device memory that each launch reads when it starts and that its last
 *     warp advances when every warp has finished, so a call enqueued now
 *     takes whatever epoch the stream order gives it. Calls must pass epoch 0
 *     (any other value: SFC_ERR_EPOCH), sfc_next_epoch returns 0,
 *     sfc_reserve_epochs is unsupported and sfc_reset sets the word back
 *     to 1. This makes calls capturable in a CUDA graph and replayable: each
 *     replay continues the sequence. A launch whose epochs would pass
 *     2^32 - 1 records SFC_ERR_EPOCH instead of running.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*,
 *     NULL = the legacy default stream). Calls on one context must be
 *     ordered on the GPU (one stream, or streams joined by events).
 *   - Device-side errors (a wait that ran out, a sentinel in an input under
 *     debug checks) are sticky: the kernel records them, every later
 *     chain launch of the context exits at once and every later single
 *     operation at its first wait check (a single operation does not load
 *     the error word before its first push, which would cost it an L2 round
 *     trip), until sfc_reset; the host refuses new work once sfc_get_status
 *     has seen the error. They are read with sfc_get_status.
 */
#ifndef SFC_H
#define SFC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct sfc_ctx sfc_ctx;

typedef enum {
  SFC_OK = 0,
  SFC_ERR_INVALID = 1,            /* bad argument; nothing was launched */
  SFC_ERR_CUDA = 2,               /* a CUDA runtime call failed */
  SFC_ERR_TIMEOUT = 3,            /* a device wait exceeded timeout_us */
  SFC_ERR_EPOCH = 4,              /* epoch is not the next one */
  SFC_ERR_RESOURCES = 5,          /* the ranks' CTAs cannot all be co-resident */
  SFC_ERR_SENTINEL_IN_INPUT = 6,  /* input holds 0xFFFF (debug checks only) */
  SFC_ERR_UNSUPPORTED = 7,        /* protocol / op / dtype combination not provided */
  SFC_ERR_ABORTED = 8,            /* context poisoned by an earlier device error */
  SFC_ERR_GUARD = 9               /* a scratch guard word was overwritten (sfc_check_guards) */
} sfc_status;

typedef enum {
  SFC_PROTO_AUTO = 0,             /* ask the selector */
  SFC_PROTO_LL = 1,
  SFC_PROTO_LL128 = 2,
  SFC_PROTO_SENTINEL = 3,
  SFC_PROTO_BARRIER_ONESHOT = 4,  /* pull, top + bottom barrier */
  SFC_PROTO_BARRIER_TWOSHOT = 5,  /* all-reduce only: reduce-scatter + all-gather */
  /* pull oneshot with the top barrier only: the caller double-buffers its
   * inputs (an input passed to operation e is not written again before
   * operation e + 2 is issued), which takes the place of the bottom barrier
   * ("SiFAR: Synchronization-Free All-Reduce for Low-Latency LLM Inference",
   * abstract: dual buffering removes the oneshot bottom barrier) */
  SFC_PROTO_BARRIER_ONESHOT_DB = 6,
  /* all-reduce only: reduce-scatter then all-gather, each phase a
   * self-synchronizing push with LL or sentinel readiness; no barrier */
  SFC_PROTO_LL_TWOSHOT = 7,
  SFC_PROTO_SENTINEL_TWOSHOT = 8,
  /* LL128 lines written and read with one warp-wide 16-byte-per-lane access
   * and no fences, relying on a 128-byte line being observed whole (not
   * promised by the PTX memory model; checked on B200 by a skewed
   * million-operation stress test). Opt-in: the built-in selector model
   * holds its measured latencies but marks it unavailable (alpha_us = -1);
   * a caller who accepts the assumption sets alpha_us = 0 in the entries it
   * wants and installs the model with sfc_set_cost_model. */
  SFC_PROTO_LL128_FAST = 9
} sfc_protocol;

#define SFC_NUM_PROTOCOLS 10
#define SFC_MAX_RANKS 8

typedef enum { SFC_BF16 = 0 } sfc_dtype;

typedef enum { SFC_OP_ALLREDUCE = 0, SFC_OP_ALLGATHER = 1 } sfc_op;

typedef struct {
  int ctas_per_rank;        /* CTAs per emulated rank; 0 = chosen per call */
  uint32_t timeout_us;      /* bound on each device-side wait; 0 = 50000 */
  int debug_checks;         /* nonzero: the kernel rejects sentinel inputs */
  uint32_t protocol_mask;   /* bit p provisions scratch for protocol p; 0 = all */
  int device_epochs;        /* nonzero: the epoch sequence lives on the device
                               (calls pass epoch 0; CUDA-graph replayable) */
} sfc_config;

/* Latency model of the selector, one entry per (op, protocol, nranks):
 * table_us[i] is the measured p50 latency (us) at 2^(SFC_COST_MIN_LOG2 + i)
 * bytes per rank (<= 0: not measured). The estimate at b bytes per rank is the
 * measured value, interpolated linearly in log2(b) between the nearest
 * measured sizes, held at the smallest measured value below it, and scaled by
 * algorithmic bytes (sfc_algorithmic_bytes) above the largest. An entry with
 * no measured size uses alpha_us + beta_us_per_byte * algorithmic bytes.
 * alpha_us < 0 marks the protocol unavailable for that rank count. */
#define SFC_COST_BUCKETS 24
#define SFC_COST_MIN_LOG2 9

typedef struct {
  double alpha_us;
  double beta_us_per_byte;
  double table_us[SFC_COST_BUCKETS];
} sfc_cost_entry;

typedef struct {
  sfc_cost_entry c[2][SFC_NUM_PROTOCOLS][SFC_MAX_RANKS + 1]; /* [op][protocol][nranks] */
} sfc_cost_model;

#define SFC_FLOOR_SMS 8        /* initiator SMs, and as many responder SMs */
#define SFC_FLOOR_LOCATIONS 8  /* flag addresses (different L2 homes) */

typedef struct {
  /* Flag round trip between two CTAs on different SMs, measured for every
   * (initiator, responder) pair of a fixed SM set chosen by %smid at each of
   * SFC_FLOOR_LOCATIONS flag addresses: one trial per (pair, location), its
   * median over the trial's round trips. */
  double flag_rtt_ns_p50;      /* median over the trials: the floor */
  double flag_rtt_ns_p10;      /* 10th / 90th percentile over the trials */
  double flag_rtt_ns_p90;
  double flag_rtt_ns_min_pair; /* fastest / slowest trial */
  double flag_rtt_ns_max_pair;
  double flag_rtt_ns_by_location[SFC_FLOOR_LOCATIONS]; /* median over the pairs at each address */
  int initiator_sm[SFC_FLOOR_SMS]; /* %smid of the initiators and responders */
  int responder_sm[SFC_FLOOR_SMS];
  int pairs;                   /* trials: SM pairs x locations */
  double l2_rtt_ns_p50;        /* dependent L2-hit loads, one thread */
  double sm_clock_ghz;         /* clock64 ticks per globaltimer ns during the run */
  double globaltimer_step_ns;  /* smallest nonzero globaltimer increment seen */
} sfc_floor_result;

/* Create a context for `nranks` (2..8) emulated ranks on the current CUDA
 * device, with scratch for messages up to `max_bytes_per_rank` bytes per rank
 * (all-gather: per shard). Allocates the scratch (per provisioned protocol:
 * 2 parities x N x (N-1) encoded slots), barrier flags and status words;
 * sentinel slots are filled with 0xFFFF, flags zeroed, next epoch = 1.
 * cfg may be NULL (defaults). Synchronous. Environment, read here:
 * SFC_TIMEOUT_MS (> 0) bounds every device wait when cfg leaves timeout_us
 * at 0; SFC_PROTOCOL (a protocol name such as "sentinel", lower case, or its
 * number) is what AUTO resolves to wherever that protocol is provisioned
 * and supports the operation. Unparsable values are ignored. */
sfc_status sfc_init(sfc_ctx** ctx, int nranks, size_t max_bytes_per_rank, const sfc_config* cfg);

/* Free everything the context owns (synchronizes the device first). */
sfc_status sfc_destroy(sfc_ctx* ctx);

/* Return the context to its initial state on `stream`: refill sentinel
 * slots, zero flags and barrier counters, clear the sticky error; the next
 * epoch becomes 1. The only way out of a device error. */
sfc_status sfc_reset(sfc_ctx* ctx, void* stream);

/* One all-reduce. in/out: HOST arrays of N DEVICE pointers, each to `count`
 * bf16 elements. After the kernel, out[r][i] = bf16_RNE(sum over q = 0..N-1,
 * in rank order, of fp32(in[q][i])) for every rank r. count == 0 is a no-op
 * that consumes no epoch. protocol AUTO asks the selector. */
sfc_status sfc_allreduce(sfc_ctx* ctx, const void* const* in, void* const* out, size_t count,
                         sfc_dtype dtype, sfc_protocol protocol, uint32_t epoch, void* stream);

/* One all-gather. in: N device pointers to `count` elements; out: N device
 * pointers to N*count elements; out[r] = in[0] || in[1] || ... || in[N-1].
 * The twoshot protocols are all-reduce algorithms (SFC_ERR_UNSUPPORTED). */
sfc_status sfc_allgather(sfc_ctx* ctx, const void* const* in, void* const* out, size_t count,
                         sfc_dtype dtype, sfc_protocol protocol, uint32_t epoch, void* stream);

/* k_ops operations issued back to back inside ONE persistent launch,
 * epochs first_epoch .. first_epoch + k_ops - 1 (the decode step's chain of
 * per-layer all-reduces). in_table / out_table: DEVICE arrays of k_ops*N
 * device pointers, entry [k*N + r] for operation k, rank r. No input may be
 * an output of the same chain. skew_ns: DEVICE array [k_ops*N] or NULL;
 * before pushing operation k, rank r spins skew_ns[k*N + r] ns (capped at
 * the timeout). timings: DEVICE array [k_ops + 1] or NULL; the library
 * clears it on `stream`, then timings[0] = earliest kernel start and
 * timings[1 + k] = latest completion of operation k over all warps, in
 * %globaltimer nanoseconds. */
sfc_status sfc_allreduce_chain(sfc_ctx* ctx, int k_ops, const void* const* in_table,
                               void* const* out_table, size_t count, sfc_dtype dtype,
                               sfc_protocol protocol, uint32_t first_epoch,
                               const uint32_t* skew_ns, uint64_t* timings, void* stream);

/* A prepared single all-reduce or all-gather, for callers that issue one
 * collective at a time on fixed buffers (a decode step that cannot chain its
 * layers' all-reduces into one launch). sfc_plan_create does once what every
 * sfc_allreduce / sfc_allgather call does: the argument and operand checks
 * (as sfc_allreduce; count == 0 -> SFC_ERR_INVALID), the protocol choice
 * (SFC_PROTO_AUTO -> the selector), the kernel and the launch shape.
 * sfc_plan_launch then takes the context's next epoch and launches on
 * `stream`: per call it costs little more than the CUDA launch. The operand
 * pointers are fixed at creation (the host arrays are copied); their
 * contents may change between launches. Launches share the context's epoch
 * sequence with every other call. A plan is valid while its context lives:
 * destroy plans first. Not thread-safe with other calls on the context. */
typedef struct sfc_plan sfc_plan;
sfc_status sfc_plan_create(sfc_ctx* ctx, sfc_op op, const void* const* in, void* const* out, size_t count,
                           sfc_dtype dtype, sfc_protocol protocol, sfc_plan** plan);
sfc_status sfc_plan_launch(sfc_plan* plan, void* stream);
sfc_status sfc_plan_destroy(sfc_plan* plan);

/* The all-gather counterpart of sfc_allreduce_chain (out entries hold
 * N*count elements). */
sfc_status sfc_allgather_chain(sfc_ctx* ctx, int k_ops, const void* const* in_table,
                               void* const* out_table, size_t count, sfc_dtype dtype,
                               sfc_protocol protocol, uint32_t first_epoch,
                               const uint32_t* skew_ns, uint64_t* timings, void* stream);

/* End-to-end all-reduce chain from HOST memory: in_host holds
 * [k_ops][N][count] bf16 contiguous, out_host receives [k_ops][N][count].
 * Copies the inputs to context-owned device staging (allocated on first use,
 * grown as needed; growing waits for the device), runs the chain, copies the
 * outputs back. The chain runs as up to 8 launches of at least 16
 * operations, and the copies of one segment overlap the run of its
 * neighbours on two context-owned copy streams; events tie them to
 * `stream`, which ends up waiting for the last copy, so the call is ordered
 * on `stream` like any other. It returns once everything is queued.
 * Page-locked host memory makes the copies asynchronous. timings as in
 * sfc_allreduce_chain. */
sfc_status sfc_allreduce_chain_host(sfc_ctx* ctx, int k_ops, const void* in_host, void* out_host,
                                    size_t count, sfc_dtype dtype, sfc_protocol protocol,
                                    uint32_t first_epoch, uint64_t* timings, void* stream);

/* The selector (cost-guided choice of the encoding by message size and rank
 * count: "flash-comm: Self-Synchronizing Collective Communication for LLM
 * Decoding", abstract; the empirical choice in "Why Microseconds Matter in AI
 * Infrastructure", section "What I learned from it"). argmin over protocols
 * of the model's latency estimate (sfc_cost_estimate); ties go to fewer
 * algorithmic bytes, then to the order SENTINEL, LL128, LL128_FAST, LL,
 * SENTINEL_TWOSHOT, LL_TWOSHOT, BARRIER_ONESHOT_DB, BARRIER_ONESHOT,
 * BARRIER_TWOSHOT. Host only. */
sfc_protocol sfc_select_protocol(const sfc_ctx* ctx, sfc_op op, size_t bytes_per_rank, int nranks);

/* The same choice from an explicit model; needs no context and no GPU. */
sfc_protocol sfc_select_protocol_model(const sfc_cost_model* model, sfc_op op,
                                       size_t bytes_per_rank, int nranks);

/* The model's latency estimate (us) for one protocol; < 0 if unavailable. */
double sfc_cost_estimate(const sfc_cost_model* model, sfc_op op, sfc_protocol protocol,
                         size_t bytes_per_rank, int nranks);

/* Replace the context's model (copied). The built-in default holds p50
 * latencies measured on a B200 by the message-size sweep. */
sfc_status sfc_set_cost_model(sfc_ctx* ctx, const sfc_cost_model* model);

/* Write the built-in default model into *model. */
void sfc_default_cost_model(sfc_cost_model* model);

/* Algorithmic bytes of one operation summed over all ranks (encoded bytes
 * written plus bytes read; the sentinel's reset writes included); the
 * roofline numerator. Returns -1 for an unsupported combination. */
double sfc_algorithmic_bytes(sfc_op op, sfc_protocol protocol, size_t count, int nranks);

/* Synchronize the context's last stream and return its sticky device status
 * (SFC_OK if none). *info (may be NULL) receives detail: for a timeout,
 * (operation index << 16) | (rank << 8) | source. The error stays set until
 * sfc_reset. */
sfc_status sfc_get_status(sfc_ctx* ctx, uint32_t* info);

/* Static English name of a status. */
const char* sfc_status_string(sfc_status s);

/* The epoch the next operation must use. */
uint32_t sfc_next_epoch(const sfc_ctx* ctx);

/* The launch shape a call would use: CTAs per rank and threads per CTA
 * (256, or 128 for LL, sentinel and one-load LL128 messages of at most
 * 64 KB per rank at 4 or more ranks when ctas_per_rank is 0). */
sfc_status sfc_launch_shape(sfc_ctx* ctx, sfc_op op, sfc_protocol protocol, size_t count,
                            int* ctas_per_rank, int* threads_per_cta);

/* Device address and byte size of one receive slot of the scratch, for
 * inspection by tests: rank `rank`'s slot for source `src` (!= rank) at
 * `parity` (0 or 1), under a self-synchronizing protocol. For the twoshot
 * protocols parity 0/1 selects a reduce-scatter slot and 2/3 the all-gather
 * slot of parity 0/1. */
sfc_status sfc_scratch_slot(sfc_ctx* ctx, sfc_protocol protocol, int rank, int parity, int src,
                            void** device_ptr, size_t* bytes);

/* Fault injection on the host side: from the next launch on, rank
 * `silent_rank` pushes nothing and arrives at no barrier (-1 = off). Its
 * peers' waits then run out after timeout_us and report SFC_ERR_TIMEOUT. */
sfc_status sfc_set_silent_rank(sfc_ctx* ctx, int silent_rank);

/* Latency floor microbenchmarks on the current device (synchronous, owns
 * its buffers): a flag round trip between two CTAs on different SMs and the
 * L2 hit latency. The speed-of-light bound of "Why Microseconds Matter in AI
 * Infrastructure", section "Defining the physical lower bound", is built
 * from such round trips. The SM pairs are fixed by %smid (every SM hosts
 * exactly one CTA of the measuring launch): SFC_FLOOR_SMS initiators and as
 * many responders spread evenly over the sorted SM ids, every initiator
 * with every responder, at SFC_FLOOR_LOCATIONS flag addresses, since where
 * a flag's L2 home sits moves one pair's round trip by up to 0.6 us on B200.
 * iters (>= 16) round trips per trial; the first iters / 8 (at most 64)
 * warm the lines and are not counted. */
sfc_status sfc_measure_floor(int iters, sfc_floor_result* out);

/* Number of kernel launches this context has issued (all entry points). */
uint64_t sfc_launch_count(const sfc_ctx* ctx);

/* Device-side LL view of a context, for user kernels that push and poll LL
 * units themselves through the device API in sfc_ll_device.cuh ("Why
 * Microseconds Matter in AI Infrastructure", section "Communication is
 * becoming part of GPU execution": LL send / receive / reduce called from
 * inside kernels). Plain data; valid while the context lives. */
typedef struct {
  unsigned char* scratch;   /* LL region; slot (recv, parity, j) at
                               ((recv * 2 + parity) * (nranks - 1) + j) * slot_stride,
                               j = src < recv ? src : src - 1 */
  uint64_t slot_stride;     /* bytes */
  int nranks;
  int* status;              /* {first error, detail, abort word, unused} */
  uint64_t timeout_ns;      /* bound on each device-side wait */
} sfc_ll_view;

/* Fill *view for the context's LL scratch (SFC_ERR_UNSUPPORTED if LL is not
 * provisioned). */
sfc_status sfc_get_ll_view(sfc_ctx* ctx, sfc_ll_view* view);

/* Reserve k consecutive epochs for a user kernel that uses the LL view:
 * *first receives the first; the context's next epoch advances by k. */
sfc_status sfc_reserve_epochs(sfc_ctx* ctx, uint32_t k, uint32_t* first);

/* Row-parallel linear layer fused with its all-reduce, for one decode token:
 * every rank r holds W[r] (bf16 [hidden][kdim], row-major: its slice of the
 * input dimension) and x[r] (bf16 [kdim]); the kernel computes the partial
 * p_r = bf16_RNE(W[r] x[r]) (fp32 accumulation) and pushes each finished
 * 8-row vector of it as LL units to every peer while the rest of W[r] is
 * still streaming; each rank then polls, reduces p_0..p_{N-1} in rank order
 * in fp32 and writes y[r] (bf16 [hidden], identical on every rank). One
 * cooperative launch (up to two CTAs per SM), no intermediate buffer in
 * global memory. hidden % 8 == 0, hidden <= max count of the context;
 * kdim % 8 == 0, kdim <= 49152; all pointers 16-byte aligned; consumes one
 * epoch. SFC_ERR_RESOURCES if a CTA's shared memory (x[r], then 20 + 32 ks
 * bytes per output vector it owns, ks <= 8) cannot fit. */
sfc_status sfc_linear_allreduce(sfc_ctx* ctx, const void* const* W, const void* const* x, void* const* y,
                                size_t hidden, size_t kdim, uint32_t epoch, void* stream);

/* The same for `tokens` (1..8) decode tokens at once: x[r] is bf16
 * [tokens][kdim], y[r] bf16 [tokens][hidden]; the weights stream once for
 * all tokens and the all-reduce covers tokens * hidden elements (one epoch).
 * tokens * hidden <= max count of the context; kdim * T <= 49152, T = tokens
 * rounded up to 1, 2, 4 or 8; 2+ tokens with hidden % 16 == 0 and
 * kdim % 32 == 0 run on the tensor cores instead, with tokens * kdim <= 49152
 * (where several warps share a tile's columns, weights that are 32-byte
 * aligned are read in 32-byte pieces, otherwise in 16-byte pieces).
 * sfc_linear_allreduce is tokens = 1. Measured on B200 against a library
 * tensor-core GEMM + all-reduce on 8192-hidden shapes: 1.06-1.23x faster at
 * 2-8 tokens; within 3 % of it on the largest shapes. */
sfc_status sfc_linear_allreduce_tokens(sfc_ctx* ctx, const void* const* W, const void* const* x, void* const* y,
                                       size_t hidden, size_t kdim, uint32_t tokens, uint32_t epoch, void* stream);

/* Every scratch region sits between two 4 KB guards filled with 0xA5 at
 * sfc_init and never written by any kernel. Synchronizes the context's last
 * stream and returns SFC_ERR_GUARD if a guard byte changed (a write outside a
 * region), else SFC_OK. A check for tests and debugging. */
sfc_status sfc_check_guards(sfc_ctx* ctx);

/* Largest per-rank element count sfc_allreduce_noalloc accepts (8 KB of bf16). */
#define SFC_NOALLOC_MAX_COUNT 4096

/* One LL all-reduce that allocates nothing. The pages have no counterpart:
 * this is a library convenience for callers that cannot call cudaMalloc when
 * they need the collective -- code inside an allocator or an out-of-memory
 * path, a process that reserved all device memory at start-up, or a host
 * library that may not own allocations. Its scratch is a file-scope static
 * device array of about 1.8 MB that every GPU loading this library keeps until
 * the process exits; no context is needed.
 *   in / out: HOST arrays of `nranks` (2..8) DEVICE pointers, 16-byte
 *   aligned, `count` bf16 elements each, no overlap; result as sfc_allreduce
 *   (rank-order fp32 sum, one bf16 rounding), every rank the same bits.
 *   count > SFC_NOALLOC_MAX_COUNT -> SFC_ERR_INVALID.
 * Set-up: the first call on a device (any count, with that device current)
 * looks up the array's device address (cudaGetSymbolAddress), the SM count
 * and the kernel's occupancy. That lookup may load this library's device code
 * and place the array in device memory, so it can fail where memory has run
 * out: make one call with count == 0 (in, out and nranks are then ignored and
 * nothing is launched) on every device at start-up, before any stream capture.
 * Each call clears the part of the array it uses (cudaMemsetAsync on
 * `stream`), then launches; it calls no cudaMalloc, cudaFree or allocating
 * library routine. All calls share the one array and it keeps the last call's
 * contents, so calls that overlap on the GPU (other streams, other threads)
 * race: order them.
 * Errors on the device (a wait that ran out, bounded by SFC_TIMEOUT_MS or
 * 50 ms) stay recorded in the array: every later call then exits at once
 * without writing its outputs, until sfc_noalloc_status has read them. */
sfc_status sfc_allreduce_noalloc(const void* const* in, void* const* out, int nranks, size_t count,
                                 void* stream);

/* Device status of the allocation-free all-reduce on the current device,
 * read after every earlier call on `stream` (synchronizes the stream):
 * SFC_OK, or the first error recorded (SFC_ERR_TIMEOUT: *info = the
 * operation, rank and source of the wait that ran out, as sfc_get_status).
 * Reading clears it, so later calls run again. Allocates nothing. */
sfc_status sfc_noalloc_status(void* stream, uint32_t* info);

#ifdef __cplusplus
}
#endif

#endif /* SFC_H */
