/* Concurrent CPU model of the self-synchronizing all-reduce and all-gather.
 *
 * TEST INFRASTRUCTURE ONLY: only tests/ and the CPU-baseline leg of bench.py
 * load it (through oracle/threaded.py). It shares no code with the CUDA
 * library and is independent of the Python oracle too: plain C11, one POSIX
 * thread per rank, C11 atomics for every word two threads exchange through.
 *
 * What it models ("Why Microseconds Matter in AI Infrastructure", section
 * "Latency can matter more than bandwidth"; "flash-comm: Self-Synchronizing
 * Collective Communication for LLM Decoding", abstract; "SiFAR:
 * Synchronization-Free All-Reduce for Low-Latency LLM Inference", abstract
 * and introduction):
 *
 *  - self-synchronizing oneshot: every rank pushes its chunk into each
 *    peer's receive slot slot[recv][epoch & 1][src], and the receiver
 *    validates units on their own:
 *      LL       8-byte unit = 32-bit data word (bf16 2j low, 2j+1 high) and a
 *               32-bit flag equal to the epoch, written as one atomic store;
 *      LL128    128-byte line = 15 data words (60 bf16) and a flag word; the
 *               data words are stored first and the flag last with release
 *               order, the reader acquires the flag before the data;
 *      sentinel raw bf16 elements into a slot pre-filled with 0xFFFF; the
 *               reader takes an element once it differs from 0xFFFF and
 *               writes 0xFFFF back before it pushes its next epoch;
 *    epoch-parity double buffering, no bottom barrier: a writer reaches
 *    epoch e+2 of a slot only after it received e+1 from the slot's reader,
 *    which that reader pushed after it finished epoch e (release stores on
 *    the pushes, acquire loads on the polls carry the order);
 *  - self-synchronizing twoshot (LL or sentinel units): shard s of every
 *    input goes to rank s (reduce-scatter slots), rank s reduces it and
 *    pushes the result to every peer (all-gather slots), both phases with
 *    epoch-parity slots; shards are whole 8-element vectors;
 *  - the explicit-barrier baselines, with the caller's input buffer made
 *    explicit (each operation first writes its input into it, standing for
 *    the layer that produces the activation): the oneshot (top barrier, read
 *    every rank's buffer, bottom barrier: the write-after-write guard), the
 *    dual-buffered oneshot (inputs alternate two buffers, top barrier only)
 *    and the twoshot (top barrier, reduce-scatter into a per-rank result
 *    buffer, middle barrier, all-gather, bottom barrier);
 *  - the reduction: fp32 round-to-nearest adds in rank order 0..N-1 starting
 *    from rank 0's value, one final rounding to bf16 (ties to even), so all
 *    ranks produce the same bits whatever order the units arrived in.
 *
 * Delays: skew_ns[k][r] holds rank r back for that long in operation k,
 * before it starts the operation (skew_after = 0) or after its pushes / its
 * top barrier and before it reads anything (skew_after = 1, a late reader).
 *
 * Floating point: binary32 adds only, built with -ffp-contract=off (no
 * excess precision on the targets this builds for, no flush-to-zero).
 */
#define _GNU_SOURCE
#include <pthread.h>
#include <sched.h>
#include <stdatomic.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <time.h>

enum {
  SFO_LL = 1,
  SFO_LL128 = 2,
  SFO_SENTINEL = 3,
  SFO_BARRIER_ONESHOT = 4,
  SFO_BARRIER_TWOSHOT = 5,
  SFO_BARRIER_ONESHOT_DB = 6,
  SFO_LL_TWOSHOT = 7,
  SFO_SENTINEL_TWOSHOT = 8
};
enum { SFO_ALLREDUCE = 0, SFO_ALLGATHER = 1 };
enum {
  SFO_OK = 0,
  SFO_EINVAL = 1,
  SFO_ETIMEOUT = 2,
  SFO_EPOST = 3, /* a slot was not left as the protocol requires */
  SFO_ENOMEM = 4,
  SFO_ETHREAD = 5
};

#define MAX_RANKS 8
#define SENTINEL_BITS 0xFFFFu
#define LL128_WORDS 16 /* 8-byte words per 128-byte line */
#define LL128_ELEMS 60 /* bf16 elements per line (15 data words) */
#define VEC 8          /* elements per twoshot shard granule */

/* ------------------------------------------------------------ bf16 codec */

static float widen(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* binary32 -> bf16, round to nearest, ties to even; NaN stays NaN with its
 * sign and the quiet bit set. */
static uint16_t narrow(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x0040u);
  uint32_t hi = u >> 16, lo = u & 0xFFFFu;
  if (lo > 0x8000u || (lo == 0x8000u && (hi & 1u))) hi += 1u;
  return (uint16_t)hi;
}

/* Rank-order sum of src[0..n-1][i], rounded once. */
static uint16_t reduce_at(const uint16_t* const* src, int n, size_t i) {
  float acc = widen(src[0][i]);
  for (int q = 1; q < n; ++q) acc = acc + widen(src[q][i]);
  return narrow(acc);
}

/* ------------------------------------------------------------ slots */

/* Receive slots [recv][parity][src], each `units` units of one encoding. */
typedef struct {
  int enc; /* SFO_LL, SFO_LL128 or SFO_SENTINEL */
  int nranks;
  size_t units;
  _Atomic uint64_t* w; /* LL units, or LL128 lines as 16 words each */
  _Atomic uint16_t* e; /* sentinel elements */
} Slots;

static size_t units_for(int enc, size_t n) {
  if (enc == SFO_LL) return (n + 1) / 2;
  if (enc == SFO_LL128) return (n + LL128_ELEMS - 1) / LL128_ELEMS * LL128_WORDS;
  return n;
}

static int slots_init(Slots* z, int enc, int nranks, size_t max_elems) {
  z->enc = enc;
  z->nranks = nranks;
  z->units = units_for(enc, max_elems);
  const size_t total = (size_t)nranks * 2 * (size_t)nranks * z->units;
  z->w = NULL;
  z->e = NULL;
  if (total == 0) return 0;
  if (enc == SFO_SENTINEL) {
    z->e = malloc(total * sizeof(*z->e));
    if (!z->e) return 1;
    for (size_t i = 0; i < total; ++i) atomic_init(&z->e[i], (uint16_t)SENTINEL_BITS);
  } else {
    z->w = malloc(total * sizeof(*z->w));
    if (!z->w) return 1;
    for (size_t i = 0; i < total; ++i) atomic_init(&z->w[i], 0); /* 0 is never an epoch */
  }
  return 0;
}

static void slots_free(Slots* z) {
  free(z->w);
  free(z->e);
}

static size_t slot_base(const Slots* z, int recv, int parity, int src) {
  return (((size_t)recv * 2 + (size_t)parity) * (size_t)z->nranks + (size_t)src) * z->units;
}

/* Writer side: n elements of x into slot[recv][epoch & 1][src]. */
static void put(Slots* z, int recv, int src, uint32_t epoch, const uint16_t* x, size_t n) {
  const size_t base = slot_base(z, recv, (int)(epoch & 1u), src);
  if (z->enc == SFO_LL) {
    for (size_t j = 0; j < units_for(SFO_LL, n); ++j) {
      uint32_t lo = x[2 * j];
      uint32_t hi = (2 * j + 1 < n) ? x[2 * j + 1] : 0u;
      uint64_t unit = (uint64_t)(lo | (hi << 16)) | ((uint64_t)epoch << 32);
      atomic_store_explicit(&z->w[base + j], unit, memory_order_release);
    }
  } else if (z->enc == SFO_LL128) {
    for (size_t line = 0; line < units_for(SFO_LL128, n) / LL128_WORDS; ++line) {
      _Atomic uint64_t* w = &z->w[base + line * LL128_WORDS];
      for (int d = 0; d < LL128_WORDS - 1; ++d) {
        uint64_t word = 0;
        for (int h = 0; h < 4; ++h) {
          size_t i = line * LL128_ELEMS + (size_t)d * 4 + (size_t)h;
          if (i < n) word |= (uint64_t)x[i] << (16 * h);
        }
        atomic_store_explicit(&w[d], word, memory_order_relaxed);
      }
      atomic_store_explicit(&w[LL128_WORDS - 1], (uint64_t)epoch, memory_order_release);
    }
  } else {
    for (size_t i = 0; i < n; ++i) atomic_store_explicit(&z->e[base + i], x[i], memory_order_release);
  }
}

/* Reader side: takes whatever units of slot[recv][epoch & 1][src] have
 * arrived, starting at unit `from`, decoding into dst (n elements); returns
 * the first unit not yet valid. */
static size_t take(Slots* z, int recv, int src, uint32_t epoch, uint16_t* dst, size_t n, size_t from) {
  const size_t base = slot_base(z, recv, (int)(epoch & 1u), src);
  const size_t units = units_for(z->enc, n);
  size_t j = from;
  if (z->enc == SFO_LL) {
    for (; j < units; ++j) {
      uint64_t unit = atomic_load_explicit(&z->w[base + j], memory_order_acquire);
      if ((uint32_t)(unit >> 32) != epoch) break;
      dst[2 * j] = (uint16_t)(unit & 0xFFFFu);
      if (2 * j + 1 < n) dst[2 * j + 1] = (uint16_t)((unit >> 16) & 0xFFFFu);
    }
  } else if (z->enc == SFO_LL128) {
    for (; j < units; j += LL128_WORDS) {
      _Atomic uint64_t* line = &z->w[base + j];
      if (atomic_load_explicit(&line[LL128_WORDS - 1], memory_order_acquire) != (uint64_t)epoch) break;
      size_t first = (j / LL128_WORDS) * LL128_ELEMS;
      for (int d = 0; d < LL128_WORDS - 1; ++d) {
        uint64_t word = atomic_load_explicit(&line[d], memory_order_relaxed);
        for (int h = 0; h < 4; ++h) {
          size_t i = first + (size_t)d * 4 + (size_t)h;
          if (i < n) dst[i] = (uint16_t)(word >> (16 * h));
        }
      }
    }
  } else { /* take the element, then put the pre-fill back */
    for (; j < units; ++j) {
      uint16_t v = atomic_load_explicit(&z->e[base + j], memory_order_acquire);
      if (v == SENTINEL_BITS) break;
      dst[j] = v;
      atomic_store_explicit(&z->e[base + j], (uint16_t)SENTINEL_BITS, memory_order_relaxed);
    }
  }
  return j;
}

/* After a chain of k_ops operations every sentinel slot holds the pre-fill
 * again and every LL / LL128 unit a chain wrote holds the epoch of the last
 * operation of its parity (0 where none wrote). `n_of(recv, src)` is the
 * element count that pair exchanges. */
static int slots_check(const Slots* z, int k_ops, size_t (*n_of)(const void*, int, int), const void* ctx) {
  for (int r = 0; r < z->nranks; ++r)
    for (int parity = 0; parity < 2; ++parity)
      for (int q = 0; q < z->nranks; ++q) {
        if (q == r) continue;
        const size_t base = slot_base(z, r, parity, q);
        const size_t units = units_for(z->enc, n_of(ctx, r, q));
        uint32_t last = (uint32_t)k_ops;
        if ((last & 1u) != (uint32_t)parity) last = last >= 1 ? last - 1 : 0;
        if (z->enc == SFO_SENTINEL) {
          for (size_t i = 0; i < z->units; ++i)
            if (atomic_load(&z->e[base + i]) != SENTINEL_BITS) return SFO_EPOST;
        } else if (z->enc == SFO_LL) {
          for (size_t j = 0; j < units; ++j)
            if ((uint32_t)(atomic_load(&z->w[base + j]) >> 32) != last) return SFO_EPOST;
        } else {
          for (size_t j = LL128_WORDS - 1; j < units; j += LL128_WORDS)
            if (atomic_load(&z->w[base + j]) != (uint64_t)last) return SFO_EPOST;
        }
      }
  return SFO_OK;
}

/* ------------------------------------------------------------ shared state */

typedef struct {
  int protocol, op, nranks, k_ops, skew_after, yield_polls;
  size_t count;
  const uint16_t* in;      /* [k][N][count] */
  uint16_t* out;           /* [k][N][count] (all-reduce) or [k][N][N*count] */
  const uint32_t* skew_ns; /* [k][N] or NULL */
  uint64_t timeout_ns;
  Slots a, b;              /* oneshot: a; twoshot: a = reduce-scatter, b = all-gather */
  size_t shard_lo[MAX_RANKS + 1]; /* twoshot shard q = [shard_lo[q], shard_lo[q + 1]) */
  uint16_t* inbuf;         /* barrier protocols: [N][2][count], the caller's input buffers */
  uint16_t* red;           /* barrier twoshot: [N][2][count], reduced shards */
  _Atomic uint32_t bar[3][MAX_RANKS]; /* top, middle, bottom barrier arrivals (epochs) */
  _Atomic int abort_flag;
  _Atomic int start;
  _Atomic int status;
} Shared;

typedef struct {
  Shared* s;
  int rank;
  uint16_t* stage; /* [N][count] decoded sources */
} Rank;

static uint64_t now_ns(void) {
  struct timespec ts;
  clock_gettime(CLOCK_MONOTONIC, &ts);
  return (uint64_t)ts.tv_sec * 1000000000ull + (uint64_t)ts.tv_nsec;
}

static void delay(const Shared* s, int k, int r, int after) {
  if (!s->skew_ns || s->skew_after != after) return;
  const uint64_t until = now_ns() + s->skew_ns[(size_t)k * s->nranks + r];
  while (now_ns() < until) {
  }
}

static void cpu_relax(void) {
#if defined(__x86_64__) || defined(__i386__)
  __builtin_ia32_pause();
#elif defined(__aarch64__)
  __asm__ __volatile__("yield");
#endif
}

/* A bounded wait: called once per unsuccessful poll. Returns nonzero when the
 * caller must give up (deadline passed or another rank gave up). */
typedef struct {
  uint64_t deadline;
  unsigned polls;
} Wait;

static Wait wait_start(const Shared* s) {
  Wait w = {now_ns() + s->timeout_ns, 0};
  return w;
}

static int wait_more(Shared* s, Wait* w) {
  cpu_relax(); /* leave the line to its writer for a moment */
  if ((++w->polls & 255u) == 0) {
    if (atomic_load_explicit(&s->abort_flag, memory_order_relaxed)) return 1;
    if (now_ns() > w->deadline) {
      int ok = SFO_OK;
      atomic_compare_exchange_strong(&s->status, &ok, SFO_ETIMEOUT);
      atomic_store(&s->abort_flag, 1);
      return 1;
    }
    if (s->yield_polls) sched_yield();
  }
  return 0;
}

static const uint16_t* input(const Shared* s, int k, int r) {
  return s->in + ((size_t)k * s->nranks + r) * s->count;
}

static uint16_t* output(const Shared* s, int k, int r) {
  const size_t width = s->op == SFO_ALLREDUCE ? s->count : (size_t)s->nranks * s->count;
  return s->out + ((size_t)k * s->nranks + r) * width;
}

/* Polls slot[me][.][q] of every q != me until n[q] elements of each have
 * arrived, decoding into dst[q]; sources are visited round-robin and each
 * pass takes whatever has arrived, so the arrival order is free. */
static int take_all(Shared* s, Slots* z, int me, uint32_t epoch, uint16_t* const* dst, const size_t* n) {
  size_t done[MAX_RANKS] = {0};
  int remaining = 0;
  for (int q = 0; q < s->nranks; ++q)
    if (q != me && units_for(z->enc, n[q]) > 0) ++remaining;
  Wait w = wait_start(s);
  while (remaining > 0) {
    int progressed = 0;
    for (int q = 0; q < s->nranks; ++q) {
      const size_t units = units_for(z->enc, n[q]);
      if (q == me || done[q] == units) continue;
      const size_t j = take(z, me, q, epoch, dst[q], n[q], done[q]);
      if (j != done[q]) progressed = 1;
      done[q] = j;
      if (j == units) --remaining;
    }
    if (!progressed && remaining > 0 && wait_more(s, &w)) return 1;
  }
  return 0;
}

static int barrier(Shared* s, int which, int r, uint32_t epoch) {
  _Atomic uint32_t* bar = s->bar[which];
  atomic_store_explicit(&bar[r], epoch, memory_order_release);
  Wait w = wait_start(s);
  for (int q = 0; q < s->nranks; ++q)
    while (atomic_load_explicit(&bar[q], memory_order_acquire) < epoch)
      if (wait_more(s, &w)) return 1;
  return 0;
}

/* ------------------------------------------------------------ one operation per protocol */

/* Self-synchronizing oneshot (LL / LL128 / sentinel). */
static int op_selfsync_oneshot(Shared* s, Rank* me, int k, uint32_t epoch) {
  const int n = s->nranks, r = me->rank;
  const size_t c = s->count;
  const uint16_t* x = input(s, k, r);
  for (int p = 0; p < n; ++p)
    if (p != r) put(&s->a, p, r, epoch, x, c);
  delay(s, k, r, 1);
  uint16_t* dst[MAX_RANKS];
  size_t len[MAX_RANKS];
  for (int q = 0; q < n; ++q) {
    dst[q] = me->stage + (size_t)q * c;
    len[q] = c;
  }
  if (take_all(s, &s->a, r, epoch, dst, len)) return 1;
  const uint16_t* src[MAX_RANKS];
  for (int q = 0; q < n; ++q) src[q] = q == r ? x : dst[q];
  uint16_t* y = output(s, k, r);
  if (s->op == SFO_ALLREDUCE) {
    for (size_t i = 0; i < c; ++i) y[i] = reduce_at(src, n, i);
  } else {
    for (int q = 0; q < n; ++q) memcpy(y + (size_t)q * c, src[q], c * sizeof(uint16_t));
  }
  return 0;
}

/* Self-synchronizing twoshot (LL or sentinel units in both phases). */
static int op_selfsync_twoshot(Shared* s, Rank* me, int k, uint32_t epoch) {
  const int n = s->nranks, r = me->rank;
  const uint16_t* x = input(s, k, r);
  const size_t lo = s->shard_lo[r], hi = s->shard_lo[r + 1], mine = hi - lo;
  for (int p = 0; p < n; ++p)
    if (p != r) put(&s->a, p, r, epoch, x + s->shard_lo[p], s->shard_lo[p + 1] - s->shard_lo[p]);
  delay(s, k, r, 1);
  uint16_t* dst[MAX_RANKS];
  size_t len[MAX_RANKS];
  for (int q = 0; q < n; ++q) {
    dst[q] = me->stage + (size_t)q * s->count;
    len[q] = mine;
  }
  if (take_all(s, &s->a, r, epoch, dst, len)) return 1;
  const uint16_t* src[MAX_RANKS];
  for (int q = 0; q < n; ++q) src[q] = q == r ? x + lo : dst[q];
  uint16_t* y = output(s, k, r);
  for (size_t i = 0; i < mine; ++i) y[lo + i] = reduce_at(src, n, i);
  for (int p = 0; p < n; ++p)
    if (p != r) put(&s->b, p, r, epoch, y + lo, mine);
  for (int q = 0; q < n; ++q) {
    dst[q] = y + s->shard_lo[q];
    len[q] = s->shard_lo[q + 1] - s->shard_lo[q];
  }
  return take_all(s, &s->b, r, epoch, dst, len);
}

/* Explicit-barrier oneshot, plain or dual-buffered, and twoshot. The input
 * is first written into the caller's buffer (one, or two alternating). */
static int op_barrier(Shared* s, Rank* me, int k, uint32_t epoch) {
  const int n = s->nranks, r = me->rank;
  const size_t c = s->count;
  const int dual = s->protocol == SFO_BARRIER_ONESHOT_DB;
  const int buf = dual ? (int)(epoch & 1u) : 0;
  uint16_t* mybuf = s->inbuf + ((size_t)r * 2 + (size_t)buf) * c;
  memcpy(mybuf, input(s, k, r), c * sizeof(uint16_t));
  if (barrier(s, 0, r, epoch)) return 1;
  delay(s, k, r, 1);
  const uint16_t* src[MAX_RANKS];
  for (int q = 0; q < n; ++q) src[q] = s->inbuf + ((size_t)q * 2 + (size_t)buf) * c;
  uint16_t* y = output(s, k, r);
  if (s->protocol != SFO_BARRIER_TWOSHOT) {
    for (size_t i = 0; i < c; ++i) y[i] = reduce_at(src, n, i);
    return dual ? 0 : barrier(s, 2, r, epoch);
  }
  /* twoshot: shard r of every input, reduced into this rank's result buffer */
  const size_t sh = (c + (size_t)n - 1) / (size_t)n;
  const int par = (int)(epoch & 1u);
  uint16_t* red_r = s->red + ((size_t)r * 2 + (size_t)par) * c;
  for (size_t i = (size_t)r * sh; i < c && i < (size_t)(r + 1) * sh; ++i) red_r[i] = reduce_at(src, n, i);
  if (barrier(s, 1, r, epoch)) return 1;
  for (int q = 0; q < n; ++q) {
    const uint16_t* red_q = s->red + ((size_t)q * 2 + (size_t)par) * c;
    for (size_t i = (size_t)q * sh; i < c && i < (size_t)(q + 1) * sh; ++i) y[i] = red_q[i];
  }
  return barrier(s, 2, r, epoch);
}

/* ------------------------------------------------------------ rank thread */

static int is_twoshot_selfsync(int p) { return p == SFO_LL_TWOSHOT || p == SFO_SENTINEL_TWOSHOT; }
static int is_barrier(int p) {
  return p == SFO_BARRIER_ONESHOT || p == SFO_BARRIER_TWOSHOT || p == SFO_BARRIER_ONESHOT_DB;
}

static void* rank_main(void* arg) {
  Rank* me = (Rank*)arg;
  Shared* s = me->s;
  while (!atomic_load_explicit(&s->start, memory_order_acquire)) {
  }
  for (int k = 0; k < s->k_ops; ++k) {
    const uint32_t epoch = (uint32_t)k + 1u;
    if (atomic_load_explicit(&s->abort_flag, memory_order_relaxed)) break;
    delay(s, k, me->rank, 0);
    int fail;
    if (is_barrier(s->protocol))
      fail = op_barrier(s, me, k, epoch);
    else if (is_twoshot_selfsync(s->protocol))
      fail = op_selfsync_twoshot(s, me, k, epoch);
    else
      fail = op_selfsync_oneshot(s, me, k, epoch);
    if (fail) break;
  }
  return NULL;
}

static size_t n_oneshot(const void* ctx, int recv, int src) {
  (void)recv;
  (void)src;
  return ((const Shared*)ctx)->count;
}
static size_t n_rs(const void* ctx, int recv, int src) {
  const Shared* s = ctx;
  (void)src;
  return s->shard_lo[recv + 1] - s->shard_lo[recv];
}
static size_t n_ag(const void* ctx, int recv, int src) {
  const Shared* s = ctx;
  (void)recv;
  return s->shard_lo[src + 1] - s->shard_lo[src];
}

/* Runs k_ops chained operations (epochs 1..k_ops) on nranks threads.
 * in: [k_ops][nranks][count] bf16 bits; out: [k_ops][nranks][count] for the
 * all-reduce, [k_ops][nranks][nranks*count] for the all-gather; skew_ns:
 * [k_ops][nranks] delays (or NULL), applied before each operation
 * (skew_after = 0) or between a rank's pushes / top barrier and its reads
 * (skew_after = 1). *seconds gets the wall time from the start signal until
 * every rank finished. Returns SFO_*. */
int sfo_threaded_chain(int protocol, int op, int nranks, size_t count, int k_ops, const uint16_t* in,
                       uint16_t* out, const uint32_t* skew_ns, int skew_after, double timeout_s, int yield_polls,
                       double* seconds) {
  if (nranks < 2 || nranks > MAX_RANKS || k_ops < 0 || !in || !out || count == 0) return SFO_EINVAL;
  if (protocol < SFO_LL || protocol > SFO_SENTINEL_TWOSHOT) return SFO_EINVAL;
  if (op != SFO_ALLREDUCE && op != SFO_ALLGATHER) return SFO_EINVAL;
  if (op == SFO_ALLGATHER && (is_barrier(protocol) || is_twoshot_selfsync(protocol))) return SFO_EINVAL;
  if (skew_after != 0 && skew_after != 1) return SFO_EINVAL;
  Shared* s = calloc(1, sizeof(Shared));
  if (!s) return SFO_ENOMEM;
  s->protocol = protocol;
  s->op = op;
  s->nranks = nranks;
  s->k_ops = k_ops;
  s->count = count;
  s->in = in;
  s->out = out;
  s->skew_ns = skew_ns;
  s->skew_after = skew_after;
  s->timeout_ns = (uint64_t)(timeout_s * 1e9);
  s->yield_polls = yield_polls;
  for (int q = 0; q < 3; ++q)
    for (int r = 0; r < MAX_RANKS; ++r) atomic_init(&s->bar[q][r], 0);
  atomic_init(&s->abort_flag, 0);
  atomic_init(&s->start, 0);
  atomic_init(&s->status, SFO_OK);
  /* twoshot shards: whole 8-element vectors, ceil(ceil(count / 8) / N) each */
  const size_t nvec = (count + VEC - 1) / VEC, per = (nvec + (size_t)nranks - 1) / (size_t)nranks;
  for (int q = 0; q <= nranks; ++q) {
    size_t lo = (size_t)q * per * VEC;
    s->shard_lo[q] = lo < count ? lo : count;
  }
  int rc = SFO_OK;
  if (protocol == SFO_LL || protocol == SFO_LL128 || protocol == SFO_SENTINEL) {
    if (slots_init(&s->a, protocol, nranks, count)) rc = SFO_ENOMEM;
  } else if (is_twoshot_selfsync(protocol)) {
    const int enc = protocol == SFO_LL_TWOSHOT ? SFO_LL : SFO_SENTINEL;
    if (slots_init(&s->a, enc, nranks, per * VEC) || slots_init(&s->b, enc, nranks, per * VEC)) rc = SFO_ENOMEM;
  } else {
    s->inbuf = calloc((size_t)nranks * 2 * count, sizeof(uint16_t));
    s->red = calloc((size_t)nranks * 2 * count, sizeof(uint16_t));
    if (!s->inbuf || !s->red) rc = SFO_ENOMEM;
  }
  Rank ranks[MAX_RANKS];
  pthread_t th[MAX_RANKS];
  int started = 0;
  for (int r = 0; r < nranks && rc == SFO_OK; ++r) {
    ranks[r].s = s;
    ranks[r].rank = r;
    ranks[r].stage = malloc((size_t)nranks * count * sizeof(uint16_t));
    if (!ranks[r].stage) {
      rc = SFO_ENOMEM;
      break;
    }
    if (pthread_create(&th[r], NULL, rank_main, &ranks[r]) != 0) {
      free(ranks[r].stage);
      rc = SFO_ETHREAD;
      break;
    }
    ++started;
  }
  if (rc != SFO_OK) atomic_store(&s->abort_flag, 1);
  const uint64_t t0 = now_ns();
  atomic_store_explicit(&s->start, 1, memory_order_release);
  for (int r = 0; r < started; ++r) pthread_join(th[r], NULL);
  const uint64_t t1 = now_ns();
  if (seconds) *seconds = (double)(t1 - t0) * 1e-9;
  for (int r = 0; r < started; ++r) free(ranks[r].stage);
  if (rc == SFO_OK) rc = atomic_load(&s->status);
  if (rc == SFO_OK && (protocol == SFO_LL || protocol == SFO_LL128 || protocol == SFO_SENTINEL))
    rc = slots_check(&s->a, k_ops, n_oneshot, s);
  if (rc == SFO_OK && is_twoshot_selfsync(protocol)) {
    rc = slots_check(&s->a, k_ops, n_rs, s);
    if (rc == SFO_OK) rc = slots_check(&s->b, k_ops, n_ag, s);
  }
  slots_free(&s->a);
  slots_free(&s->b);
  free(s->inbuf);
  free(s->red);
  free(s);
  return rc;
}
