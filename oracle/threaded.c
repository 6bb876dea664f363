/* Concurrent CPU model of the self-synchronizing all-reduce and all-gather.
 *
 * TEST INFRASTRUCTURE ONLY: only tests/ and the CPU-baseline leg of bench.py
 * load it (through oracle/threaded.py). It shares no code with the CUDA
 * library and is independent of the Python oracle too: plain C11, one POSIX
 * thread per rank, C11 atomics for every shared word.
 *
 * What it models ("Why Microseconds Matter in AI Infrastructure", section
 * "Latency can matter more than bandwidth"; "flash-comm: Self-Synchronizing
 * Collective Communication for LLM Decoding", abstract; "SiFAR:
 * Synchronization-Free All-Reduce for Low-Latency LLM Inference", abstract):
 *
 *  - every rank pushes its chunk into each peer's receive slot
 *    slot[recv][epoch & 1][src], and the receiver validates units on their own:
 *      LL       8-byte unit = 32-bit data word (bf16 2j low, 2j+1 high) and a
 *               32-bit flag equal to the epoch, written as one atomic store;
 *      LL128    128-byte line = 15 data words (60 bf16) and a flag word; the
 *               data words are stored first and the flag last with release
 *               order, the reader acquires the flag before the data;
 *      sentinel raw bf16 elements into a slot pre-filled with 0xFFFF; the
 *               reader takes an element once it differs from 0xFFFF and
 *               writes 0xFFFF back before it pushes its next epoch;
 *  - epoch-parity double buffering with no bottom barrier: a writer reaches
 *    epoch e+2 of a slot only after it received e+1 from the slot's reader,
 *    which that reader pushed after it finished epoch e (release stores on
 *    the pushes, acquire loads on the polls carry the order);
 *  - the explicit-barrier oneshot for comparison: a top barrier, a direct
 *    read of every rank's input, a bottom barrier;
 *  - the reduction: fp32 round-to-nearest adds in rank order 0..N-1 starting
 *    from rank 0's value, one final rounding to bf16 (ties to even), so all
 *    ranks produce the same bits whatever order the units arrived in.
 *
 * Floating point: binary32 adds only, built with -ffp-contract=off on an
 * SSE target (no excess precision, no flush-to-zero).
 */
#define _GNU_SOURCE
#include <pthread.h>
#include <sched.h>
#include <stdatomic.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <time.h>

enum { SFO_LL = 1, SFO_LL128 = 2, SFO_SENTINEL = 3, SFO_BARRIER_ONESHOT = 4 };
enum { SFO_ALLREDUCE = 0, SFO_ALLGATHER = 1 };
enum {
  SFO_OK = 0,
  SFO_EINVAL = 1,
  SFO_ETIMEOUT = 2,
  SFO_EPOST = 3, /* a slot was not left as the protocol requires */
  SFO_ENOMEM = 4,
  SFO_ETHREAD = 5
};

#define SENTINEL_BITS 0xFFFFu
#define LL128_WORDS 16     /* 8-byte words per 128-byte line */
#define LL128_ELEMS 60     /* bf16 elements per line (15 data words) */

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

/* ------------------------------------------------------------ shared state */

typedef struct {
  int protocol, op, nranks, k_ops;
  size_t count;
  const uint16_t* in;   /* [k][N][count] */
  uint16_t* out;        /* [k][N][count] (all-reduce) or [k][N][N*count] */
  const uint32_t* skew_ns; /* [k][N] or NULL */
  uint64_t timeout_ns;
  size_t units;         /* per (recv, parity, src) slot */
  /* one of the following holds the slots, [recv][parity][src][units] */
  _Atomic uint64_t* ll;     /* LL units, or LL128 lines as 16 words each */
  _Atomic uint16_t* sent;   /* sentinel elements */
  _Atomic uint32_t* bar_top; /* [N] barrier arrivals (epochs) */
  _Atomic uint32_t* bar_bot;
  _Atomic int abort_flag;
  _Atomic int start;
  _Atomic int status;
  int yield_polls;      /* yield the core while polling (more threads than cores) */
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

static void spin_until(uint64_t t) {
  while (now_ns() < t) {
  }
}

/* A bounded wait: called once per unsuccessful poll. Returns nonzero when the
 * caller must give up (deadline passed or another rank gave up). */
typedef struct {
  uint64_t deadline;
  unsigned polls;
} Wait;

static void cpu_relax(void) {
#if defined(__x86_64__) || defined(__i386__)
  __builtin_ia32_pause();
#elif defined(__aarch64__)
  __asm__ __volatile__("yield");
#endif
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

static size_t slot_index(const Shared* s, int recv, int parity, int src) {
  return (((size_t)recv * 2 + (size_t)parity) * (size_t)s->nranks + (size_t)src) * s->units;
}

static const uint16_t* input(const Shared* s, int k, int r) {
  return s->in + ((size_t)k * s->nranks + r) * s->count;
}

/* ------------------------------------------------------------ push */

static void push(Shared* s, int r, int k, uint32_t epoch) {
  const uint16_t* x = input(s, k, r);
  const int parity = (int)(epoch & 1u);
  for (int p = 0; p < s->nranks; ++p) {
    if (p == r) continue;
    const size_t base = slot_index(s, p, parity, r);
    if (s->protocol == SFO_LL) {
      for (size_t j = 0; j < s->units; ++j) {
        uint32_t lo = x[2 * j];
        uint32_t hi = (2 * j + 1 < s->count) ? x[2 * j + 1] : 0u;
        uint64_t unit = (uint64_t)(lo | (hi << 16)) | ((uint64_t)epoch << 32);
        atomic_store_explicit(&s->ll[base + j], unit, memory_order_release);
      }
    } else if (s->protocol == SFO_LL128) {
      for (size_t line = 0; line < s->units / LL128_WORDS; ++line) {
        _Atomic uint64_t* w = &s->ll[base + line * LL128_WORDS];
        for (int d = 0; d < LL128_WORDS - 1; ++d) {
          uint64_t word = 0;
          for (int h = 0; h < 4; ++h) {
            size_t i = line * LL128_ELEMS + (size_t)d * 4 + (size_t)h;
            if (i < s->count) word |= (uint64_t)x[i] << (16 * h);
          }
          atomic_store_explicit(&w[d], word, memory_order_relaxed);
        }
        atomic_store_explicit(&w[LL128_WORDS - 1], (uint64_t)epoch, memory_order_release);
      }
    } else { /* sentinel */
      for (size_t i = 0; i < s->count; ++i)
        atomic_store_explicit(&s->sent[base + i], x[i], memory_order_release);
    }
  }
}

/* ------------------------------------------------------------ poll */

/* Waits until every unit of every source validates for `epoch`, decoding
 * into stage[q]; sources are visited round-robin and each pass takes whatever
 * has arrived, so the arrival order is free. Returns nonzero on give-up. */
static int poll_all(Shared* s, Rank* me, uint32_t epoch) {
  const int n = s->nranks, r = me->rank, parity = (int)(epoch & 1u);
  size_t* done = calloc((size_t)n, sizeof(size_t));
  if (!done) return 1;
  int remaining = n - 1;
  Wait w = {now_ns() + s->timeout_ns, 0};
  while (remaining > 0) {
    int progressed = 0;
    for (int q = 0; q < n; ++q) {
      if (q == r || done[q] == s->units) continue;
      const size_t base = slot_index(s, r, parity, q);
      uint16_t* dst = me->stage + (size_t)q * s->count;
      size_t j = done[q];
      if (s->protocol == SFO_LL) {
        for (; j < s->units; ++j) {
          uint64_t unit = atomic_load_explicit(&s->ll[base + j], memory_order_acquire);
          if ((uint32_t)(unit >> 32) != epoch) break;
          dst[2 * j] = (uint16_t)(unit & 0xFFFFu);
          if (2 * j + 1 < s->count) dst[2 * j + 1] = (uint16_t)((unit >> 16) & 0xFFFFu);
        }
      } else if (s->protocol == SFO_LL128) {
        for (; j < s->units; j += LL128_WORDS) {
          _Atomic uint64_t* line = &s->ll[base + j];
          if (atomic_load_explicit(&line[LL128_WORDS - 1], memory_order_acquire) != (uint64_t)epoch) break;
          size_t first = (j / LL128_WORDS) * LL128_ELEMS;
          for (int d = 0; d < LL128_WORDS - 1; ++d) {
            uint64_t word = atomic_load_explicit(&line[d], memory_order_relaxed);
            for (int h = 0; h < 4; ++h) {
              size_t i = first + (size_t)d * 4 + (size_t)h;
              if (i < s->count) dst[i] = (uint16_t)(word >> (16 * h));
            }
          }
        }
      } else { /* sentinel: take the element, then put the pre-fill back */
        for (; j < s->units; ++j) {
          uint16_t v = atomic_load_explicit(&s->sent[base + j], memory_order_acquire);
          if (v == SENTINEL_BITS) break;
          dst[j] = v;
          atomic_store_explicit(&s->sent[base + j], (uint16_t)SENTINEL_BITS, memory_order_relaxed);
        }
      }
      if (j != done[q]) progressed = 1;
      done[q] = j;
      if (j == s->units) --remaining;
    }
    if (!progressed && remaining > 0 && wait_more(s, &w)) {
      free(done);
      return 1;
    }
  }
  free(done);
  return 0;
}

/* ------------------------------------------------------------ barriers */

static int barrier(Shared* s, _Atomic uint32_t* bar, int r, uint32_t epoch) {
  atomic_store_explicit(&bar[r], epoch, memory_order_release);
  Wait w = {now_ns() + s->timeout_ns, 0};
  for (int q = 0; q < s->nranks; ++q)
    while (atomic_load_explicit(&bar[q], memory_order_acquire) < epoch)
      if (wait_more(s, &w)) return 1;
  return 0;
}

/* ------------------------------------------------------------ reduce / copy */

static void finish(Shared* s, Rank* me, int k, int from_stage) {
  const int n = s->nranks, r = me->rank;
  const size_t c = s->count;
  const uint16_t* src[8];
  for (int q = 0; q < n; ++q)
    src[q] = (q == r || !from_stage) ? input(s, k, q) : me->stage + (size_t)q * c;
  if (s->op == SFO_ALLREDUCE) {
    uint16_t* y = s->out + ((size_t)k * n + r) * c;
    for (size_t i = 0; i < c; ++i) {
      float acc = widen(src[0][i]);
      for (int q = 1; q < n; ++q) acc = acc + widen(src[q][i]);
      y[i] = narrow(acc);
    }
  } else {
    uint16_t* y = s->out + ((size_t)k * n + r) * (size_t)n * c;
    for (int q = 0; q < n; ++q) memcpy(y + (size_t)q * c, src[q], c * sizeof(uint16_t));
  }
}

/* ------------------------------------------------------------ rank thread */

static void* rank_main(void* arg) {
  Rank* me = (Rank*)arg;
  Shared* s = me->s;
  while (!atomic_load_explicit(&s->start, memory_order_acquire)) {
  }
  for (int k = 0; k < s->k_ops; ++k) {
    const uint32_t epoch = (uint32_t)k + 1u;
    if (atomic_load_explicit(&s->abort_flag, memory_order_relaxed)) break;
    if (s->skew_ns) spin_until(now_ns() + s->skew_ns[(size_t)k * s->nranks + me->rank]);
    if (s->protocol == SFO_BARRIER_ONESHOT) {
      if (barrier(s, s->bar_top, me->rank, epoch)) break;
      finish(s, me, k, 0);
      if (barrier(s, s->bar_bot, me->rank, epoch)) break;
    } else {
      push(s, me->rank, k, epoch);
      if (poll_all(s, me, epoch)) break;
      finish(s, me, k, 1);
    }
  }
  return NULL;
}

/* After a chain every sentinel slot holds the pre-fill again, and every LL /
 * LL128 slot last written holds that epoch's flag. */
static int check_slots(const Shared* s) {
  const int n = s->nranks;
  for (int r = 0; r < n; ++r)
    for (int parity = 0; parity < 2; ++parity)
      for (int q = 0; q < n; ++q) {
        if (q == r) continue;
        const size_t base = slot_index(s, r, parity, q);
        /* the last epoch of this parity, or 0 when it was never written */
        uint32_t last = (uint32_t)s->k_ops;
        if ((last & 1u) != (uint32_t)parity) last = last >= 1 ? last - 1 : 0;
        if (s->protocol == SFO_SENTINEL) {
          for (size_t i = 0; i < s->units; ++i)
            if (atomic_load(&s->sent[base + i]) != SENTINEL_BITS) return SFO_EPOST;
        } else if (s->protocol == SFO_LL) {
          for (size_t j = 0; j < s->units; ++j)
            if ((uint32_t)(atomic_load(&s->ll[base + j]) >> 32) != last) return SFO_EPOST;
        } else if (s->protocol == SFO_LL128) {
          for (size_t j = LL128_WORDS - 1; j < s->units; j += LL128_WORDS)
            if (atomic_load(&s->ll[base + j]) != (uint64_t)last) return SFO_EPOST;
        }
      }
  return SFO_OK;
}

/* Runs k_ops chained operations (epochs 1..k_ops) on nranks threads.
 * in: [k_ops][nranks][count] bf16 bits; out: [k_ops][nranks][count] for the
 * all-reduce, [k_ops][nranks][nranks*count] for the all-gather; skew_ns:
 * [k_ops][nranks] delays before each rank's push (or NULL). *seconds gets the
 * wall time from the start signal until every rank finished. Returns SFO_*. */
int sfo_threaded_chain(int protocol, int op, int nranks, size_t count, int k_ops, const uint16_t* in,
                       uint16_t* out, const uint32_t* skew_ns, double timeout_s, int yield_polls,
                       double* seconds) {
  if (nranks < 2 || nranks > 8 || k_ops < 0 || !in || !out || count == 0) return SFO_EINVAL;
  if (protocol < SFO_LL || protocol > SFO_BARRIER_ONESHOT) return SFO_EINVAL;
  if (op != SFO_ALLREDUCE && op != SFO_ALLGATHER) return SFO_EINVAL;
  if (op == SFO_ALLGATHER && protocol == SFO_BARRIER_ONESHOT) return SFO_EINVAL;
  Shared s;
  memset(&s, 0, sizeof s);
  s.protocol = protocol;
  s.op = op;
  s.nranks = nranks;
  s.k_ops = k_ops;
  s.count = count;
  s.in = in;
  s.out = out;
  s.skew_ns = skew_ns;
  s.timeout_ns = (uint64_t)(timeout_s * 1e9);
  s.yield_polls = yield_polls;
  const size_t slots = (size_t)nranks * 2 * (size_t)nranks;
  int rc = SFO_OK;
  if (protocol == SFO_LL) {
    s.units = (count + 1) / 2;
  } else if (protocol == SFO_LL128) {
    s.units = (count + LL128_ELEMS - 1) / LL128_ELEMS * LL128_WORDS;
  } else if (protocol == SFO_SENTINEL) {
    s.units = count;
  }
  if (protocol == SFO_LL || protocol == SFO_LL128) {
    s.ll = calloc(slots * s.units, sizeof(*s.ll)); /* zero: never a valid epoch */
    if (!s.ll) return SFO_ENOMEM;
    for (size_t i = 0; i < slots * s.units; ++i) atomic_init(&s.ll[i], 0);
  } else if (protocol == SFO_SENTINEL) {
    s.sent = malloc(slots * s.units * sizeof(*s.sent));
    if (!s.sent) return SFO_ENOMEM;
    for (size_t i = 0; i < slots * s.units; ++i) atomic_init(&s.sent[i], (uint16_t)SENTINEL_BITS);
  } else {
    s.bar_top = calloc((size_t)nranks, sizeof(*s.bar_top));
    s.bar_bot = calloc((size_t)nranks, sizeof(*s.bar_bot));
    if (!s.bar_top || !s.bar_bot) rc = SFO_ENOMEM;
  }
  Rank ranks[8];
  pthread_t th[8];
  int started = 0;
  for (int r = 0; r < nranks && rc == SFO_OK; ++r) {
    ranks[r].s = &s;
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
  if (rc != SFO_OK) atomic_store(&s.abort_flag, 1);
  const uint64_t t0 = now_ns();
  atomic_store_explicit(&s.start, 1, memory_order_release);
  for (int r = 0; r < started; ++r) pthread_join(th[r], NULL);
  const uint64_t t1 = now_ns();
  if (seconds) *seconds = (double)(t1 - t0) * 1e-9;
  for (int r = 0; r < started; ++r) free(ranks[r].stage);
  if (rc == SFO_OK) rc = atomic_load(&s.status);
  if (rc == SFO_OK) rc = check_slots(&s);
  free(s.ll);
  free(s.sent);
  free(s.bar_top);
  free(s.bar_bot);
  return rc;
}
