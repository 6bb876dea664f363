"""Step-by-step simulator of the N-rank protocols over a byte-level memory.

Self-synchronizing protocols (LL, LL128, sentinel), after "flash-comm:
Self-Synchronizing Collective Communication for LLM Decoding", abstract, and
"Why Microseconds Matter in AI Infrastructure", section "Latency can matter
more than bandwidth":

* every rank keeps a receive slot per (parity, source) in its own scratch;
* at epoch e a rank *pushes* the units of its input into each peer's slot at
  parity e & 1 (the sender writes into the receiver's memory -- the plainest
  reading of "receivers directly validate the blocks they need");
* it *polls* its own slots, accepting every unit that validates for epoch e,
  in whatever order they land;
* when every unit of every source is in, it reduces in fixed rank order
  0..N-1 (own contribution read from its input) and writes its output;
* sentinel only: it writes the sentinel back over the slots it consumed, and
  those writes land before its next push;
* then it moves to epoch e+1. There is no barrier: the double buffer (two
  parities) makes a peer's receipt of data the evidence that the other buffer
  may be reused (same page, same section, on double buffering).

Explicit-barrier baselines (pull), after "SiFAR: Synchronization-Free
All-Reduce for Low-Latency LLM Inference", abstract:

* oneshot: produce input, top barrier, pull every peer's input and reduce,
  bottom barrier (the bottom barrier guards the write-after-write on the input
  buffer that the next operation's producer overwrites);
* twoshot: produce, top barrier, reduce-scatter (rank r reduces shard r from
  every input into its reduction buffer), middle barrier, all-gather (pull
  every reduced shard), bottom barrier.

A scheduler decides which enabled action happens next: a pending store
lands, or a rank takes its next step (push / poll / barrier arrive / pull).
Stores are atomic per unit (8-byte LL unit, 128-byte LL128 line, 2-byte
sentinel element). Every memory unit carries a shadow tag (writer, epoch) so
that the checks below can tell stale data from fresh data:

* no unit is accepted unless its shadow says (expected source, current epoch);
* no store lands over a unit whose previous epoch the receiver has not yet
  consumed (at most one outstanding epoch per parity per slot);
* no rank waits forever (deadlock = no enabled action while a rank is not done);
* every output equals the closed form, and the N outputs of an operation are
  identical;
* after the chain every sentinel slot is back to the sentinel and every LL /
  LL128 flag in a parity's slot equals the last epoch that used that parity;
* no delivered element is the sentinel pattern.

The ``bug`` argument plants a known mistake so that tests can prove the checks
catch it: ``single_buffer`` (ignore parity), ``no_reset`` (sentinel not
rewritten), ``arrival_order`` (reduce in arrival order instead of rank order),
``no_bottom_barrier``, ``no_top_barrier``, ``no_mid_barrier`` (barrier
baselines).

Observation from this model: in the pull twoshot the middle barrier of
operation k and the top barrier of k+1 already order every reuse of the
input and reduction buffers, so dropping the twoshot bottom barrier breaks no
check here; the baseline keeps it because the SiFAR abstract describes
twoshot with a bottom barrier it cannot avoid.
"""

import copy

import numpy as np

from . import protocols as P
from . import reference
from .bf16 import BF16_SENTINEL, bf16_bits_to_f32, f32_to_bf16_bits

__all__ = ["ChainSim", "run_chain", "run_fifo", "BARRIER_ONESHOT", "BARRIER_TWOSHOT", "BARRIER_ONESHOT_DB",
           "ALL_PROTOCOLS"]

BARRIER_ONESHOT = "barrier_oneshot"
BARRIER_TWOSHOT = "barrier_twoshot"
# SiFAR's oneshot with dual-buffered inputs: the caller alternates two input
# buffers per rank (operation k writes buffer k % 2), so no bottom barrier
BARRIER_ONESHOT_DB = "barrier_oneshot_db"
BARRIER_PROTOCOLS = (BARRIER_ONESHOT, BARRIER_TWOSHOT, BARRIER_ONESHOT_DB)
ALL_PROTOCOLS = P.SELF_SYNC + BARRIER_PROTOCOLS

ALLREDUCE = "allreduce"
ALLGATHER = "allgather"


class _Rank:
    """Per-rank protocol state (plain data, copyable)."""

    def __init__(self, n, units):
        self.op = 0               # index of the operation in progress
        self.phase = "push"       # self-sync: push | poll | done
        self.accepted = {}        # src -> bool[units]
        self.staged = {}          # src -> uint16[count]
        self.arrival = []         # sources in completion order
        self.done_epoch = 0       # last epoch fully consumed
        self.pulled = {}          # barrier: src -> data pulled for this op
        self.red = None           # twoshot: reduced shard
        self.n = n
        self.units = units


class ChainSim:
    """K chained collectives on N emulated ranks.

    ``inputs``: uint16 [K, N, count] bf16 bit patterns, one input per
    (operation, rank). ``proto``: one of ``ALL_PROTOCOLS``. ``op``:
    ``"allreduce"`` or ``"allgather"``.
    """

    def __init__(self, proto, inputs, op=ALLREDUCE, first_epoch=1, bug=None, sentinel_reset="after_all"):
        x = np.asarray(inputs, dtype=np.uint16)
        if sentinel_reset not in ("after_all", "on_accept"):
            raise ValueError(sentinel_reset)
        # when the sentinel reader writes the fill back: after every source of
        # the epoch is in ("after_all", the page's order: consume, then reset)
        # or in the same atomic step that accepts each unit ("on_accept")
        self.sentinel_reset = sentinel_reset
        if x.ndim != 3:
            raise ValueError("inputs must be [K, N, count]")
        self.proto = proto
        self.op = op
        self.inputs = x
        self.K, self.N, self.count = x.shape
        if self.N < 2:
            raise ValueError("need at least two ranks")
        self.first_epoch = first_epoch
        self.bug = bug
        self.violations = []
        self.steps = 0
        out_len = self.count if op == ALLREDUCE else self.N * self.count
        self.outputs = np.zeros((self.K, self.N, out_len), dtype=np.uint16)
        self.completed = np.zeros((self.K, self.N), dtype=bool)
        self.pending = []  # list of store records (dicts)
        if proto in P.SELF_SYNC:
            self._init_self_sync()
        elif proto in BARRIER_PROTOCOLS:
            if proto == BARRIER_TWOSHOT and op != ALLREDUCE:
                raise ValueError("twoshot is an all-reduce algorithm")
            self._init_barrier()
        else:
            raise ValueError(proto)

    # ------------------------------------------------------------------ setup
    def _init_self_sync(self):
        units = P.unit_count(self.proto, self.count)
        self.units = units
        self.mem = {}
        self.shadow = {}
        for r in range(self.N):
            for par in (0, 1):
                for q in range(self.N):
                    if q == r:
                        continue
                    self.mem[(r, par, q)] = P.initial_slot(self.proto, self.count)
                    self.shadow[(r, par, q)] = [None] * units
        self.ranks = [_Rank(self.N, units) for _ in range(self.N)]
        for r in range(self.N):
            self._begin_op(r)

    def _init_barrier(self):
        self.units = 0
        self.ranks = [_Rank(self.N, 0) for _ in range(self.N)]
        self.bar = [0] * self.N
        # input buffer of each rank: (op index it holds, data); the producer
        # of operation k writes it when the rank starts operation k.
        self.inbuf = [[(-1, np.zeros(self.count, dtype=np.uint16)) for _ in range(2)] for _ in range(self.N)]
        shard = -(-self.count // self.N)
        self.shard = shard
        self.redbuf = [(-1, np.zeros(shard, dtype=np.uint16)) for _ in range(self.N)]
        for rk in self.ranks:
            rk.phase = "produce"

    def _epoch(self, k):
        return self.first_epoch + k

    def _parity(self, e):
        if self.bug == "single_buffer":
            return 0
        return e & 1

    def _begin_op(self, r):
        rk = self.ranks[r]
        rk.accepted = {}
        rk.staged = {}
        rk.arrival = []
        for q in range(self.N):
            if q == r:
                continue
            rk.accepted[q] = np.zeros(self.units, dtype=bool)
            rk.staged[q] = np.zeros(self.count, dtype=np.uint16)
        rk.phase = "push" if rk.op < self.K else "done"

    # ------------------------------------------------------------- interface
    def enabled_actions(self):
        acts = []
        for r, rk in enumerate(self.ranks):
            if rk.phase == "done":
                continue
            if self.proto in P.SELF_SYNC:
                # a poll that would accept nothing leaves the state unchanged,
                # so only productive polls count as actions; a state where no
                # action is left while a rank is unfinished is a deadlock
                if rk.phase == "push" or self._poll_would_progress(r):
                    acts.append(("step", r))
            else:
                if self._barrier_can_step(r):
                    acts.append(("step", r))
        for i in range(len(self.pending)):
            acts.append(("land", i))
        return acts

    def finished(self):
        return all(rk.phase == "done" for rk in self.ranks)

    def apply(self, act):
        self.steps += 1
        kind, arg = act
        if kind == "land":
            self._land(self.pending.pop(arg))
        elif self.proto in P.SELF_SYNC:
            self._self_sync_step(arg)
        else:
            self._barrier_step(arg)

    def clone(self):
        return copy.deepcopy(self)

    def state_key(self):
        """Hashable summary of the whole state (for exhaustive search)."""
        parts = []
        if self.proto in P.SELF_SYNC:
            for key in sorted(self.mem):
                parts.append(self.mem[key].tobytes())
                parts.append(tuple(self.shadow[key]))
            for rk in self.ranks:
                acc = tuple(rk.accepted[q].tobytes() for q in sorted(rk.accepted))
                stg = tuple(rk.staged[q].tobytes() for q in sorted(rk.staged))
                parts.append((rk.op, rk.phase, acc, stg, tuple(rk.arrival)))
        else:
            for rk in self.ranks:
                parts.append((rk.op, rk.phase, tuple(sorted(rk.pulled))))
            parts.append(tuple(self.bar))
            parts.append(tuple(b[0] for bufs in self.inbuf for b in bufs))
            parts.append(tuple(b[0] for b in self.redbuf))
        pend = sorted((s["dst"], s["par"], s["src"], s["j"], s["epoch"]) for s in self.pending)
        parts.append(tuple(pend))
        return tuple(parts)

    # ------------------------------------------------------- self-sync steps
    def _self_sync_step(self, r):
        rk = self.ranks[r]
        if rk.phase == "push":
            self._push(r)
            rk.phase = "poll"
        elif rk.phase == "poll":
            self._poll(r)

    def _push(self, r):
        rk = self.ranks[r]
        k = rk.op
        e = self._epoch(k)
        par = self._parity(e)
        data = self.inputs[k, r]
        for p in range(self.N):
            if p == r:
                continue
            for j, (off, body) in enumerate(P.encode_all(self.proto, data, e)):
                self.pending.append(dict(dst=p, par=par, src=r, j=j, off=off,
                                         body=body, epoch=e))

    def _land(self, s):
        key = (s["dst"], s["par"], s["src"])
        prev = self.shadow[key][s["j"]]
        reader = self.ranks[s["dst"]]
        if prev is not None and prev[1] != s["epoch"] and reader.done_epoch < prev[1]:
            self.violations.append(
                f"store of epoch {s['epoch']} from rank {s['src']} overwrote unit {s['j']} "
                f"of rank {s['dst']}'s slot still holding unconsumed epoch {prev[1]}")
        if self.bug != "single_buffer" and (s["epoch"] & 1) != s["par"]:
            self.violations.append("store landed in the wrong parity")
        buf = self.mem[key]
        off = s["off"]
        buf[off:off + s["body"].size] = s["body"]
        self.shadow[key][s["j"]] = (s["src"], s["epoch"])

    def _poll_would_progress(self, r):
        rk = self.ranks[r]
        e = self._epoch(rk.op)
        par = self._parity(e)
        for q, acc in rk.accepted.items():
            slot = self.mem[(r, par, q)]
            for j in range(self.units):
                if not acc[j] and P.validate_unit(self.proto, slot, j, e):
                    return True
        return self.units == 0

    def _poll(self, r):
        rk = self.ranks[r]
        k = rk.op
        e = self._epoch(k)
        par = self._parity(e)
        for q in range(self.N):
            if q == r:
                continue
            acc = rk.accepted[q]
            if acc.all():
                continue
            slot = self.mem[(r, par, q)]
            for j in range(self.units):
                if acc[j] or not P.validate_unit(self.proto, slot, j, e):
                    continue
                tag = self.shadow[(r, par, q)][j]
                if tag != (q, e):
                    self.violations.append(
                        f"rank {r} epoch {e} accepted unit {j} from source {q} "
                        f"tagged {tag}")
                lo, vals = P.decode_unit(self.proto, slot, j, self.count)
                rk.staged[q][lo:lo + vals.size] = vals
                acc[j] = True
                if self.proto == P.SENTINEL and self.sentinel_reset == "on_accept" and self.bug != "no_reset":
                    off, body = P.reset_unit_bytes(self.proto, j)
                    slot[off:off + body.size] = body
                    self.shadow[(r, par, q)][j] = None
            if acc.all():
                rk.arrival.append(q)
        if all(rk.accepted[q].all() for q in rk.accepted):
            self._finish_self_sync(r)

    def _finish_self_sync(self, r):
        rk = self.ranks[r]
        k = rk.op
        e = self._epoch(k)
        par = self._parity(e)
        rows = {q: rk.staged[q] for q in rk.staged}
        rows[r] = self.inputs[k, r]
        if self.op == ALLREDUCE:
            if self.bug == "arrival_order":
                order = [r] + rk.arrival  # own first, then as they came in
            else:
                order = list(range(self.N))
            acc = bf16_bits_to_f32(rows[order[0]]).copy()
            for q in order[1:]:
                acc = np.add(acc, bf16_bits_to_f32(rows[q]), dtype=np.float32)
            self.outputs[k, r] = f32_to_bf16_bits(acc)
        else:
            self.outputs[k, r] = np.concatenate([rows[q] for q in range(self.N)])
        self.completed[k, r] = True
        if self.proto == P.SENTINEL and self.bug != "no_reset" and self.sentinel_reset == "after_all":
            for q in range(self.N):
                if q == r:
                    continue
                buf = self.mem[(r, par, q)]
                for j in range(self.units):
                    off, body = P.reset_unit_bytes(self.proto, j)
                    buf[off:off + body.size] = body
                    self.shadow[(r, par, q)][j] = None
        rk.done_epoch = e
        rk.op += 1
        self._begin_op(r)

    # --------------------------------------------------------- barrier steps
    def _bar_target(self, e, phase):
        return (e << 2) | phase

    def _barrier_can_step(self, r):
        rk = self.ranks[r]
        e = self._epoch(rk.op)
        ph = rk.phase
        if ph.startswith("wait"):
            phase = {"wait_top": 1, "wait_mid": 2, "wait_bottom": 3}[ph]
            target = self._bar_target(e, phase)
            return all(self.bar[q] >= target for q in range(self.N))
        return True

    def _barrier_step(self, r):
        rk = self.ranks[r]
        k = rk.op
        e = self._epoch(k)
        N = self.N
        ph = rk.phase
        if ph == "produce":
            # the producer of operation k overwrites this rank's input buffer
            self.inbuf[r][self._inslot(k)] = (k, self.inputs[k, r].copy())
            rk.pulled = {}
            rk.phase = "arrive_top"
        elif ph == "arrive_top":
            self.bar[r] = self._bar_target(e, 1)
            rk.phase = "pull" if self.bug == "no_top_barrier" else "wait_top"
        elif ph == "wait_top":
            rk.phase = "pull"
        elif ph == "pull":
            if self.proto in (BARRIER_ONESHOT, BARRIER_ONESHOT_DB):
                src = next(q for q in range(N) if q not in rk.pulled)
                tag, data = self.inbuf[src][self._inslot(k)]
                if tag != k:
                    self.violations.append(
                        f"rank {r} op {k} pulled rank {src}'s input holding op {tag}")
                rk.pulled[src] = data.copy()
                if len(rk.pulled) == N:
                    rows = np.stack([rk.pulled[q] for q in range(N)])
                    if self.op == ALLREDUCE:
                        self.outputs[k, r] = reference.allreduce(rows)
                    else:
                        self.outputs[k, r] = rows.reshape(-1)
                    self.completed[k, r] = True
                    rk.phase = "next" if self.proto == BARRIER_ONESHOT_DB else "arrive_bottom"
            else:  # twoshot reduce-scatter: shard r of every input
                src = next(q for q in range(N) if q not in rk.pulled)
                tag, data = self.inbuf[src][self._inslot(k)]
                if tag != k:
                    self.violations.append(
                        f"rank {r} op {k} pulled rank {src}'s input holding op {tag}")
                lo, hi = self._shard_range(r)
                rk.pulled[src] = data[lo:hi].copy()
                if len(rk.pulled) == N:
                    rows = np.stack([rk.pulled[q] for q in range(N)])
                    red = reference.allreduce(rows) if hi > lo else np.zeros(0, np.uint16)
                    buf = np.zeros(self.shard, dtype=np.uint16)
                    buf[: hi - lo] = red
                    self.redbuf[r] = (k, buf)
                    rk.pulled = {}
                    rk.phase = "arrive_mid"
        elif ph == "arrive_mid":
            self.bar[r] = self._bar_target(e, 2)
            rk.phase = "gather" if self.bug == "no_mid_barrier" else "wait_mid"
        elif ph == "wait_mid":
            rk.phase = "gather"
        elif ph == "gather":
            src = next(q for q in range(N) if q not in rk.pulled)
            tag, data = self.redbuf[src]
            if tag != k:
                self.violations.append(
                    f"rank {r} op {k} gathered rank {src}'s shard holding op {tag}")
            rk.pulled[src] = data.copy()
            if len(rk.pulled) == N:
                out = np.zeros(self.count, dtype=np.uint16)
                for q in range(N):
                    lo, hi = self._shard_range(q)
                    out[lo:hi] = rk.pulled[q][: hi - lo]
                self.outputs[k, r] = out
                self.completed[k, r] = True
                rk.phase = "arrive_bottom"
        elif ph == "arrive_bottom":
            self.bar[r] = self._bar_target(e, 3)
            rk.phase = "next" if self.bug == "no_bottom_barrier" else "wait_bottom"
        elif ph in ("wait_bottom", "next"):
            rk.done_epoch = e
            rk.op += 1
            rk.pulled = {}
            rk.phase = "produce" if rk.op < self.K else "done"

    def _inslot(self, k):
        """Input buffer that operation k uses: alternating under dual buffering."""
        if self.proto == BARRIER_ONESHOT_DB and self.bug != "single_input_buffer":
            return k % 2
        return 0

    def _shard_range(self, q):
        lo = min(q * self.shard, self.count)
        hi = min(lo + self.shard, self.count)
        return lo, hi

    # ---------------------------------------------------------------- checks
    def final_checks(self):
        """Checks that need the whole run; returns the list of violations."""
        v = list(self.violations)
        if not self.finished():
            v.append("deadlock: no enabled action while a rank is not done")
            return v
        for k in range(self.K):
            rows = self.inputs[k]
            want = reference.allreduce(rows) if self.op == ALLREDUCE else reference.allgather(rows)
            for r in range(self.N):
                if not np.array_equal(self.outputs[k, r], want):
                    v.append(f"op {k} rank {r}: output differs from the closed form")
            if not all(np.array_equal(self.outputs[k, 0], self.outputs[k, r]) for r in range(self.N)):
                v.append(f"op {k}: ranks disagree")
            finite = np.isfinite(bf16_bits_to_f32(want))
            if np.any((self.outputs[k] == BF16_SENTINEL) & finite[None, :]):
                v.append(f"op {k}: sentinel pattern delivered")
        if self.proto == P.SENTINEL:
            for key, buf in self.mem.items():
                if not np.all(buf == 0xFF):
                    v.append(f"sentinel slot {key} not reset after the chain")
        elif self.proto in (P.LL, P.LL128) and self.bug is None and self.count > 0:
            last = {}
            for k in range(self.K):
                e = self._epoch(k)
                last[e & 1] = e
            for (r, par, q), buf in self.mem.items():
                if par not in last:
                    continue
                for j in range(self.units):
                    if not P.validate_unit(self.proto, buf, j, last[par]):
                        v.append(f"slot {(r, par, q)} unit {j} flag is not epoch {last[par]}")
                        break
        return v


def run_fifo(proto, inputs, op=ALLREDUCE, first_epoch=1, sentinel_reset="after_all"):
    """One fixed, cheap schedule for large inputs: in rounds, every rank takes
    its enabled step, then every pending store lands in issue order.
    Linear in the number of units; returns (sim, violations)."""
    sim = _make_sim(proto, inputs, op, first_epoch, None, sentinel_reset)
    while not sim.finished():
        steps = [a for a in sim.enabled_actions() if a[0] == "step"]
        for a in steps:
            sim.apply(a)
        landed = bool(sim.pending)
        while sim.pending:
            sim.apply(("land", 0))
        if not steps and not landed:
            break
    return sim, sim.final_checks()


def run_chain(proto, inputs, op=ALLREDUCE, first_epoch=1, schedule="random", seed=0,
              slow_rank=None, bug=None, max_steps=2_000_000, sentinel_reset="after_all"):
    """Run one schedule to completion; returns (sim, violations).

    ``schedule``: ``"random"`` picks uniformly among enabled actions;
    ``"adversarial"`` additionally holds back ``slow_rank`` (its steps and
    the stores it sent) until nothing else can happen, then lets one through;
    ``"inorder"`` always takes the first enabled action.
    """
    sim = _make_sim(proto, inputs, op, first_epoch, bug, sentinel_reset)
    rng = np.random.default_rng(seed)
    while not sim.finished() and sim.steps < max_steps:
        acts = sim.enabled_actions()
        if not acts:
            break
        if schedule == "inorder":
            act = acts[0]
        elif schedule == "adversarial" and slow_rank is not None:
            def is_slow(a):
                if a[0] == "step":
                    return a[1] == slow_rank
                st = sim.pending[a[1]]
                return (st["src"] if "src" in st else st["key"][3]) == slow_rank

            fast = [a for a in acts if not is_slow(a)]
            pool = fast if fast else acts
            act = pool[rng.integers(len(pool))]
        else:
            act = acts[rng.integers(len(acts))]
        sim.apply(act)
    return sim, sim.final_checks()


# --------------------------------------------------------------------------
# Self-synchronizing twoshot: reduce-scatter then all-gather, each phase a
# self-synchronizing push with the same readiness encodings and epoch-parity
# double buffering; no barrier anywhere. The large-message variant of the
# same path (twoshot moves 2(N-1)/N of a message per rank instead of N-1
# copies; "SiFAR: Synchronization-Free All-Reduce for Low-Latency LLM
# Inference", abstract: twoshot does better at higher TP degrees).
LL_TWOSHOT = "ll_twoshot"
SENTINEL_TWOSHOT = "sentinel_twoshot"
SELF_SYNC_TWOSHOT = (LL_TWOSHOT, SENTINEL_TWOSHOT)
ALL_PROTOCOLS = ALL_PROTOCOLS + SELF_SYNC_TWOSHOT
__all__ += ["TwoshotSim", "LL_TWOSHOT", "SENTINEL_TWOSHOT", "SELF_SYNC_TWOSHOT", "shard_bounds"]


def shard_bounds(count, n, q, vector=8):
    """Elements [lo, hi) of shard q: shards are whole `vector`-element
    vectors, ceil(ceil(count / vector) / n) of them each; the last ones may be
    short or empty. (The partition changes no result; tiny exhaustive checks
    use vector=1 so that every shard holds data.)"""
    sz = vector * (-(-(-(-count // vector)) // n))
    lo = min(q * sz, count)
    return lo, min(lo + sz, count)


class TwoshotSim:
    """K chained self-synchronizing twoshot all-reduces on N ranks.

    Observation from this model: each slot of either phase is written again
    only after a full exchange of the other phase, so even a single buffer
    (no parity) passes every check here; the GPU keeps the epoch-parity
    double buffer of the oneshot protocols all the same.

    Per operation at epoch e, rank r: (1) pushes shard s of its input into
    rank s's reduce-scatter slot (parity e & 1, source r) for every s != r;
    (2) polls its reduce-scatter slots until shard r of every peer's input is
    in, and reduces shard r in rank order (own part from its input); (3)
    pushes the reduced shard into every peer's all-gather slot; (4) polls its
    all-gather slots until every other shard is in; the output is the shards
    in order. Same unit atomicity, shadow tags and checks as ``ChainSim``.
    """

    def __init__(self, proto, inputs, first_epoch=1, bug=None, sentinel_reset="after_all", vector=8):
        if proto not in SELF_SYNC_TWOSHOT:
            raise ValueError(proto)
        x = np.asarray(inputs, dtype=np.uint16)
        self.proto = proto
        self.enc = P.LL if proto == LL_TWOSHOT else P.SENTINEL
        self.inputs = x
        self.K, self.N, self.count = x.shape
        self.first_epoch = first_epoch
        self.bug = bug
        self.sentinel_reset = sentinel_reset
        self.violations = []
        self.steps = 0
        self.outputs = np.zeros((self.K, self.N, self.count), dtype=np.uint16)
        self.pending = []
        self.bounds = [shard_bounds(self.count, self.N, q, vector) for q in range(self.N)]
        self.mem, self.shadow = {}, {}
        for r in range(self.N):
            for par in (0, 1):
                for q in range(self.N):
                    if q == r:
                        continue
                    # reduce-scatter slot carries shard r; all-gather slot shard q
                    for region, sh in (("rs", r), ("ag", q)):
                        n_el = self.bounds[sh][1] - self.bounds[sh][0]
                        key = (region, r, par, q)
                        self.mem[key] = P.initial_slot(self.enc, n_el)
                        self.shadow[key] = [None] * P.unit_count(self.enc, n_el)
        # consumed[region] = last epoch whose slots of that region the rank
        # has fully read
        self.ranks = [dict(op=0, phase="rs_push", acc={}, staged={}, red=None, consumed={"rs": 0, "ag": 0})
                      for _ in range(self.N)]
        for r in range(self.N):
            self._begin(r)

    def _epoch(self, k):
        return self.first_epoch + k

    def _par(self, e):
        return 0 if self.bug == "single_buffer" else e & 1

    def _n_el(self, region, recv, src):
        sh = recv if region == "rs" else src
        return self.bounds[sh][1] - self.bounds[sh][0]

    def _begin(self, r):
        rk = self.ranks[r]
        rk["acc"], rk["staged"] = {}, {}
        for region in ("rs", "ag"):
            for q in range(self.N):
                if q != r:
                    n_el = self._n_el(region, r, q)
                    rk["acc"][(region, q)] = np.zeros(P.unit_count(self.enc, n_el), dtype=bool)
                    rk["staged"][(region, q)] = np.zeros(n_el, dtype=np.uint16)
        rk["phase"] = "rs_push" if rk["op"] < self.K else "done"

    # interface ------------------------------------------------------------
    def finished(self):
        return all(rk["phase"] == "done" for rk in self.ranks)

    def enabled_actions(self):
        acts = []
        for r, rk in enumerate(self.ranks):
            ph = rk["phase"]
            if ph in ("rs_push", "ag_push") or (ph in ("rs_poll", "ag_poll") and self._productive(r)):
                acts.append(("step", r))
        acts.extend(("land", i) for i in range(len(self.pending)))
        return acts

    def apply(self, act):
        self.steps += 1
        kind, arg = act
        if kind == "land":
            self._land(self.pending.pop(arg))
            return
        rk = self.ranks[arg]
        if rk["phase"] == "rs_push":
            self._push(arg, "rs")
            rk["phase"] = "rs_poll"
        elif rk["phase"] == "ag_push":
            self._push(arg, "ag")
            rk["phase"] = "ag_poll"
        else:
            self._poll(arg, rk["phase"][:2])

    def clone(self):
        return copy.deepcopy(self)

    def state_key(self):
        parts = []
        for key in sorted(self.mem):
            parts.append(self.mem[key].tobytes())
            parts.append(tuple(self.shadow[key]))
        for rk in self.ranks:
            acc = tuple(rk["acc"][k].tobytes() for k in sorted(rk["acc"]))
            stg = tuple(rk["staged"][k].tobytes() for k in sorted(rk["staged"]))
            red = None if rk["red"] is None else rk["red"].tobytes()
            parts.append((rk["op"], rk["phase"], acc, stg, red))
        parts.append(tuple(sorted((s["key"], s["j"], s["epoch"]) for s in self.pending)))
        return tuple(parts)

    # steps ----------------------------------------------------------------
    def _push(self, r, region):
        rk = self.ranks[r]
        k = rk["op"]
        e = self._epoch(k)
        par = self._par(e)
        for p in range(self.N):
            if p == r:
                continue
            if region == "rs":
                lo, hi = self.bounds[p]
                data = self.inputs[k, r, lo:hi]
            else:
                data = rk["red"]
            for j, (off, body) in enumerate(P.encode_all(self.enc, data, e)):
                self.pending.append(dict(key=(region, p, par, r), j=j, off=off, body=body, epoch=e))

    def _land(self, s):
        key = s["key"]
        prev = self.shadow[key][s["j"]]
        reader = self.ranks[key[1]]
        if prev is not None and prev[1] != s["epoch"] and reader["consumed"][key[0]] < prev[1]:
            self.violations.append(f"store of epoch {s['epoch']} overwrote unconsumed epoch {prev[1]} in {key}")
        buf = self.mem[key]
        buf[s["off"]:s["off"] + s["body"].size] = s["body"]
        self.shadow[key][s["j"]] = (key[3], s["epoch"])

    def _productive(self, r):
        rk = self.ranks[r]
        region = rk["phase"][:2]
        e = self._epoch(rk["op"])
        par = self._par(e)
        for (reg, q), acc in rk["acc"].items():
            if reg != region:
                continue
            slot = self.mem[(region, r, par, q)]
            for j in range(acc.size):
                if not acc[j] and P.validate_unit(self.enc, slot, j, e):
                    return True
        return all(acc.all() for (reg, _), acc in rk["acc"].items() if reg == region)

    def _poll(self, r, region):
        rk = self.ranks[r]
        k = rk["op"]
        e = self._epoch(k)
        par = self._par(e)
        for (reg, q), acc in rk["acc"].items():
            if reg != region or acc.all():
                continue
            key = (region, r, par, q)
            slot = self.mem[key]
            n_el = self._n_el(region, r, q)
            for j in range(acc.size):
                if acc[j] or not P.validate_unit(self.enc, slot, j, e):
                    continue
                if self.shadow[key][j] != (q, e):
                    self.violations.append(f"rank {r} epoch {e} accepted {key} unit {j} tagged "
                                           f"{self.shadow[key][j]}")
                lo, vals = P.decode_unit(self.enc, slot, j, n_el)
                rk["staged"][(region, q)][lo:lo + vals.size] = vals
                acc[j] = True
                if self.enc == P.SENTINEL and self.sentinel_reset == "on_accept" and self.bug != "no_reset":
                    off, body = P.reset_unit_bytes(self.enc, j)
                    slot[off:off + body.size] = body
                    self.shadow[key][j] = None
        if not all(acc.all() for (reg, _), acc in rk["acc"].items() if reg == region):
            return
        if self.enc == P.SENTINEL and self.sentinel_reset == "after_all" and self.bug != "no_reset":
            for (reg, q), acc in rk["acc"].items():
                if reg == region:
                    key = (region, r, par, q)
                    for j in range(acc.size):
                        off, body = P.reset_unit_bytes(self.enc, j)
                        self.mem[key][off:off + body.size] = body
                        self.shadow[key][j] = None
        rk["consumed"][region] = e
        if region == "rs":
            lo, hi = self.bounds[r]
            rows = np.stack([self.inputs[k, q, lo:hi] if q == r else rk["staged"][("rs", q)]
                             for q in range(self.N)])
            rk["red"] = reference.allreduce(rows) if hi > lo else np.zeros(0, dtype=np.uint16)
            rk["phase"] = "ag_push"
        else:
            out = np.zeros(self.count, dtype=np.uint16)
            for q in range(self.N):
                lo, hi = self.bounds[q]
                out[lo:hi] = rk["red"] if q == r else rk["staged"][("ag", q)]
            self.outputs[k, r] = out
            rk["op"] += 1
            rk["red"] = None
            self._begin(r)

    def final_checks(self):
        v = list(self.violations)
        if not self.finished():
            v.append("deadlock: no enabled action while a rank is not done")
            return v
        for k in range(self.K):
            want = reference.allreduce(self.inputs[k])
            for r in range(self.N):
                if not np.array_equal(self.outputs[k, r], want):
                    v.append(f"op {k} rank {r}: output differs from the closed form")
        if self.enc == P.SENTINEL:
            for key, buf in self.mem.items():
                if not np.all(buf == 0xFF):
                    v.append(f"sentinel slot {key} not reset after the chain")
        return v


def _make_sim(proto, inputs, op, first_epoch, bug, sentinel_reset, vector=8):
    if proto in SELF_SYNC_TWOSHOT:
        if op != ALLREDUCE:
            raise ValueError("twoshot is an all-reduce algorithm")
        return TwoshotSim(proto, inputs, first_epoch=first_epoch, bug=bug, sentinel_reset=sentinel_reset,
                          vector=vector)
    return ChainSim(proto, inputs, op=op, first_epoch=first_epoch, bug=bug, sentinel_reset=sentinel_reset)
