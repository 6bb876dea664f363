"""Cost-guided protocol choice, restated plainly. PARITY UNPINNED.

"flash-comm: Self-Synchronizing Collective Communication for LLM Decoding",
abstract: a selector adapts the readiness encoding to the message size and the
number of GPUs, weighing synchronization overhead against extra transfer
cost. "Why Microseconds Matter in AI Infrastructure", section "What I learned
from it": the choice there was made from measurements, a predictive model
being future work. Neither page gives a functional form or a number.

Reading taken: per protocol p and rank count N a latency estimate T_p(S, N)
built from measurements (the empirical selection of the review): the p50
latency measured at power-of-two message sizes, interpolated linearly in
log2(S) between the nearest measured sizes, held at the smallest measured
value below them, and scaled by the algorithmic traffic bytes_p(S, N) above
the largest; with no measurements, alpha_p(N) + beta_p(N) * bytes_p(S, N)
(the synchronization cost plus the transfer cost the flash-comm abstract
weighs). The choice is the argmin; on a tie the protocol that moves fewer
bytes wins, then the earlier one in the order
sentinel < LL128 < LL128 one-load < LL < sentinel twoshot < LL twoshot <
dual-buffered oneshot < barrier oneshot < barrier twoshot.

Which protocol wins where cannot be checked against the pages (they give no
numbers): parity unpinned. The estimate and the argmin with its tie-break are
pinned by hand examples in the tests.
"""

import math

from . import protocols as P

__all__ = ["TIE_ORDER", "algorithmic_bytes", "estimate", "choose"]

TIE_ORDER = (P.SENTINEL, P.LL128, "ll128_fast", P.LL, "sentinel_twoshot", "ll_twoshot", "barrier_oneshot_db",
             "barrier_oneshot", "barrier_twoshot")


def algorithmic_bytes(proto, count, n, op="allreduce"):
    """Bytes one operation moves, summed over the N ranks.

    Self-sync all-reduce, per rank: read own input (S), write the encoded
    chunk to N-1 peers, read N-1 encoded chunks, write the output (S); the
    sentinel reader also rewrites what it consumed. Barrier oneshot: each rank
    reads N inputs and writes one output. Barrier twoshot: each rank reads its
    shard of N inputs (S), writes its reduced shard (S/N), reads N shards (S)
    and writes the output (S). All-gather: read own shard, write and read N-1
    encoded shards, write N shards.
    """
    s = 2 * count
    if proto == "ll128_fast":  # the LL128 layout, moved without fences
        proto = P.LL128
    if proto in P.SELF_SYNC:
        enc = P.slot_bytes(proto, count)
        reset = (n - 1) * s if proto == P.SENTINEL else 0
        if op == "allreduce":
            return n * (s + 2 * (n - 1) * enc + s + reset)
        return n * (s + 2 * (n - 1) * enc + n * s + reset)
    if proto in ("barrier_oneshot", "barrier_oneshot_db"):
        if op == "allreduce":
            return n * (n * s + s)
        return n * (n * s + n * s)
    if proto == "barrier_twoshot":
        return n * (s + s / n + s + s)
    if proto in ("ll_twoshot", "sentinel_twoshot"):
        # read own input, push and poll N-1 encoded shards in each of the two
        # phases, write the output; the sentinel rewrites what it consumed
        shard = -(-count // n)
        sh = 2 * shard
        enc = P.slot_bytes(P.LL, shard) if proto == "ll_twoshot" else sh
        reset = 2 * (n - 1) * sh if proto == "sentinel_twoshot" else 0
        return n * (s + 4 * (n - 1) * enc + s + reset)
    raise ValueError(proto)


MIN_LOG2 = 9


def estimate(entry, proto, bytes_per_rank, n, op="allreduce"):
    """Latency estimate of one protocol; ``entry`` = (alpha, beta, table)
    with table[i] the p50 at 2**(MIN_LOG2 + i) bytes per rank (<= 0 = not
    measured). None if the protocol is unavailable (alpha < 0)."""
    alpha, beta, table = entry
    if alpha < 0:
        return None
    b = algorithmic_bytes(proto, bytes_per_rank // 2, n, op)
    measured = [i for i, t in enumerate(table) if t > 0]
    if not measured:
        return alpha + beta * b
    k = math.log2(max(bytes_per_rank, 1)) - MIN_LOG2
    first, last = measured[0], measured[-1]
    if k <= first:
        return table[first]
    if k >= last:
        ref = (2 ** (MIN_LOG2 + last)) // 2
        return table[last] * b / algorithmic_bytes(proto, ref, n, op)
    lo = math.floor(k)
    while lo > first and not table[lo] > 0:
        lo -= 1
    hi = math.ceil(k)
    while hi < last and not table[hi] > 0:
        hi += 1
    if hi == lo:
        return table[lo]
    return table[lo] + (table[hi] - table[lo]) * (k - lo) / (hi - lo)


def choose(model, bytes_per_rank, n, op="allreduce"):
    """argmin over ``model[proto] = (alpha, beta, table)``; returns the protocol."""
    best = None
    for proto in TIE_ORDER:
        if proto not in model:
            continue
        if op == "allgather" and proto in ("barrier_twoshot", "ll_twoshot", "sentinel_twoshot"):
            continue
        t = estimate(model[proto], proto, bytes_per_rank, n, op)
        if t is None:
            continue
        b = algorithmic_bytes(proto, bytes_per_rank // 2, n, op)
        key = (t, b, TIE_ORDER.index(proto))
        if best is None or key < best[0]:
            best = (key, proto)
    return None if best is None else best[1]
