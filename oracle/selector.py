"""Cost-guided protocol choice, restated plainly. PARITY UNPINNED.

"flash-comm: Self-Synchronizing Collective Communication for LLM Decoding",
abstract: a selector adapts the readiness encoding to the message size and the
number of GPUs, weighing synchronization overhead against extra transfer
cost. "Why Microseconds Matter in AI Infrastructure", section "What I learned
from it": the choice there was made from measurements, a predictive model
being future work. Neither page gives a functional form or a number.

Reading taken: per protocol p and rank count N a latency estimate

    T_p(S, N) = alpha_p(N) + beta_p(N) * bytes_p(S, N)

where bytes_p is the algorithmic traffic of one operation (encoded bytes
written plus bytes read over all ranks), alpha and beta are fitted on the
machine, and the choice is the argmin; on a tie the protocol that moves
fewer bytes wins, then the earlier one in the order
sentinel < LL128 < LL < barrier oneshot < barrier twoshot.

Which protocol wins where cannot be checked against the pages (they give no
numbers): parity unpinned. The argmin and tie-break are pinned by hand
examples in the tests.
"""

from . import protocols as P

__all__ = ["TIE_ORDER", "algorithmic_bytes", "choose"]

TIE_ORDER = (P.SENTINEL, P.LL128, P.LL, "barrier_oneshot", "barrier_twoshot")


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
    if proto in P.SELF_SYNC:
        enc = P.slot_bytes(proto, count)
        reset = (n - 1) * s if proto == P.SENTINEL else 0
        if op == "allreduce":
            return n * (s + 2 * (n - 1) * enc + s + reset)
        return n * (s + 2 * (n - 1) * enc + n * s + reset)
    if proto == "barrier_oneshot":
        if op == "allreduce":
            return n * (n * s + s)
        return n * (n * s + n * s)
    if proto == "barrier_twoshot":
        return n * (s + s / n + s + s)
    raise ValueError(proto)


def choose(coeffs, count, n, op="allreduce", candidates=None):
    """argmin over ``coeffs[proto] = (alpha, beta)``; returns the protocol."""
    best = None
    for proto in TIE_ORDER:
        if proto not in coeffs:
            continue
        if candidates is not None and proto not in candidates:
            continue
        if op == "allgather" and proto == "barrier_twoshot":
            continue
        alpha, beta = coeffs[proto]
        b = algorithmic_bytes(proto, count, n, op)
        t = alpha + beta * b
        key = (t, b, TIE_ORDER.index(proto))
        if best is None or key < best[0]:
            best = (key, proto)
    return None if best is None else best[1]
