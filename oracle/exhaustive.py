"""Brute-force checks of the protocol logic on tiny inputs.

Three enumerations, each over a space small enough to cover completely:

1. ``landing_subsets`` -- for one epoch and every receiver, every subset of
   the units its peers send (every prefix of every landing order is such a
   subset), on top of slot contents left by the previous use of the same
   parity (epoch e-2, or the initial fill). At each subset the receiver's poll
   must accept exactly the landed units, decode them to the sender's data,
   report completion only when all have landed, and then produce the closed
   form. "flash-comm: Self-Synchronizing Collective Communication for LLM
   Decoding", abstract: receivers validate the blocks they need.
2. ``arrival_orders`` -- for every receiver, every order in which the N
   contributions (own included) reach it: (N!)^N combinations. Staging in
   arrival order and reducing in rank order must give the same bits on every
   rank (same abstract: transport order decoupled from reduction order).
3. ``explore_interleavings`` -- a depth-first search over every interleaving
   of the simulator's actions (pushes, polls, store landings) for a short
   chain, with memoised states. Every reachable state is checked for the
   simulator's violations and every terminal state for the final checks;
   a reachable state with no enabled action and unfinished ranks is a
   deadlock.
"""

import itertools

import numpy as np

from . import protocols as P
from . import reference
from .bf16 import bf16_bits_to_f32, f32_to_bf16_bits
from .simulator import _make_sim

__all__ = ["landing_subsets", "arrival_orders", "explore_interleavings"]


def _slot_after(proto, data, epoch, count):
    """Slot contents after every unit of ``data`` at ``epoch`` landed."""
    buf = P.initial_slot(proto, count)
    for off, body in P.encode_all(proto, data, epoch):
        buf[off:off + body.size] = body
    return buf


def landing_subsets(proto, inputs, epoch, stale_inputs=None, bug=None):
    """Check every landing subset for every receiver at one epoch.

    ``inputs``: uint16 [N, count] (this epoch). ``stale_inputs``: [N, count]
    sent at epoch-2 into the same parity, or None for the first use of the
    parity. ``bug="no_reset"`` leaves sentinel slots holding stale data
    instead of the sentinel. Returns (checked_subsets, violations).
    """
    x = np.asarray(inputs, dtype=np.uint16)
    n, count = x.shape
    units = P.unit_count(proto, count)
    want = reference.allreduce(x)
    violations = []
    checked = 0
    for r in range(n):
        peers = [q for q in range(n) if q != r]
        base = {}
        for q in peers:
            if stale_inputs is None or epoch <= 2:
                base[q] = P.initial_slot(proto, count)
            elif proto == P.SENTINEL and bug != "no_reset":
                base[q] = P.initial_slot(proto, count)  # reset after consuming
            else:
                base[q] = _slot_after(proto, stale_inputs[q], epoch - 2, count)
        fresh = {q: P.encode_all(proto, x[q], epoch) for q in peers}
        all_units = [(q, j) for q in peers for j in range(units)]
        for mask in range(1 << len(all_units)):
            landed = {all_units[i] for i in range(len(all_units)) if (mask >> i) & 1}
            mem = {q: base[q].copy() for q in peers}
            for (q, j) in landed:
                off, body = fresh[q][j]
                mem[q][off:off + body.size] = body
            accepted = set()
            staged = {q: np.zeros(count, dtype=np.uint16) for q in peers}
            for q in peers:
                for j in range(units):
                    if P.validate_unit(proto, mem[q], j, epoch):
                        accepted.add((q, j))
                        lo, vals = P.decode_unit(proto, mem[q], j, count)
                        staged[q][lo:lo + vals.size] = vals
            checked += 1
            if accepted != landed:
                violations.append(
                    f"receiver {r} epoch {epoch}: accepted {sorted(accepted - landed)} "
                    f"not landed / missed {sorted(landed - accepted)}")
                continue
            for (q, j) in landed:
                lo, hi = P.unit_elements(proto, count, j)
                if not np.array_equal(staged[q][lo:hi], x[q][lo:hi]):
                    violations.append(f"receiver {r}: unit {(q, j)} decoded wrongly")
            if len(landed) == len(all_units):
                rows = np.stack([x[r] if q == r else staged[q] for q in range(n)])
                if not np.array_equal(reference.allreduce(rows), want):
                    violations.append(f"receiver {r}: complete poll reduced wrongly")
    return checked, violations


def arrival_orders(inputs, bug=None):
    """Every arrival order at every receiver; returns (combinations, violations).

    With ``bug="arrival_order"`` each receiver folds in arrival order, which
    the check must flag whenever the sum is order sensitive.
    """
    x = np.asarray(inputs, dtype=np.uint16)
    n = x.shape[0]
    want = reference.allreduce(x)
    per_rank = []
    for r in range(n):
        outs = []
        for order in itertools.permutations(range(n)):
            staged = {}
            for q in order:  # contributions land in this order
                staged[q] = x[q]
            fold = order if bug == "arrival_order" else range(n)
            fold = list(fold)
            acc = bf16_bits_to_f32(staged[fold[0]]).copy()
            for q in fold[1:]:
                acc = np.add(acc, bf16_bits_to_f32(staged[q]), dtype=np.float32)
            outs.append(f32_to_bf16_bits(acc))
        per_rank.append(outs)
    violations = []
    combos = 0
    for choice in itertools.product(*[range(len(o)) for o in per_rank]):
        combos += 1
        results = [per_rank[r][c] for r, c in enumerate(choice)]
        if not all(np.array_equal(results[0], res) for res in results):
            violations.append(f"ranks disagree under arrival orders {choice}")
            break
        if not np.array_equal(results[0], want):
            violations.append(f"result differs from the closed form under {choice}")
            break
    return combos, violations


def explore_interleavings(proto, inputs, op="allreduce", bug=None, max_states=2_000_000,
                          sentinel_reset="after_all", vector=8):
    """Depth-first search over all interleavings; returns (states, violations)."""
    root = _make_sim(proto, inputs, op, 1, bug, sentinel_reset, vector)
    seen = set()
    stack = [root]
    violations = []
    while stack:
        sim = stack.pop()
        key = sim.state_key()
        if key in seen:
            continue
        seen.add(key)
        if len(seen) > max_states:
            violations.append("state budget exceeded")
            break
        if sim.violations:
            violations.extend(sim.violations)
            break
        acts = sim.enabled_actions()
        if not acts:
            v = sim.final_checks()
            if v:
                violations.extend(v)
                break
            continue
        for act in acts:
            child = sim.clone()
            child.apply(act)
            stack.append(child)
    return len(seen), violations
