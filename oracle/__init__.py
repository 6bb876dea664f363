"""CPU oracle for the self-synchronizing all-reduce and all-gather.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or
execute anything in this package: only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py`` use it. It shares no code,
table, constant or helper with the CUDA library under
``latency_self_synchronizing_b200/``, and it never imports that package; the
seeded input generator is the only thing both sides use, and callers pass its
arrays in.

Everything here is deliberately plain: NumPy float32 adds for the fp32
arithmetic (IEEE 754 round-to-nearest-even, no flush-to-zero), integer bit
manipulation for the bfloat16 codec, and Python loops over ranks, units and
schedules. No blocking, fusion or reordering beyond what the definitions state.

Sources followed (page title, section):

* "flash-comm: Self-Synchronizing Collective Communication for LLM Decoding",
  abstract -- each block carries its own readiness evidence, the receiver
  validates the blocks it needs, transport order is decoupled from reduction
  order, and the same mechanism serves a standalone all-gather.
* "Why Microseconds Matter in AI Infrastructure", section "Latency can matter
  more than bandwidth" -- LL flag packing (data and flag in one atomic store),
  the sentinel protocol (pre-filled receive buffer, polled until it changes,
  then reset) and double buffering; section "Defining the physical lower bound"
  -- the speed-of-light latency formula.
* "SiFAR: Synchronization-Free All-Reduce for Low-Latency LLM Inference",
  abstract -- oneshot/twoshot with top and bottom barriers, the bottom barrier
  as a write-after-write guard.

Parity status of each part (what pins it, independent of the code itself):

* ``bf16``        -- pinned: IEEE 754 worked values, ties, overflow,
                     subnormals, and the torch library conversion.
* ``reference``   -- pinned: an order-sensitive worked example whose answer is
                     derived by hand, the fp64 error bound, brute force.
* ``protocols`` / ``simulator`` / ``exhaustive`` -- pinned to the closed form by
                     enumeration of every landing subset and arrival order at
                     N=2-3, an exhaustive interleaving search at N=2, random and
                     adversarial schedules, and planted mistakes that the checks
                     must catch.
* ``threaded``    -- (``threaded.c``, plain C, one POSIX thread per rank, C11
                     atomics) every protocol on real threads: pinned to the
                     closed forms under the CPU's own interleavings and seeded
                     delays, with planted mistakes (a dropped sentinel reset,
                     a reversed reduction order, one receive buffer, no bottom
                     barrier, one input buffer in the dual-buffered oneshot)
                     that the checks catch. Not imported here: it compiles on
                     first use.
* ``linear``      -- the row-parallel linear layer and its all-reduce (the
                     fused layer): pinned by hand-worked values, one-hot
                     inputs that pick weight columns, additivity over ranks
                     and tokens, and an error bound that must cover simulated
                     fp32 / bf16 arithmetic in four summation orders while
                     catching a dropped block of products.
* ``sol``         -- pinned: the worked example on the first page.
* ``selector``    -- parity unpinned: the pages give no cost-model numbers, so
                     which protocol wins where cannot be checked against them;
                     only the argmin and its tie-break are pinned by hand
                     examples.
"""

from . import bf16, reference, protocols, simulator, exhaustive, sol, selector, linear  # noqa: F401
