"""Speed-of-light latency bound of a small-message all-reduce.

"Why Microseconds Matter in AI Infrastructure", section "Defining the physical
lower bound": the smallest thing that must move is one 128-byte cache line,
and the bound is two L2 round trips plus one remote store,

    L_SoL = 2 * L_L2_RTT + L_remote_store

with the page's worked example 2 * 0.306 us + 0.792 us = 1.404 us on two
GB200 GPUs (instruction scheduling and the reduction itself are ignored).
"""

__all__ = ["sol_latency"]


def sol_latency(l2_rtt, remote_store):
    """Lower bound in the units of the arguments."""
    if l2_rtt < 0 or remote_store < 0:
        raise ValueError("latencies are non-negative")
    return 2.0 * l2_rtt + remote_store
