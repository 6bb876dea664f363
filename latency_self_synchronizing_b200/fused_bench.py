"""Timing of the fused row-parallel linear + all-reduce against the unfused
pair (a batched matrix-vector product for all ranks, then an all-reduce).

    python -m latency_self_synchronizing_b200.fused_bench [--nranks 4] [--hidden 8192]
        [--kdim 7168] [--tokens 1] [--iters 50]

Shapes default to a Llama-3.1-70B MLP down projection with 4-way tensor
parallelism (hidden 8192, intermediate 28672 / 4 = 7168 per rank), one
decode token (--tokens: 1..8 tokens of a decode step in one call). Weights
are normal(0, 0.05), drawn on the device by torch's
seeded generator (timing only; parity is the tests' job). Consecutive calls
use different copies of the weights (at least 320 MB in all), so no call
finds its weights in L2 and every call streams them from HBM. Time per
layer = mean over `iters` back-to-back calls between two CUDA events (median
of 5 such runs). Prints one JSON line: microseconds per layer for both, and
the fused kernel's weight-streaming bandwidth against the measured HBM copy
bandwidth.
"""

import argparse
import json
import os
import statistics

import torch

from . import api


def _events(fn, iters, reps=5, warmup=5):
    """Median over `reps` of the mean time per call of `iters` back-to-back
    calls between two events (a decode step issues its layers back to back,
    so host-side call overhead overlaps the previous layer's GPU time)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(iters):
            fn()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b) * 1e3 / iters)
    return statistics.median(times)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--nranks", type=int, default=4)
    ap.add_argument("--hidden", type=int, default=8192)
    ap.add_argument("--kdim", type=int, default=7168)
    ap.add_argument("--tokens", type=int, default=1)
    ap.add_argument("--iters", type=int, default=50)
    a = ap.parse_args(argv)
    n, hidden, kdim, tokens = a.nranks, a.hidden, a.kdim, a.tokens
    dev = torch.device("cuda")
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    wbytes = n * hidden * kdim * 2
    # enough weight copies, used in turn, that consecutive layers never find
    # their weights in the 126 MB L2 (a decode step's layers are distinct)
    copies = max(2, -(-(320 << 20) // wbytes))
    ws = [(torch.randn(n, hidden, kdim, generator=gen, device=dev) * 0.05).to(torch.bfloat16) for _ in range(copies)]
    x = torch.randn(n, tokens, kdim, generator=gen, device=dev).to(torch.bfloat16)
    y = torch.empty(n, tokens, hidden, dtype=torch.bfloat16, device=dev)
    part = torch.empty(n, tokens, hidden, dtype=torch.bfloat16, device=dev)
    y2 = torch.empty(n, tokens, hidden, dtype=torch.bfloat16, device=dev)
    comm = api.Communicator(n, tokens * hidden * 2)
    Ws = [[w[r] for r in range(n)] for w in ws]
    X = [x[r] if tokens > 1 else x[r, 0] for r in range(n)]
    Y = [y[r] if tokens > 1 else y[r, 0] for r in range(n)]
    P = [part[r].view(-1) for r in range(n)]
    Y2 = [y2[r].view(-1) for r in range(n)]
    turn = [0]

    def fused():
        turn[0] = (turn[0] + 1) % copies
        comm.linear_allreduce(Ws[turn[0]], X, Y)

    def unfused():
        turn[0] = (turn[0] + 1) % copies
        torch.bmm(x, ws[turn[0]].transpose(1, 2), out=part)
        comm.allreduce(P, Y2, protocol="auto")

    t_f = _events(fused, a.iters)
    t_u = _events(unfused, a.iters)
    st, _ = comm.status()
    if st != api.Status.OK:
        raise RuntimeError(f"device status {st.name}")
    peak = 6650.0
    try:
        peak = float(json.load(open(os.path.join(os.path.dirname(os.path.dirname(__file__)),
                                                 "MEASURED_PEAKS.json")))["hbm_gbs"])
    except (OSError, KeyError, ValueError):
        pass
    print(json.dumps({"nranks": n, "hidden": hidden, "kdim": kdim, "tokens": tokens, "weight_copies": copies,
                      "fused_us": t_f,
                      "unfused_us": t_u,
                      "unfused_selected_protocol": comm.select_protocol("allreduce", tokens * hidden * 2).name.lower(),
                      "fused_weight_gbs": wbytes / (t_f * 1e-6) / 1e9, "hbm_peak_gbs": peak,
                      "fused_frac": wbytes / (t_f * 1e-6) / 1e9 / peak}))
    comm.close()


if __name__ == "__main__":
    main()
