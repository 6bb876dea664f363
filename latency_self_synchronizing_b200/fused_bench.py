"""Timing of the fused row-parallel linear + all-reduce against the unfused
pair (a batched matrix-vector product for all ranks, then an all-reduce).

    python -m latency_self_synchronizing_b200.fused_bench [--nranks 4] [--hidden 8192]
        [--kdim 7168] [--iters 50]

Shapes default to a Llama-3.1-70B MLP down projection with 4-way tensor
parallelism (hidden 8192, intermediate 28672 / 4 = 7168 per rank), one
decode token. Weights are normal(0, 0.05), drawn on the device by torch's
seeded generator (timing only; parity is the tests' job). The weights of all
ranks (N * hidden * kdim * 2 bytes) exceed L2, so every iteration reads them
from HBM. Prints one JSON line: microseconds per layer for both, and the
fused kernel's weight-streaming bandwidth against the measured HBM copy
bandwidth.
"""

import argparse
import json
import os
import statistics

import torch

from . import api


def _events(fn, iters, warmup=5):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    times = []
    for _ in range(iters):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b) * 1e3)
    return statistics.median(times)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--nranks", type=int, default=4)
    ap.add_argument("--hidden", type=int, default=8192)
    ap.add_argument("--kdim", type=int, default=7168)
    ap.add_argument("--iters", type=int, default=50)
    a = ap.parse_args(argv)
    n, hidden, kdim = a.nranks, a.hidden, a.kdim
    dev = torch.device("cuda")
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    w = (torch.randn(n, hidden, kdim, generator=gen, device=dev) * 0.05).to(torch.bfloat16)
    x = torch.randn(n, kdim, 1, generator=gen, device=dev).to(torch.bfloat16)
    y = torch.empty(n, hidden, dtype=torch.bfloat16, device=dev)
    part = torch.empty(n, hidden, 1, dtype=torch.bfloat16, device=dev)
    y2 = torch.empty(n, hidden, dtype=torch.bfloat16, device=dev)
    comm = api.Communicator(n, hidden * 2)
    W = [w[r] for r in range(n)]
    X = [x[r, :, 0] for r in range(n)]
    Y = [y[r] for r in range(n)]
    P = [part[r, :, 0] for r in range(n)]
    Y2 = [y2[r] for r in range(n)]

    def fused():
        comm.linear_allreduce(W, X, Y)

    def unfused():
        torch.bmm(w, x, out=part)
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
    wbytes = n * hidden * kdim * 2
    print(json.dumps({"nranks": n, "hidden": hidden, "kdim": kdim, "fused_us": t_f, "unfused_us": t_u,
                      "unfused_selected_protocol": comm.select_protocol("allreduce", hidden * 2).name.lower(),
                      "fused_weight_gbs": wbytes / (t_f * 1e-6) / 1e9, "hbm_peak_gbs": peak,
                      "fused_frac": wbytes / (t_f * 1e-6) / 1e9 / peak}))
    comm.close()


if __name__ == "__main__":
    main()
