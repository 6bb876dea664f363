"""Message-size sweep and selector calibration.

    python -m latency_self_synchronizing_b200.sweep [--nranks 2 4 8] [--op allreduce]
        [--protocols ll ll128 sentinel barrier_oneshot barrier_twoshot]
        [--min-bytes 1024] [--max-bytes 67108864] [--k-ops 50] [--reps 3]
        [--out sweep.jsonl] [--fit model.json]

For every (rank count, protocol, size) it runs `--reps` chains of `--k-ops`
operations in one persistent launch each and reports p50 / p99 microseconds
per operation (from the in-kernel completion stamps, first 5 operations of
each chain dropped), the mean from CUDA events, and the achieved algorithmic
bandwidth. Inputs are normal(0,1) bf16 drawn on the device by torch's seeded
generator (the sweep checks no values; parity is the tests' job); operations
cycle through at most 8 distinct inputs per rank so that the largest sizes
fit.

`--fit` fits, per (op, protocol, N), T = alpha + beta * bytes by least squares
weighted by 1/T (relative error), and writes the coefficients as JSON; the
selector's choice under the fitted model is reported at every point together
with the measured best (regret = chosen p50 / best p50).
"""

import argparse
import json
import statistics
import sys

import numpy as np
import torch

from . import api

DROP_FIRST = 5


def _percentile(v, q):
    v = sorted(v)
    return float(v[min(len(v) - 1, max(0, int(round(q * (len(v) - 1)))))]) if v else float("nan")


def measure_point(comm, op, proto, count, k_ops, reps, gen, dev):
    n = comm.nranks
    distinct = min(k_ops, 8)
    stride = (count + 7) // 8 * 8
    xin = torch.randn(distinct * n * stride, generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
    out_count = count if op == "allreduce" else n * count
    ostride = (out_count + 7) // 8 * 8
    outb = torch.empty(2 * n * ostride, dtype=torch.bfloat16, device=dev)
    tin = torch.tensor([xin.data_ptr() + 2 * stride * ((k % distinct) * n + r)
                        for k in range(k_ops) for r in range(n)], dtype=torch.int64, device=dev)
    tout = torch.tensor([outb.data_ptr() + 2 * ostride * ((k % 2) * n + r)
                         for k in range(k_ops) for r in range(n)], dtype=torch.int64, device=dev)
    fn = comm.allreduce_chain if op == "allreduce" else comm.allgather_chain
    lat, ev_us = [], []
    for rep in range(reps + 1):
        t = torch.zeros(k_ops + 1, dtype=torch.int64, device=dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn(tin, tout, count, k_ops, protocol=proto, timings=t)
        b.record()
        torch.cuda.synchronize()
        if rep == 0:
            continue  # warm-up chain
        h = t.cpu().numpy().astype(np.int64)
        d = np.diff(h[1:])
        lat.extend((d[DROP_FIRST - 1:] / 1e3).tolist())
        ev_us.append(a.elapsed_time(b) * 1e3 / k_ops)
    st, info = comm.status()
    if st != api.Status.OK:
        raise RuntimeError(f"{proto} N={n} count={count}: device status {st.name} info {info:#x}")
    p50 = _percentile(lat, 0.5)
    nbytes = api.algorithmic_bytes(op, proto, count, n)
    return {"op": op, "protocol": proto, "nranks": n, "bytes_per_rank": 2 * count, "count": count,
            "p50_us": p50, "p99_us": _percentile(lat, 0.99), "mean_us_events": statistics.mean(ev_us),
            "algorithmic_bytes": nbytes, "gbs_p50": nbytes / (p50 * 1e-6) / 1e9 if p50 > 0 else None,
            "ctas_per_rank": comm.launch_shape(op, proto, count)[0]}


def fit(points):
    """{(op, proto, n): (alpha_us, beta_us_per_byte)} by 1/T-weighted least squares."""
    groups = {}
    for p in points:
        groups.setdefault((p["op"], p["protocol"], p["nranks"]), []).append(p)
    out = {}
    for key, pts in groups.items():
        x = np.array([p["algorithmic_bytes"] for p in pts], dtype=np.float64)
        y = np.array([p["p50_us"] for p in pts], dtype=np.float64)
        w = 1.0 / y
        A = np.stack([np.ones_like(x), x], axis=1) * w[:, None]
        coef, *_ = np.linalg.lstsq(A, y * w, rcond=None)
        alpha, beta = float(coef[0]), float(coef[1])
        if beta < 0:  # flat curve: latency-bound everywhere
            alpha, beta = float(np.median(y)), 0.0
        if alpha < 0:
            alpha = 0.0
        out[key] = (alpha, beta)
    return out


def model_from_fit(coeffs):
    m = api.default_cost_model()
    for (op, proto, n), (a, b) in coeffs.items():
        o = int(api.as_op(op))
        pr = int(api.as_protocol(proto))
        m.c[o][pr][n].alpha_us = a
        m.c[o][pr][n].beta_us_per_byte = b
    return m


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--nranks", type=int, nargs="+", default=[2, 4, 8])
    ap.add_argument("--op", default="allreduce", choices=["allreduce", "allgather"])
    ap.add_argument("--protocols", nargs="+",
                    default=["ll", "ll128", "sentinel", "barrier_oneshot", "barrier_twoshot"])
    ap.add_argument("--min-bytes", type=int, default=1024)
    ap.add_argument("--max-bytes", type=int, default=64 << 20)
    ap.add_argument("--k-ops", type=int, default=50)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--ctas-per-rank", type=int, default=0)
    ap.add_argument("--out", default=None)
    ap.add_argument("--fit", default=None)
    a = ap.parse_args(argv)
    dev = torch.device("cuda")
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    sizes = []
    b = a.min_bytes
    while b <= a.max_bytes:
        sizes.append(b)
        b *= 2
    protos = [p for p in a.protocols if not (a.op == "allgather" and p == "barrier_twoshot")]
    points = []
    sink = open(a.out, "w") if a.out else None
    for n in a.nranks:
        for proto in protos:
            comm = api.Communicator(n, max(sizes), protocols=[proto], ctas_per_rank=a.ctas_per_rank)
            try:
                for nbytes in sizes:
                    k = a.k_ops if nbytes <= (8 << 20) else max(8, a.k_ops // 5)
                    pt = measure_point(comm, a.op, proto, nbytes // 2, k, a.reps, gen, dev)
                    points.append(pt)
                    line = json.dumps(pt)
                    print(line, flush=True)
                    if sink:
                        sink.write(line + "\n")
            finally:
                comm.close()
                torch.cuda.empty_cache()
    if a.fit:
        coeffs = fit(points)
        model = model_from_fit(coeffs)
        best = {}
        for p in points:
            key = (p["op"], p["nranks"], p["bytes_per_rank"])
            if key not in best or p["p50_us"] < best[key]["p50_us"]:
                best[key] = p
        regrets = []
        for key, bp in sorted(best.items()):
            op, n, nbytes = key
            chosen = api.select_protocol_model(model, op, nbytes, n).name.lower()
            cp = next(p for p in points if (p["op"], p["nranks"], p["bytes_per_rank"]) == key
                      and p["protocol"] == chosen)
            r = cp["p50_us"] / bp["p50_us"]
            regrets.append(r)
            print(json.dumps({"selector": chosen, "best": bp["protocol"], "op": op, "nranks": n,
                              "bytes_per_rank": nbytes, "regret": r}), flush=True)
        out = {"coefficients": [{"op": k[0], "protocol": k[1], "nranks": k[2], "alpha_us": v[0],
                                 "beta_us_per_byte": v[1]} for k, v in sorted(coeffs.items())],
               "regret_median": statistics.median(regrets), "regret_max": max(regrets)}
        with open(a.fit, "w") as f:
            json.dump(out, f, indent=1)
        print(json.dumps({"regret_median": out["regret_median"], "regret_max": out["regret_max"]}))
    if sink:
        sink.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
