"""Message-size sweep and selector calibration.

    python -m latency_self_synchronizing_b200.sweep [--nranks 2 4 8] [--op allreduce]
        [--protocols ll ll128 sentinel barrier_oneshot barrier_twoshot]
        [--min-bytes 1024] [--max-bytes 67108864 | --sizes B ...] [--k-ops 50] [--reps 3]
        [--out sweep.jsonl] [--model-from SWEEP.jsonl ...] [--report selector.json]

For every (rank count, protocol, size) it runs `--reps` chains of `--k-ops`
operations in one persistent launch each and reports p50 / p99 microseconds
per operation (from the in-kernel completion stamps, first 5 operations of
each chain dropped), the mean from CUDA events, and the achieved algorithmic
bandwidth. Inputs are normal(0,1) bf16 drawn on the device by torch's seeded
generator (the sweep checks no values; parity is the tests' job); operations
cycle through at most 8 distinct inputs per rank so that the largest sizes
fit.

After the sweep the selector is evaluated at every swept size: its choice
under the latency model (the built-in table, or one built from earlier sweep
files given with `--model-from`) against the protocol measured fastest there
(regret = chosen p50 / best p50). `--sizes` sweeps explicit sizes (e.g. the
midpoints 1.5 * 2^k between the table's measured sizes, for an
out-of-sample check).
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


def measure_point(comm, op, proto, count, k_ops, reps, gen, dev, distinct=None):
    """p50 / p99 per operation of `reps` chains of k_ops operations (after one
    warm-up chain). Operations cycle through `distinct` inputs per rank
    (default min(k_ops, 8)); more distinct inputs than fit in L2 make every
    chain read its inputs from HBM."""
    n = comm.nranks
    distinct = min(k_ops, 8) if distinct is None else max(1, min(k_ops, int(distinct)))
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
            "algbw_gbs_p50": 2 * count / (p50 * 1e-6) / 1e9 if p50 > 0 else None,
            "ctas_per_rank": comm.launch_shape(op, proto, count)[0]}


def evaluate_selector(points, model):
    """Per swept (op, N, size): the model's choice vs the measured fastest of
    the protocols the model may choose (an opt-in protocol the model marks
    unavailable is not a candidate)."""
    best = {}
    for p in points:
        key = (p["op"], p["nranks"], p["bytes_per_rank"])
        if api.cost_estimate(model, p["op"], p["protocol"], p["bytes_per_rank"], p["nranks"]) < 0:
            continue
        if key not in best or p["p50_us"] < best[key]["p50_us"]:
            best[key] = p
    rows = []
    for key, bp in sorted(best.items()):
        op, n, nbytes = key
        chosen = api.select_protocol_model(model, op, nbytes, n).name.lower()
        cps = [p for p in points if (p["op"], p["nranks"], p["bytes_per_rank"]) == key and p["protocol"] == chosen]
        if not cps:
            continue
        rows.append({"op": op, "nranks": n, "bytes_per_rank": nbytes, "selector": chosen,
                     "best": bp["protocol"], "regret": cps[0]["p50_us"] / bp["p50_us"]})
    return rows


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--nranks", type=int, nargs="+", default=[2, 4, 8])
    ap.add_argument("--op", default="allreduce", choices=["allreduce", "allgather"])
    ap.add_argument("--protocols", nargs="+",
                    default=["ll", "ll128", "sentinel", "barrier_oneshot", "barrier_twoshot", "barrier_oneshot_db",
                             "ll_twoshot", "sentinel_twoshot", "ll128_fast"])
    ap.add_argument("--min-bytes", type=int, default=1024)
    ap.add_argument("--max-bytes", type=int, default=64 << 20)
    ap.add_argument("--k-ops", type=int, default=50)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--ctas-per-rank", type=int, default=0)
    ap.add_argument("--sizes", type=int, nargs="+", default=None, help="explicit bytes per rank")
    ap.add_argument("--out", default=None)
    ap.add_argument("--model-from", nargs="+", default=None, help="sweep JSONL files for the selector model")
    ap.add_argument("--report", default=None, help="write the selector evaluation here (JSON)")
    a = ap.parse_args(argv)
    dev = torch.device("cuda")
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    sizes = []
    b = a.min_bytes
    while b <= a.max_bytes:
        sizes.append(b)
        b *= 2
    if a.sizes:
        sizes = sorted(a.sizes)
    ar_only = ("barrier_twoshot", "ll_twoshot", "sentinel_twoshot")
    protos = [p for p in a.protocols if not (a.op == "allgather" and p in ar_only)]
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
    if a.model_from:
        from .gen_cost_table import cost_model_from_points, load_points

        model = cost_model_from_points(load_points(a.model_from))
    else:
        model = api.default_cost_model()
    rows = evaluate_selector(points, model)
    for row in rows:
        print(json.dumps(dict(row, kind="selector")), flush=True)
    if rows:
        regrets = [r["regret"] for r in rows]
        summary = {"regret_median": statistics.median(regrets), "regret_max": max(regrets),
                   "points": len(rows)}
        print(json.dumps(summary), flush=True)
        if a.report:
            with open(a.report, "w") as f:
                json.dump({"summary": summary, "rows": rows}, f, indent=1)
    if sink:
        sink.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
