"""Benchmark: p50 / p99 microseconds per emulated N-rank all-reduce.

Default workload ``decode_h8192``: 4 emulated ranks, sentinel protocol with
epoch-parity double buffering, hidden 8192 x tokens {1, 2, 4, 8} (16-128 KB
per rank), normal(0,1) inputs, 160 chained all-reduces per decode step
(80 layers x 2). One step = one persistent launch of 160 chained
all-reduces for each of the four token counts. The headline value is the p50
per-operation latency at 1 token (16 KB per rank), taken from in-kernel
%globaltimer completion stamps; every size is reported under ``per_size``.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {sfc,reference}]

Under torchrun each process runs its own emulated instance on its own GPU
(replicas: the method emulates all ranks inside one GPU); the reported
latency is the maximum over processes.

``--impl reference`` times the CPU oracle (the protocol simulator) on the
host cores on a bounded sample of the same workload.
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "p50 us per emulated N-rank all-reduce vs size; achieved HBM GB/s vs roofline"
NRANKS = 4
HIDDEN = 8192
TOKENS = (1, 2, 4, 8)
K_OPS = 160
PROTOCOL = "sentinel"
DROP_FIRST = 5  # per-chain warm-up operations left out of the percentiles


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max_over_ranks(values, device=None):
    """Element-wise maximum of a list of floats over all processes (the
    replicas' reported latencies); the identity with one process."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def _percentile(v, q):
    v = sorted(v)
    if not v:
        return float("nan")
    i = min(len(v) - 1, max(0, int(round(q * (len(v) - 1)))))
    return float(v[i])


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """SM clock and throttle-reason samples (NVML, read only) every 2 ms while
    the timed region runs; nvidia-smi is the fallback when NVML is missing."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.samples = []
        self.stop_flag = False
        self.thread = None
        self.err = None

    def _run(self):
        import pynvml

        try:
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            while not self.stop_flag:
                sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                try:
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                except AttributeError:
                    rs = pynvml.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                self.samples.append((sm, rs))
                time.sleep(0.002)
        except Exception as e:  # NVML missing or refused: report it
            self.err = repr(e)

    def start(self):
        import threading

        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()
        t0 = time.time()
        while not self.samples and self.err is None and time.time() - t0 < 5:
            time.sleep(0.005)

    def stop(self):
        self.stop_flag = True
        if self.thread is not None:
            self.thread.join(timeout=5)
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "samples": 0, "reasons": [self.err or "no samples"]}
        reasons = sorted({n for _, rs in self.samples for n, bit in self.REASONS.items() if rs & bit})
        return {"sm_mhz": statistics.median(s for s, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples), "reasons": reasons, "source": "NVML"}


# ----------------------------------------------------------------- oracle
def time_oracle(sample_ops=3, tokens=1, budget_s=25.0):
    """The CPU oracle (protocol simulator, fixed linear schedule) on a
    bounded sample of the workload; returns (us per all-reduce, description)."""
    from latency_self_synchronizing_b200.inputs import make_inputs
    from oracle import simulator

    count = HIDDEN * tokens
    x = make_inputs(seed=0, k_ops=sample_ops, nranks=NRANKS, count=count, dist="normal", params=(1.0,))
    t0 = time.perf_counter()
    done = 0
    for k in range(sample_ops):
        _, v = simulator.run_fifo(PROTOCOL, x[k:k + 1])
        if v:
            raise RuntimeError(f"oracle reported violations: {v[:2]}")
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    desc = (f"oracle protocol simulator ({PROTOCOL}, fixed schedule), {NRANKS} ranks, hidden {HIDDEN} x "
            f"{tokens} token(s), {done} all-reduce(s), single thread")
    return dt / done * 1e6, desc


def time_threaded(tokens=TOKENS):
    """The concurrent CPU model (one thread per rank, C11 atomics, same
    protocol and chain) on the bench's workload; returns ({tokens: us per
    all-reduce}, threads, description). Every output is checked against the
    closed form on op 0 and the last op."""
    from latency_self_synchronizing_b200.inputs import make_inputs
    from oracle import reference, threaded

    per = {}
    for t in tokens:
        x = make_inputs(seed=0, k_ops=K_OPS, nranks=NRANKS, count=HIDDEN * t, dist="normal", params=(1.0,))
        out, secs = threaded.chain(PROTOCOL, x)
        for k in (0, K_OPS - 1):
            if not all(np.array_equal(out[k, r], reference.allreduce(x[k])) for r in range(NRANKS)):
                raise RuntimeError("threaded CPU model disagrees with the closed form")
        per[t] = secs / K_OPS * 1e6
    threads = NRANKS
    desc = (f"threaded C model ({PROTOCOL}), {NRANKS} threads, {K_OPS} chained all-reduces per size, "
            f"hidden {HIDDEN} x {list(tokens)} token(s)")
    return per, threads, desc


def cpu_baselines(sample_ops=8, tokens=TOKENS):
    """The bench line's two CPU figures: the oracle's simulator on a bounded
    sample (`cpu_baseline`) and the concurrent C model on whole chains
    (`cpu_threaded`, reported as an error string if it cannot run)."""
    v, desc = time_oracle(sample_ops=sample_ops)
    cpu = {"value": v, "unit": "us", "cores": 1, "kind": "oracle", "sample": desc, "host_cores": os.cpu_count()}
    try:
        per, threads, desc = time_threaded(tokens)
        cpu_threaded = {"value": per[tokens[0]], "unit": "us", "cores": min(threads, os.cpu_count() or 1),
                        "kind": "concurrent CPU model", "sample": desc, "host_cores": os.cpu_count(),
                        "us_per_op_by_tokens": {str(t): v for t, v in per.items()}}
    except (OSError, RuntimeError, subprocess.CalledProcessError) as exc:  # a side figure: keep the line
        cpu_threaded = {"value": None, "error": f"{type(exc).__name__}: {exc}"}
    return cpu, cpu_threaded


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    vals = []
    desc = ""
    for _ in range(args.warmup):
        time_oracle(sample_ops=1)
    for _ in range(args.steps):
        v, desc = time_oracle(sample_ops=1)
        vals.append(v)
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "us", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": value / 1e3, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": _config(),
        "cpu_baseline": {"value": value, "unit": "us", "cores": 1, "kind": "oracle", "sample": desc,
                         "host_cores": os.cpu_count()},
        "e2e": {"value": value, "unit": "us", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def _config():
    return {"workload": "decode_h8192", "nranks": NRANKS, "protocol": PROTOCOL, "hidden": HIDDEN,
            "tokens": list(TOKENS), "headline_tokens": 1, "k_ops_per_chain": K_OPS,
            "bytes_per_rank": [2 * HIDDEN * t for t in TOKENS], "inputs": "normal(0,1), seed 0",
            "l2": "flushed between steps (write of 2x L2 size, outside the timed events)",
            "parallelism": "replicas (emulated ranks inside each GPU)"}


# ---------------------------------------------------------------- targets
TARGET_RANKS = (2, 4, 8)
TARGET_SMALL = (1024, 16384)        # bytes per rank: latency target, <= 3x the flag round trip
TARGET_LARGE = (1 << 20, 16 << 20)  # bytes per rank: bandwidth target, >= 0.5 of the HBM roofline
L2_BYTES = 126 * 1024 * 1024


def large_point_inputs(nranks, nbytes, l2_bytes=L2_BYTES):
    """Distinct inputs per chain for a bandwidth point: enough operations
    that the chain's inputs are at least twice the L2 (every operation reads
    its inputs from HBM), at least 8, at most 128 and at most 1.5 GB."""
    per_op = nranks * nbytes
    need = -(-2 * l2_bytes // per_op)
    cap = max(8, (3 << 29) // per_op)
    return int(min(128, cap, max(8, need)))


def measure_targets(dev, floor_us, peak_gbs, large_only=False):
    """The selector's protocol at the target points, measured as chains
    outside the timed region: p50 per operation against the flag round-trip
    floor at small sizes; algorithmic and recorded-DRAM bandwidth fractions
    at large sizes (inputs larger than L2). large_only skips the small
    points (the launches an ncu traffic capture records, in this order)."""
    import torch

    from latency_self_synchronizing_b200 import api, sweep

    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    small, large = [], []
    for n in TARGET_RANKS:
        sel = api.Communicator(n, 1 << 10)  # every protocol provisioned: the selector's own choice
        try:
            chosen = {b: sel.select_protocol("allreduce", b, n).name.lower() for b in TARGET_SMALL + TARGET_LARGE}
        finally:
            sel.close()
        for b in () if large_only else TARGET_SMALL:
            proto = chosen[b]
            comm = api.Communicator(n, b, protocols=[proto])
            try:
                pt = sweep.measure_point(comm, "allreduce", proto, b // 2, 100, 3, gen, dev)
            finally:
                comm.close()
            small.append({"nranks": n, "bytes_per_rank": b, "protocol": proto, "p50_us": pt["p50_us"],
                          "p99_us": pt["p99_us"], "floor_ratio": pt["p50_us"] / floor_us,
                          "met": pt["p50_us"] / floor_us <= 3.0})
        for b in TARGET_LARGE:
            proto = chosen[b]
            k = large_point_inputs(n, b)
            comm = api.Communicator(n, b, protocols=[proto])
            try:
                torch.cuda.nvtx.range_push("targets_large")  # the launches an ncu traffic capture records
                pt = sweep.measure_point(comm, "allreduce", proto, b // 2, k, 3, gen, dev, distinct=k)
                torch.cuda.nvtx.range_pop()
                shape = comm.launch_shape("allreduce", proto, b // 2)
            finally:
                comm.close()
                torch.cuda.empty_cache()
            alg = pt["algorithmic_bytes"] / (pt["p50_us"] * 1e-6) / 1e9
            key = f"sfc_kernel<{n}, {proto}, allreduce> x {k} ops, {b} B/rank"
            traffic = recorded_traffic(key, grid=n * shape[0], block=shape[1])
            dram = None if traffic is None else traffic / k / (pt["p50_us"] * 1e-6) / 1e9
            large.append({"nranks": n, "bytes_per_rank": b, "protocol": proto, "p50_us": pt["p50_us"],
                          "p99_us": pt["p99_us"], "k_ops": k, "algorithmic_bytes_per_op": pt["algorithmic_bytes"],
                          "algorithmic_gbs": alg, "algorithmic_frac": alg / peak_gbs,
                          "dram_bytes_per_op": None if traffic is None else traffic / k,
                          "dram_gbs": dram, "dram_frac": None if dram is None else dram / peak_gbs,
                          "met": alg / peak_gbs >= 0.5, "ncu_key": key})
    return {"small": small, "large": large,
            "what": "selector's protocol per point; chains of 100 ops (small, 8 distinct inputs) or of k distinct "
                    "inputs totalling >= 2x L2 (large); p50 from completion stamps; floor = flag round trip; "
                    "dram = ncu-recorded DRAM bytes of the same launch (null when the kernels changed since)",
            "small_met": all(p["met"] for p in small) if small else None,
            "large_met": all(p["met"] for p in large)}


def run_targets_only(args):
    """--targets-only: the target points alone, one JSON line (no timed step,
    no floor unless small points are measured)."""
    import torch

    from latency_self_synchronizing_b200 import api

    torch.cuda.set_device(_dist()[2])
    dev = torch.device("cuda", _dist()[2])
    floor_us = float("nan") if args.large_only else api.measure_floor(500)["flag_rtt_ns_p50"] / 1e3
    t = measure_targets(dev, floor_us, _peaks()["hbm_gbs"], large_only=args.large_only)
    print(json.dumps({"targets": t, "floor_us": floor_us}))
    return 0


# -------------------------------------------------------------------- GPU
def run_gpu(args):
    import torch
    import torch.distributed as dist

    from latency_self_synchronizing_b200 import api
    from latency_self_synchronizing_b200.inputs import make_inputs

    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    if ws > 1:
        dist.init_process_group("nccl", device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    peaks = _peaks()
    max_count = HIDDEN * max(TOKENS)
    comm = api.Communicator(NRANKS, max_count * 2, protocols=[PROTOCOL, "ll", "ll128"])
    floor = api.measure_floor(500)

    # operands: 160 distinct inputs per rank, outputs alternate two buffers
    chains = []
    for t in TOKENS:
        count = HIDDEN * t
        x = make_inputs(seed=0, k_ops=K_OPS, nranks=NRANKS, count=count, dist="normal", params=(1.0,))
        xin = torch.from_numpy(x.reshape(-1).view(np.int16)).to(dev)
        outb = torch.zeros(2 * NRANKS * count, dtype=torch.int16, device=dev)
        tin = torch.tensor([xin.data_ptr() + 2 * count * i for i in range(K_OPS * NRANKS)], dtype=torch.int64,
                           device=dev)
        tout = torch.tensor([outb.data_ptr() + 2 * count * ((k % 2) * NRANKS + r)
                             for k in range(K_OPS) for r in range(NRANKS)], dtype=torch.int64, device=dev)
        chains.append(dict(tokens=t, count=count, x=x, xin=xin, outb=outb, tin=tin, tout=tout))
    l2_flush = torch.empty(2 * 126 * 1024 * 1024, dtype=torch.int8, device=dev)
    stream = torch.cuda.current_stream()

    def step(timings=None, events=None):
        for i, c in enumerate(chains):
            if events is not None:
                events[i][0].record(stream)
            comm.allreduce_chain(c["tin"], c["tout"], c["count"], K_OPS, protocol=PROTOCOL,
                                 timings=None if timings is None else timings[i])
            if events is not None:
                events[i][1].record(stream)

    for _ in range(args.warmup):
        l2_flush.zero_()
        step()
    torch.cuda.synchronize()
    st, info = comm.status()
    if st != api.Status.OK:
        raise RuntimeError(f"device status {st.name} info {info:#x}")

    tims = [[torch.zeros(K_OPS + 1, dtype=torch.int64, device=dev) for _ in TOKENS] for _ in range(args.steps)]
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in TOKENS]
           for _ in range(args.steps)]
    launches0 = comm.launch_count
    clocks = ClockSampler(local)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t_start = time.perf_counter()
    wall0 = torch.cuda.Event(enable_timing=True)
    wall1 = torch.cuda.Event(enable_timing=True)
    wall0.record(stream)
    torch.cuda.nvtx.range_push("timed")  # ncu captures select this range (--nvtx --nvtx-include timed/)
    for s in range(args.steps):
        l2_flush.zero_()
        step(tims[s], evs[s])
    torch.cuda.nvtx.range_pop()
    wall1.record(stream)
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    clk = clocks.stop()
    gpu_launches = comm.launch_count - launches0
    st, info = comm.status()
    if st != api.Status.OK:
        raise RuntimeError(f"device status {st.name} info {info:#x}")

    # per-size latencies from the completion stamps
    per_size = []
    step_ms = []
    for s in range(args.steps):
        step_ms.append(sum(evs[s][i][0].elapsed_time(evs[s][i][1]) for i in range(len(TOKENS))))
    for i, c in enumerate(chains):
        lat = []
        launch_ms = []
        for s in range(args.steps):
            h = tims[s][i].cpu().numpy().astype(np.int64)
            d = np.diff(h[1:])  # completion(k) - completion(k-1), k >= 1
            lat.extend((d[DROP_FIRST - 1:] / 1e3).tolist())
            launch_ms.append(evs[s][i][0].elapsed_time(evs[s][i][1]))
        count = c["count"]
        bytes_op = api.algorithmic_bytes("allreduce", PROTOCOL, count, NRANKS)
        p50 = _percentile(lat, 0.5)
        mean_launch_us = statistics.mean(launch_ms) * 1e3
        per_size.append({
            "tokens": c["tokens"], "bytes_per_rank": 2 * count, "p50_us": p50, "p99_us": _percentile(lat, 0.99),
            "mean_us_from_events": mean_launch_us / K_OPS,
            "algorithmic_bytes_per_op": bytes_op,
            "achieved_gbs_p50": bytes_op / (p50 * 1e-6) / 1e9 if p50 > 0 else None,
            "algbw_gbs_p50": 2 * count / (p50 * 1e-6) / 1e9 if p50 > 0 else None,
            "achieved_gbs_launch": bytes_op * K_OPS / (mean_launch_us * 1e-6) / 1e9,
            "floor_ratio_p50": p50 / (floor["flag_rtt_ns_p50"] / 1e3),
            "launch_shape": comm.launch_shape("allreduce", PROTOCOL, count),
        })
        torch.cuda.synchronize()

    # correctness spot check of the last step's final outputs (bits only, no oracle)
    # is done by the test suite; here only the status is checked.

    # e2e: host buffers through the C ABI, copies inside the timed region
    t1 = chains[0]
    hin = torch.from_numpy(t1["x"].view(np.int16)).view(torch.bfloat16).contiguous().pin_memory()
    hout = torch.empty_like(hin).pin_memory()
    e2e_ms = []
    for s in range(args.warmup + args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        comm.allreduce_chain_host(hin, hout, protocol=PROTOCOL)
        b.record(stream)
        torch.cuda.synchronize()
        if s >= args.warmup:
            e2e_ms.append(a.elapsed_time(b))
    e2e_us = statistics.median(e2e_ms) * 1e3 / K_OPS
    h2d = hin.numel() * 2

    # single calls (one launch per all-reduce, launch included): reported
    # beside the chained latency, not the headline
    xs = [torch.from_numpy(t1["x"][0, r].view(np.int16)).view(torch.bfloat16).to(dev) for r in range(NRANKS)]
    ys = [torch.empty_like(t) for t in xs]
    for _ in range(20):
        comm.allreduce(xs, ys, protocol=PROTOCOL)
    torch.cuda.synchronize()
    n_calls = 200
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(n_calls):
        comm.allreduce(xs, ys, protocol=PROTOCOL)
    b.record(stream)
    torch.cuda.synchronize()
    single_b2b = a.elapsed_time(b) * 1e3 / n_calls
    # the same call prepared once (sfc_plan_create), launched back to back
    plan = comm.plan(xs, ys, protocol=PROTOCOL)
    for _ in range(20):
        plan.launch()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(n_calls):
        plan.launch()
    b.record(stream)
    torch.cuda.synchronize()
    plan_b2b = a.elapsed_time(b) * 1e3 / n_calls
    plan.close()
    iso = []
    for _ in range(50):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        comm.allreduce(xs, ys, protocol=PROTOCOL)
        b.record(stream)
        torch.cuda.synchronize()
        iso.append(a.elapsed_time(b) * 1e3)
    # the same calls captured in a CUDA graph (device-epoch context) and
    # replayed: launch gaps on the GPU only, no host work per call
    gcomm = api.Communicator(NRANKS, 2 * t1["count"], device_epochs=True, protocols=[PROTOCOL])
    gys = [torch.empty_like(t) for t in xs]
    gcomm.allreduce(xs, gys, protocol=PROTOCOL)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(K_OPS):
            gcomm.allreduce(xs, gys, protocol=PROTOCOL)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    g_us = []
    for _ in range(5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        graph.replay()
        b.record(stream)
        torch.cuda.synchronize()
        g_us.append(a.elapsed_time(b) * 1e3 / K_OPS)
    gst, ginfo = gcomm.status()
    if gst != api.Status.OK:
        raise RuntimeError(f"graph context status {gst.name} info {ginfo:#x}")
    if not torch.equal(gys[0], ys[0]):
        raise RuntimeError("graph-replayed all-reduce differs from the eager one")
    del graph
    gcomm.close()
    single = {"back_to_back_us": single_b2b, "plan_back_to_back_us": plan_b2b,
              "isolated_us_p50": _percentile(iso, 0.5),
              "graph_replay_us": statistics.median(g_us), "unit": "us",
              "what": f"sfc_allreduce, one launch per call, {2 * t1['count']} B/rank; back to back = "
                      f"{n_calls} calls between two events; plan = the same call prepared once "
                      f"(sfc_plan_create) and launched {n_calls} times; isolated = one call between two events; "
                      f"graph replay = {K_OPS} calls captured in one CUDA graph (device epochs), per call"}
    st, info = comm.status()
    if st != api.Status.OK:
        raise RuntimeError(f"device status {st.name} info {info:#x}")

    head = per_size[0]
    value = head["p50_us"]
    value, e2e_us = reduce_max_over_ranks([value, e2e_us], device=dev)

    dom = per_size[-1]  # largest size: most time per step
    ach = dom["achieved_gbs_launch"]
    key = f"sfc_kernel<{NRANKS}, sentinel, allreduce> x {K_OPS} ops, {dom['bytes_per_rank']} B/rank"
    roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": ach / peaks["hbm_gbs"],
            "traffic": recorded_traffic(key, grid=NRANKS * dom["launch_shape"][0], block=dom["launch_shape"][1]),
            "algorithmic_bytes_per_launch": dom["algorithmic_bytes_per_op"] * K_OPS,
            "peak_source": peaks["source"], "kernel": key}

    targets = None if args.no_targets else measure_targets(dev, floor["flag_rtt_ns_p50"] / 1e3, peaks["hbm_gbs"])

    cpu = cpu_threaded = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu, cpu_threaded = cpu_baselines()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "us", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": statistics.mean(step_ms), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": _config(), "per_size": per_size,
            "floor": {"flag_rtt_us_p50": floor["flag_rtt_ns_p50"] / 1e3,
                      "flag_rtt_us_p10": floor["flag_rtt_ns_p10"] / 1e3,
                      "flag_rtt_us_p90": floor["flag_rtt_ns_p90"] / 1e3,
                      "flag_rtt_us_fastest_trial": floor["flag_rtt_ns_min_pair"] / 1e3,
                      "flag_rtt_us_slowest_trial": floor["flag_rtt_ns_max_pair"] / 1e3,
                      "flag_rtt_us_by_location": [v / 1e3 for v in floor["flag_rtt_ns_by_location"]],
                      "initiator_sms": floor["initiator_sm"], "responder_sms": floor["responder_sm"],
                      "trials": floor["pairs"],
                      "statistic": "median over (SM pair x flag address) trials of each trial's median round trip",
                      "l2_rtt_us": floor["l2_rtt_ns_p50"] / 1e3,
                      "sol_analogue_us": (2 * floor["l2_rtt_ns_p50"] + floor["flag_rtt_ns_p50"] / 2) / 1e3,
                      "globaltimer_step_ns": floor["globaltimer_step_ns"], "sm_clock_ghz": floor["sm_clock_ghz"],
                      "headline_ratio": value / (floor["flag_rtt_ns_p50"] / 1e3)},
            "roofline": roof,
            "targets": targets,
            "cpu_baseline": cpu,
            "cpu_threaded": cpu_threaded,
            "e2e": {"value": e2e_us, "unit": "us", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": h2d,
                    "min_max": [min(e2e_ms) * 1e3 / K_OPS, max(e2e_ms) * 1e3 / K_OPS],
                    "what": f"sfc_allreduce_chain_host, {K_OPS} ops at {2 * t1['count']} B/rank, per op"},
            "single_call": single,
            "gpu_launches": int(gpu_launches),
            "wall_s": time.perf_counter() - t_start,
            "clocks": clk,
        }
        print(json.dumps(line))
    comm.close()
    if ws > 1:
        dist.destroy_process_group()
    return 0


KERNEL_SOURCES = ("latency_self_synchronizing_b200/csrc/sfc_kernels.cu",
                  "latency_self_synchronizing_b200/csrc/sfc_device.cuh",
                  "latency_self_synchronizing_b200/csrc/sfc_internal.h",
                  "include/sfc.h", "include/sfc_ll_device.cuh")


def _code_only(text):
    """C/C++ source with comments removed and whitespace runs collapsed
    (string and character literals kept as they are)."""
    out, i, n = [], 0, len(text)
    while i < n:
        ch = text[i]
        if text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif ch in "\"'":
            j = i + 1
            while j < n and text[j] != ch:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            out.append(ch)
            i += 1
    return " ".join("".join(out).split())


def _nvcc_version():
    from latency_self_synchronizing_b200 import build

    try:
        out = subprocess.run([build._nvcc(), "--version"], capture_output=True, text=True, timeout=60).stdout
    except (OSError, RuntimeError, subprocess.SubprocessError):
        return "nvcc: unknown"
    return " ".join(line for line in out.splitlines() if "release" in line or "Build" in line)


def kernel_sources_sha():
    """SHA-256 over the code of the chain kernels' device sources (kernels,
    device helpers, the parameter block and its constants, the public
    headers they include), comments and layout excluded, plus the nvcc
    architecture flags, compile flags and compiler version the library is
    built with. How a chain is launched is checked live instead: a recorded
    capture also names its grid and block."""
    import hashlib

    from latency_self_synchronizing_b200 import build

    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        h.update(rel.encode())
        h.update(_code_only(open(os.path.join(ROOT, rel), encoding="utf-8").read()).encode())
    flags = [f for f in build.FLAGS if not f.startswith("/")]  # include paths differ between machines
    h.update(" ".join(build.ARCH + flags).encode())
    h.update(_nvcc_version().encode())
    return h.hexdigest()


def recorded_traffic(key, grid=None, block=None):
    """DRAM bytes per launch recorded from an ncu capture of this kernel and
    workload (profiles/ncu_traffic.json), or None when the kernel sources have
    changed since the capture or the launch now has another grid or block."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        rec = json.load(open(path))
    except (OSError, ValueError):
        return None
    if rec.get("kernel_sources_sha") != kernel_sources_sha():
        return None
    ent = rec.get("launches", {}).get(key)
    if ent is None:
        return None
    if (grid is not None and ent.get("grid") != grid) or (block is not None and ent.get("block") != block):
        return None
    return float(ent["dram_bytes_per_launch"])


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured (MEASURED_PEAKS.json hbm_gbs)"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "source": "fallback 6.65 TB/s"}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["sfc", "reference"], default="sfc")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-targets", action="store_true", help="skip the selector target points")
    ap.add_argument("--targets-only", action="store_true", help="measure only the selector target points")
    ap.add_argument("--large-only", action="store_true", help="with --targets-only: the >= 1 MB points only")
    args = ap.parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.targets_only:
        return run_targets_only(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
