"""Record DRAM traffic from an ncu capture into profiles/ncu_traffic.json.

    python -m latency_self_synchronizing_b200.ncu_record bench   LAUNCHES.csv
    python -m latency_self_synchronizing_b200.ncu_record targets LAUNCHES.csv

LAUNCHES.csv is ncu's `--csv --log-file` output of a capture with the
metrics dram__bytes_read.sum, dram__bytes_write.sum and gpu__time_duration.sum
of the chain kernels (`-k regex:sfc_kernel`):

* bench: `python bench.py --steps 2 --warmup 3 --no-cpu-baseline --no-targets`
  captured with `--nvtx --nvtx-include timed/ -c 4` (the first timed step:
  one chain launch per token count);
* targets: `python bench.py --targets-only --large-only` captured with
  `--nvtx --nvtx-include targets_large/`, every launch (per large point one
  warm-up chain and three timed chains, points in the order the bench
  measures them).

The entries are keyed as bench.py looks them up (kernel, operations, bytes
per rank, grid, block) and stamped with the current kernel-source hash, so
the bench reports them only while the kernels are the ones captured. Only
parses and writes JSON; runs nothing on a GPU.
"""

import csv
import io
import json
import os
import statistics
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TRAFFIC = os.path.join(ROOT, "profiles", "ncu_traffic.json")


def _bench():
    sys.path.insert(0, ROOT)
    import bench

    return bench


def read_launches(path):
    """[{id, name, grid, block, dram_bytes, duration_us}] in launch order."""
    lines = [ln for ln in open(path, encoding="utf-8", errors="replace") if ln.startswith('"')]
    rows = list(csv.DictReader(io.StringIO("".join(lines))))
    by_id = {}
    for row in rows:
        lid = int(row["ID"])
        ent = by_id.setdefault(lid, {"id": lid, "name": row["Kernel Name"], "grid": row["Grid Size"],
                                     "block": row["Block Size"], "m": {}})
        val = float(row["Metric Value"].replace(",", ""))
        unit = row["Metric Unit"].strip().lower()
        scale = {"byte": 1, "kbyte": 1e3, "mbyte": 1e6, "gbyte": 1e9, "ns": 1e-3, "nsecond": 1e-3, "us": 1,
                 "usecond": 1, "ms": 1e3, "msecond": 1e3}.get(unit, 1)
        ent["m"][row["Metric Name"]] = val * scale
    out = []
    for lid in sorted(by_id):
        e = by_id[lid]
        m = e["m"]
        out.append({"id": lid, "name": e["name"], "grid": int(e["grid"].strip("()").split(",")[0]),
                    "block": int(e["block"].strip("()").split(",")[0]),
                    "dram_bytes": m.get("dram__bytes_read.sum", 0.0) + m.get("dram__bytes_write.sum", 0.0),
                    "duration_us": m.get("gpu__time_duration.sum")})
    return [x for x in out if "sfc_kernel" in x["name"]]


def _save(entries, command):
    bench = _bench()
    try:
        rec = json.load(open(TRAFFIC))
    except (OSError, ValueError):
        rec = {}
    sha = bench.kernel_sources_sha()
    if rec.get("kernel_sources_sha") != sha:
        rec = {"launches": {}}
    rec["what"] = ("DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of chain kernels, "
                   "from ncu captures of the commands listed")
    rec["kernel_sources_sha"] = sha
    rec.setdefault("commands", [])
    if command not in rec["commands"]:
        rec["commands"].append(command)
    rec.setdefault("launches", {}).update(entries)
    rec["keyed_on"] = ("kernel_sources_sha = SHA-256 of the chain kernels' device sources (comments and layout "
                       "excluded), the nvcc flags and the compiler version (bench.py kernel_sources_sha); grid "
                       "and block = the captured launch, which bench.py compares with the live one")
    with open(TRAFFIC, "w") as f:
        json.dump(rec, f, indent=1)
        f.write("\n")


def record_bench(path):
    bench = _bench()
    launches = read_launches(path)
    if len(launches) != len(bench.TOKENS):
        raise SystemExit(f"expected {len(bench.TOKENS)} chain launches, found {len(launches)}")
    entries = {}
    for t, la in zip(bench.TOKENS, launches):
        b = 2 * bench.HIDDEN * t
        key = f"sfc_kernel<{bench.NRANKS}, {bench.PROTOCOL}, allreduce> x {bench.K_OPS} ops, {b} B/rank"
        entries[key] = {"dram_bytes_per_launch": la["dram_bytes"], "duration_us_under_ncu": la["duration_us"],
                        "grid": la["grid"], "block": la["block"]}
    _save(entries, "ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum "
                   "--clock-control none --nvtx --nvtx-include timed/ -k regex:sfc_kernel -c 4 --csv "
                   "--log-file LAUNCHES.csv python bench.py --steps 2 --warmup 3 --no-cpu-baseline --no-targets")
    return entries


def record_targets(path):
    bench = _bench()
    from latency_self_synchronizing_b200 import api

    model = api.default_cost_model()
    launches = read_launches(path)
    points = [(n, b) for n in bench.TARGET_RANKS for b in bench.TARGET_LARGE]
    per_point = len(launches) // len(points) if points else 0
    if per_point < 2 or per_point * len(points) != len(launches):
        raise SystemExit(f"{len(launches)} chain launches for {len(points)} points")
    entries = {}
    for i, (n, b) in enumerate(points):
        group = launches[i * per_point:(i + 1) * per_point][1:]  # the first chain is the warm-up
        proto = api.select_protocol_model(model, "allreduce", b, n).name.lower()
        k = bench.large_point_inputs(n, b)
        key = f"sfc_kernel<{n}, {proto}, allreduce> x {k} ops, {b} B/rank"
        entries[key] = {"dram_bytes_per_launch": statistics.median(x["dram_bytes"] for x in group),
                        "duration_us_under_ncu": statistics.median(x["duration_us"] for x in group),
                        "grid": group[0]["grid"], "block": group[0]["block"]}
    _save(entries, "ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum "
                   "--clock-control none --nvtx --nvtx-include targets_large/ -k regex:sfc_kernel --csv "
                   "--log-file LAUNCHES.csv python bench.py --targets-only --large-only")
    return entries


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    if len(argv) != 2 or argv[0] not in ("bench", "targets"):
        raise SystemExit(__doc__)
    ent = record_bench(argv[1]) if argv[0] == "bench" else record_targets(argv[1])
    for k, v in ent.items():
        print(k, v)
    return 0


if __name__ == "__main__":
    sys.exit(main())
