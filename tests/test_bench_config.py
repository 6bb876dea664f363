"""bench.py measures the named decode workload it reports (no GPU needed)."""
import importlib.util
import os

from latency_self_synchronizing_b200.workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_bench_constants_are_the_decode_h8192_workload():
    b = _bench()
    w = WORKLOADS["decode_h8192"]
    assert b.NRANKS == w["nranks"]
    assert [b.PROTOCOL] == w["protocols"]
    assert [b.HIDDEN * t for t in b.TOKENS] == w["counts"]
    assert b.K_OPS == w["k_ops"]
    cfg = b._config()
    assert cfg["workload"] == "decode_h8192"
    assert cfg["bytes_per_rank"] == [2 * c for c in w["counts"]]
    assert cfg["nranks"] == w["nranks"] and cfg["protocol"] == b.PROTOCOL and cfg["k_ops_per_chain"] == b.K_OPS


def test_bench_metric_is_time_like():
    b = _bench()
    assert "p50" in b.METRIC


def test_cpu_baselines_shape():
    """The two CPU figures of the bench line, on the smallest sample."""
    import json

    b = _bench()
    cpu, thr = b.cpu_baselines(sample_ops=1, tokens=(1,))
    assert cpu["kind"] == "oracle" and cpu["cores"] == 1 and cpu["value"] > 0 and cpu["host_cores"] >= 1
    assert thr["value"] > 0 and thr["cores"] >= 1 and set(thr["us_per_op_by_tokens"]) == {"1"}
    json.dumps({"cpu_baseline": cpu, "cpu_threaded": thr})


def test_recorded_traffic_is_keyed_on_device_sources_and_launch_shape(monkeypatch):
    b = _bench()
    key = "sfc_kernel<4, sentinel, allreduce> x 160 ops, 131072 B/rank"
    import json

    rec = json.load(open(os.path.join(ROOT, "profiles", "ncu_traffic.json")))
    ent = rec["launches"][key]
    if rec["kernel_sources_sha"] == b.kernel_sources_sha():
        assert b.recorded_traffic(key, grid=ent["grid"], block=ent["block"]) == ent["dram_bytes_per_launch"]
        assert b.recorded_traffic(key, grid=ent["grid"] // 2, block=ent["block"]) is None
        assert b.recorded_traffic(key, grid=ent["grid"], block=ent["block"] // 2) is None
    monkeypatch.setattr(b, "kernel_sources_sha", lambda: "0" * 64)  # the kernels changed since the capture
    assert b.recorded_traffic(key, grid=ent["grid"], block=ent["block"]) is None
    for rel in b.KERNEL_SOURCES:
        assert os.path.exists(os.path.join(ROOT, rel)), rel


def test_large_target_points_read_their_inputs_from_hbm():
    b = _bench()
    for n in b.TARGET_RANKS:
        for nbytes in b.TARGET_LARGE:
            k = b.large_point_inputs(n, nbytes)
            assert 8 <= k <= 128
            total = k * n * nbytes
            assert total <= (3 << 29) or k == 8          # bounded device memory
            assert total >= 2 * b.L2_BYTES or k == 128   # inputs twice the L2 unless capped


def test_ncu_record_parses_a_launch_list(tmp_path, monkeypatch):
    from latency_self_synchronizing_b200 import ncu_record

    hdr = '"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size",' \
          '"Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"\n'
    rows = []
    for lid, (name, grid) in enumerate([("void sfc::sfc_kernel<4, 3, 0>(sfc::KParams)", 32),
                                        ("void other_kernel(int)", 1)]):
        for metric, unit, val in [("dram__bytes_read.sum", "Mbyte", "10.5"), ("dram__bytes_write.sum", "Kbyte", "500"),
                                  ("gpu__time_duration.sum", "usecond", "278.5")]:
            rows.append(f'"{lid}","1","python","h","{name}","1","7","(128, 1, 1)","({grid}, 1, 1)","0","10.0",'
                        f'"Command line profiler metrics","{metric}","{unit}","{val}"\n')
    p = tmp_path / "launches.csv"
    p.write_text("==PROF== noise\n" + hdr + "".join(rows))
    got = ncu_record.read_launches(str(p))
    assert len(got) == 1  # only the chain kernels
    assert got[0]["grid"] == 32 and got[0]["block"] == 128
    assert got[0]["dram_bytes"] == 10.5e6 + 500e3
    assert got[0]["duration_us"] == 278.5
