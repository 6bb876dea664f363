"""Host logic of the selector tooling (no GPU): the measured table's
provenance, its bucketing, the model built from sweep points, and the regret
evaluation of the sweep."""
import glob
import math
import os

import pytest

from latency_self_synchronizing_b200 import api, gen_cost_table as gct, sweep

PKG = os.path.dirname(os.path.abspath(api.__file__))
CAL = sorted(glob.glob(os.path.join(PKG, "calibration", "*.jsonl")))


def test_builtin_table_is_the_committed_calibration(tmp_path):
    """The table compiled into libsfc is exactly what the generator writes
    from the committed sweep files."""
    assert CAL, "no calibration sweeps committed"
    out = gct.write_header(gct.load_points(CAL), str(tmp_path / "t.h"))
    assert open(out).read() == open(gct.DEFAULT_OUT).read()


def test_builtin_model_reproduces_the_calibration_points():
    """Every measured power-of-two point of the calibration is what the
    library's built-in model estimates there."""
    m = api.default_cost_model()
    checked = 0
    for p in gct.load_points(CAL):
        b = int(p["bytes_per_rank"])
        if b & (b - 1) or not gct.MIN_LOG2 <= int(math.log2(b)) < gct.MIN_LOG2 + gct.BUCKETS:
            continue
        if p["protocol"] == "ll128_fast":  # opt-in: no estimate in the default model
            continue
        est = api.cost_estimate(m, p["op"], p["protocol"], b, p["nranks"])
        assert est == pytest.approx(round(float(p["p50_us"]), 3), abs=5e-4), p
        checked += 1
    assert checked > 500


def _pt(op, proto, n, b, p50):
    return {"op": op, "protocol": proto, "nranks": n, "bytes_per_rank": b, "p50_us": p50}


def test_table_from_points_buckets():
    pts = [_pt("allreduce", "ll", 4, 512, 1.0), _pt("allreduce", "ll", 4, 1024, 2.0),
           _pt("allreduce", "ll", 4, 1536, 9.0),       # not a power of two: ignored
           _pt("allreduce", "ll", 4, 256, 9.0),        # below the first bucket: ignored
           _pt("allreduce", "ll", 4, 1 << 33, 9.0)]    # past the last bucket: ignored
    row = gct.table_from_points(pts)[("allreduce", "ll", 4)]
    assert row[0] == 1.0 and row[1] == 2.0
    assert sum(v is not None for v in row) == 2


def test_model_from_points_interpolates_in_log2_and_chooses_the_minimum():
    # values below every built-in entry, so that only these two compete
    pts = [_pt("allreduce", "ll", 4, 1 << 12, 0.2), _pt("allreduce", "ll", 4, 1 << 14, 0.4),
           _pt("allreduce", "sentinel", 4, 1 << 12, 0.3), _pt("allreduce", "sentinel", 4, 1 << 14, 0.3)]
    m = gct.cost_model_from_points(pts)
    # halfway in log2 between 4 KB and 16 KB is 8 KB: 0.2 + (0.4 - 0.2) / 2
    assert api.cost_estimate(m, "allreduce", "ll", 1 << 13, 4) == pytest.approx(0.3)
    assert api.select_protocol_model(m, "allreduce", 1 << 12, 4) == api.Protocol.LL
    assert api.select_protocol_model(m, "allreduce", 1 << 14, 4) == api.Protocol.SENTINEL


def test_evaluate_selector_regret():
    m = api.default_cost_model()
    b, n = 1 << 14, 4
    chosen = api.select_protocol_model(m, "allreduce", b, n).name.lower()
    other = "barrier_twoshot" if chosen != "barrier_twoshot" else "ll"
    pts = [_pt("allreduce", chosen, n, b, 2.0), _pt("allreduce", other, n, b, 1.0),
           _pt("allreduce", "ll128_fast", n, b, 0.1)]  # opt-in, not a candidate of the default model
    rows = sweep.evaluate_selector(pts, m)
    assert len(rows) == 1
    r = rows[0]
    assert r["selector"] == chosen and r["best"] == other and r["regret"] == pytest.approx(2.0)
