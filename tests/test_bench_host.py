"""bench.py's host-side bookkeeping, on CPU: the algorithmic work each stage is divided by, the
peak denominators, and the measured-traffic table.

The per-stage formulas are checked against totals derived independently from the method's data
flow (per configuration: forward bytes, backward bytes, attention FLOPs), so that a dropped or
doubled term in any stage shows up as a wrong total.
"""
import importlib.util
import json
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_host_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


# Totals of the method's data flow, counted once (bf16, e = 2 bytes):
#   forward  = read Q, K, V + write pyramid levels + write and read the scores + gather
#              (read and write 3 * S rows) + scatter (read O_sub, write O), plus the int32 ids
#   backward = span sums (read dO, write dO_sub) + gather backward (read 3 fp32 sub-gradients,
#              write dQ, dK, dV), plus the ids
#   attention FLOPs: 2 B H S^2 d forward and 5 B H S^2 d backward (causal)
# in GB (1e9 bytes) and GFLOP, rounded to the digits below. The table's forward total counts
# O_sub in bf16; the library keeps O_sub in fp32, which adds B H S d (4 - 2) bytes to the scatter.
EXPECTED = {
    "32k": dict(fwd=0.79, bwd=0.65, attn_fwd=69, attn_bwd=172),
    "llama530m-98k": dict(fwd=1.11, bwd=0.89, attn_fwd=77, attn_bwd=193),
    "128k": dict(fwd=5.88, bwd=4.77, attn_fwd=550, attn_bwd=1374),
    "1m": dict(fwd=11.06, bwd=8.83, attn_fwd=550, attn_bwd=1374),
}


def _levels_rows(w):
    return sum(w.N // w.p ** l for l in range(1, w.L))


@pytest.mark.parametrize("name", sorted(EXPECTED))
def test_stage_work_matches_the_data_flow_totals(name):
    bench = _bench()
    w = bench.WORKLOADS[name]
    work = bench.stage_work(w, {"R": _levels_rows(w)})
    kinds = {k: v[0] for k, v in work.items()}
    assert kinds == {"pyramid_score": "hbm", "select": "hbm", "gather": "hbm", "attn_fwd": "tensor",
                     "scatter": "hbm", "scatter_bwd": "hbm", "attn_bwd": "tensor", "gather_bwd": "hbm"}
    osub_fp32_extra = w.B * w.H * w.S * w.d * (4 - 2)
    fwd = sum(work[k][1] for k in ("pyramid_score", "select", "gather", "scatter")) - osub_fp32_extra
    bwd = sum(work[k][1] for k in ("scatter_bwd", "gather_bwd"))
    want = EXPECTED[name]
    assert fwd / 1e9 == pytest.approx(want["fwd"], abs=0.006)
    assert bwd / 1e9 == pytest.approx(want["bwd"], abs=0.006)
    assert work["attn_fwd"][1] / 1e9 == pytest.approx(want["attn_fwd"], rel=0.005)
    assert work["attn_bwd"][1] / 1e9 == pytest.approx(want["attn_bwd"], rel=0.005)


def test_peaks_come_from_the_measured_file():
    bench = _bench()
    pk, src = bench.peaks()
    with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
        raw = json.load(f)
    assert src == "measured"
    for key in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained"):
        assert pk[key] == raw[key] > 0  # the denominators are the file's, not the fallback


def test_measured_traffic_names_real_workloads_and_stages():
    bench = _bench()
    stages = set(bench.stage_work(bench.WORKLOADS["128k"], {"R": _levels_rows(bench.WORKLOADS["128k"])}))
    assert set(bench.STAGE_SOURCES) == stages
    for (workload, stage), (nbytes, digest, how) in bench.MEASURED_TRAFFIC.items():
        assert workload in bench.WORKLOADS
        assert stage in stages
        assert isinstance(nbytes, int) and nbytes > 0 and len(digest) == 16 and how


def test_traffic_goes_stale_when_the_kernel_sources_change():
    bench = _bench()
    digest = bench.source_digest("attn_bwd")
    bench.MEASURED_TRAFFIC[("128k", "attn_bwd")] = (123, digest, "test")
    assert bench.traffic_of("128k", "attn_bwd") == (123, False, "test")
    bench.MEASURED_TRAFFIC[("128k", "attn_bwd")] = (123, "0" * 16, "test")
    nbytes, stale, _ = bench.traffic_of("128k", "attn_bwd")
    assert nbytes is None and stale
    assert bench.traffic_of("1m", "select")[0] is None
