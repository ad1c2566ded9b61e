"""bench.py's CPU baselines (the oracle timed on the host cores): one core,
and one spawned process per core, on a small workload."""
import bench
from sp_synth import WORKLOADS


def test_cpu_baselines_report_their_sample_and_cores():
    w = WORKLOADS["C2"].replace(s=64, b=1)
    cb = bench.cpu_baseline(w, bench.fwd_bytes(w), bench.bwd_bytes(w), budget_s=0.2)
    assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] > 0
    ac = cb["all_cores"]
    assert ac["kind"] == "oracle" and ac["cores"] >= 1 and ac["value"] > 0
    assert "one process per core" in ac["sample"]
