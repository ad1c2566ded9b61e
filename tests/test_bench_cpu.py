"""bench.py's CPU baselines (the oracle timed on the host cores): one core,
and one spawned process per core, on a small workload; and the source set
that keys the recorded traffic."""
import os

import bench
from sp_synth import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_cpu_baselines_report_their_sample_and_cores():
    w = WORKLOADS["C2"].replace(s=64, b=1)
    cb = bench.cpu_baseline(w, bench.fwd_bytes(w), bench.bwd_bytes(w), budget_s=0.2)
    assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] > 0
    ac = cb["all_cores"]
    assert ac["kind"] == "oracle" and ac["cores"] >= 1 and ac["value"] > 0
    assert "one process per core" in ac["sample"]


def test_algorithmic_bytes_follow_the_stated_formulas():
    """The roofline's numerator: C2's forward reads t+1 rows and writes 2 rows
    of 2 bytes per element plus the mask and statistics (1.114 GB), and the
    backward the same with the parameter gradients.  With an fp32 residual
    stream its tensors count 4 bytes per element."""
    w = WORKLOADS["C2"]
    N, h, t = w.rows, w.h, w.t
    sbh, W = N * h, (h + 31) // 32
    fwd = (t + 1) * 2 * sbh + 3 * 2 * h + 2 * 2 * sbh + 4 * W * N + 8 * N
    bwd = (t + 1) * 2 * sbh + 4 * W * N + 8 * N + 2 * h + 2 * 2 * sbh + 4 * h * 3
    assert bench.fwd_bytes(w) == fwd and round(fwd / 1e9, 3) == 1.114
    assert bench.bwd_bytes(w) == bwd
    wr = w.replace(res_dtype="f32")
    assert bench.fwd_bytes(wr) == fwd + 2 * 2 * sbh          # residual, residual_out
    assert bench.bwd_bytes(wr) == bwd + 2 * 2 * sbh          # x, dresidual_in
    assert bench.bwd_bytes(wr, with_drnext=True) == bwd + 3 * 2 * sbh + 2 * sbh
    # the entry: read x, write the gathered rows
    e = bench.entry_fwd_bytes(w)
    assert e == 2 * sbh + 2 * 2 * h + 2 * sbh + 8 * N


def test_traffic_hash_covers_the_streaming_kernels_sources():
    """The recorded DRAM traffic is keyed by a hash of the files the streaming
    kernels are built from: their translation units and every file those
    include, transitively, and nothing else."""
    import re
    csrc = os.path.join(ROOT, "sp_region_b200", "csrc")
    todo, seen = ["sp_region.cu", "sp_inst_fwd.cu", "sp_inst_bwd.cu"], set()
    while todo:
        f = todo.pop()
        path = os.path.join(csrc, f)
        if f in seen or not os.path.exists(path):
            continue
        seen.add(f)
        todo += re.findall(r'#include "([^"]+)"', open(path).read())
    assert seen == set(bench.STREAMING_SOURCES)
