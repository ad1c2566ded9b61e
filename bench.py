#!/usr/bin/env python
"""Benchmark of the B200 sequence-parallel boundary (forward + backward).

One step is one pass of the whole hot path over one batch of synthetic input
(the C2 workload: s=2048, b=4, h=6144, t=8 emulated ranks, bf16 I/O, fp32
arithmetic, LayerNorm, dropout p=0.1, bias):

  forward   sp_rs_bias_dropout_add_norm_fwd: reduce-scatter of the 8 partial
            sums + bias + dropout + residual + LayerNorm + all-gather write
  backward  sp_rs_norm_dropout_bwd: reduce-scatter of the 8 upstream gradient
            partials + LayerNorm / residual / dropout backward + all-gathered
            dY + dgamma / dbeta / dbias

The metric is achieved HBM bandwidth on the algorithmic bytes of both calls
(GB/s), with tokens/s and the fraction of the measured HBM peak beside it.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]

With N > 1 (launched by torch.distributed.run) every rank runs an independent
replica on its own GPU (weak scaling; the path has no exchange between
replicas); the time is the maximum over ranks.  ``--mode ranks`` instead runs
the boundary itself on t = N ranks, the partial sums, gathered outputs and
gradients in symmetric memory reached by the kernels over NVLink, beside
NCCL's all-reduce and reduce-scatter + all-gather on the same bytes.
``--impl reference`` times the CPU oracle on the host cores instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SP-boundary fwd+bwd achieved HBM GB/s (% of B200 peak); tokens/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ----------------------------------------------------------------------------
# algorithmic bytes (per call), from the data each call must move
# ----------------------------------------------------------------------------

# E: bytes per element of the I/O dtype; Er: of the residual stream
# (residual, residual_out, x, dR_next, dresidual_in), fp32 with --residual-f32
def fwd_bytes(w, n_gathered=1, with_mask=True):
    E, Er, N, h = w.elem_bytes, w.res_elem_bytes, w.rows, w.h
    sbh = N * h
    W = (h + 31) // 32
    params = h * E * (1 + (1 if w.has_bias else 0) +
                      (1 if (w.has_beta and w.norm == "layernorm") else 0))
    rd = w.t * E * sbh + Er * sbh + params
    stats = (8 if w.norm == "layernorm" else 4) * N
    wr = Er * sbh + E * sbh * n_gathered + (4 * W * N if with_mask else 0) + stats
    return rd + wr


def all_gather_bytes(w, n_out):
    """Standalone all-gather: every shard read once, written n_out times."""
    return w.elem_bytes * w.rows * w.h * (1 + n_out)


def bwd_bytes(w, with_drnext=False):
    E, Er, N, h = w.elem_bytes, w.res_elem_bytes, w.rows, w.h
    sbh = N * h
    W = (h + 31) // 32
    stats = (8 if w.norm == "layernorm" else 4) * N
    rd = w.t * E * sbh + Er * sbh + 4 * W * N + stats + h * E
    if with_drnext:
        rd += Er * sbh
    ngrad = 1 + (1 if w.norm == "layernorm" else 0) + (1 if w.has_bias else 0)
    wr = Er * sbh + E * sbh + 4 * h * ngrad
    return rd + wr


def entry_fwd_bytes(w, n_gathered=1):
    """Entry into a TP region: read x, write the gathered norm output."""
    E, Er, N, h = w.elem_bytes, w.res_elem_bytes, w.rows, w.h
    params = h * E * (1 + (1 if w.norm == "layernorm" else 0))
    stats = (8 if w.norm == "layernorm" else 4) * N
    return Er * N * h + params + n_gathered * E * N * h + stats


def entry_bwd_bytes(w):
    """Its backward: reduce-scatter of t upstream partials, norm backward from
    x and the statistics, the residual-stream gradient written."""
    E, Er, N, h = w.elem_bytes, w.res_elem_bytes, w.rows, w.h
    stats = (8 if w.norm == "layernorm" else 4) * N
    ngrad = 1 + (1 if w.norm == "layernorm" else 0)
    return (w.t * E + Er) * N * h + stats + h * E + Er * N * h + 4 * h * ngrad


def workload_of(args):
    """The named workload; --residual-f32 keeps its residual stream in fp32."""
    import sp_synth
    w = sp_synth.WORKLOADS[args.workload]
    if getattr(args, "residual_f32", False) and w.dtype == "bf16":
        w = w.replace(res_dtype="f32")
    return w


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (no MEASURED_PEAKS.json)"


def measured_tensor_peak():
    """Dense bf16 TFLOP/s for a kernel timed on its own (the burst figure)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops)"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback (no MEASURED_PEAKS.json)"


# the translation units of the streaming kernels (k_fwd_tma, k_bwd_tma,
# k_colreduce, k_norm_ag) and every file they include: the recorded traffic
# depends on these and on nothing else (the linears and ring attention are
# built in their own unit)
STREAMING_SOURCES = ("sp_region.cu", "sp_inst_fwd.cu", "sp_inst_bwd.cu", "sp_bwd.cuh",
                     "sp_device.cuh", "sp_entry.cuh", "sp_fwd.cuh", "sp_gather.cuh",
                     "sp_host.h", "sp_plans.h")


def kernel_sources_sha():
    """Hash of the sources the streaming kernels are built from (their csrc
    files and the header)."""
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "sp_region_b200", "csrc")
    files = [os.path.join(csrc, f) for f in sorted(STREAMING_SOURCES)]
    for f in files + [os.path.join(ROOT, "include", "sp_region.h")]:
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:12]


def recorded_traffic(kernel_key):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    sha = kernel_sources_sha()
    for line in open(p):
        if line.startswith("#") or "=" not in line:
            continue
        kv = dict(x.split("=", 1) for x in line.split())
        if kv.get("key") == kernel_key and kv.get("src_sha1") == sha:
            return float(kv["dram_bytes_per_launch"])
    return None


# ----------------------------------------------------------------------------
# aggregation over ranks (N independent replicas)
# ----------------------------------------------------------------------------

def max_over_ranks(local_ms, device=None):
    """The job's time is the slowest rank's: all-reduce MAX of the local
    device-timed milliseconds (a no-op without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or \
            dist.get_world_size() == 1:
        return float(local_ms)
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_step, steps, world, max_ms):
    """Whole-job GB/s: the bytes every rank processed over the job's time."""
    return bytes_per_step * world * steps / (max_ms * 1e-3) / 1e9


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.samples = []   # (host time, sm, max, power, reasons...)
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev),
                 f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 7:
                self.samples.append((time.time(), *parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0, t1):
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed"
        if not win:
            win = self.samples
            window = "whole run (timed region shorter than the sampling period)"
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                    "samples": 0, "note": "nvidia-smi unavailable"}
        sm = [num(s[1]) for s in win if num(s[1]) is not None]
        mx = [num(s[2]) for s in win if num(s[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = sorted({names[i] for s in win for i in range(4)
                          if s[4 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(win), "window": window}


# ----------------------------------------------------------------------------
# the GPU arm
# ----------------------------------------------------------------------------

def run_ours(args):
    import torch
    import torch.distributed as dist
    import sp_synth
    import sp_region_b200 as sp

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    w = workload_of(args)
    w = w.replace(seed=w.seed + 1000 * rank)   # each replica its own batch
    N, h, t = w.rows, w.h, w.t
    dt = w.torch_dtype
    res_f32 = w.res != w.dtype
    cfg = sp.make_cfg(w.s, w.b, h, t, dtype=w.dtype, norm=w.norm, eps=w.eps,
                      p_drop=w.p_drop, seed=w.drop_seed, offset=w.drop_offset,
                      fwd_plan=args.fwd_plan, bwd_plan=args.bwd_plan,
                      res_f32=res_f32)

    parts = sp_synth.draw_partials(w, dev)
    bias, gamma, beta = sp_synth.draw_params(w, dev)
    if not w.has_bias:
        bias = None
    if not w.has_beta or w.norm == "rmsnorm":
        beta = None
    res = sp_synth.draw_residual(w, dev)
    dparts = sp_synth.draw_grad_partials(w, dev)
    rdt = w.res_torch_dtype
    rout = torch.empty((N, h), dtype=rdt, device=dev)
    out = torch.empty((N, h), dtype=dt, device=dev)
    mask = torch.empty((N, (h + 31) // 32), dtype=torch.int32, device=dev)
    mean = torch.empty(N, dtype=torch.float32, device=dev)
    rstd = torch.empty(N, dtype=torch.float32, device=dev)
    dres = torch.empty((N, h), dtype=rdt, device=dev)
    dY = torch.empty((N, h), dtype=dt, device=dev)
    dg = torch.empty(h, dtype=torch.float32, device=dev)
    db = torch.empty(h, dtype=torch.float32, device=dev) \
        if w.norm == "layernorm" else None
    dc = torch.empty(h, dtype=torch.float32, device=dev) if bias is not None \
        else None
    ws = torch.empty(sp.sp_bwd_workspace_bytes(cfg, local) // 4,
                     dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def fwd():
        sp.sp_rs_bias_dropout_add_norm_fwd(cfg, parts, bias, res, gamma, beta,
                                           rout, [out], mask, mean, rstd,
                                           stream=stream)

    def bwd():
        sp.sp_rs_norm_dropout_bwd(cfg, dparts, None, rout, gamma, mask, mean,
                                  rstd, dres, dY, dg, db, dc, ws,
                                  stream=stream)

    if args.op == "entry":
        # the entry into a TP region: norm of the shard then all-gather; its
        # backward: reduce-scatter of the upstream partials, norm backward
        cfg0 = sp.make_cfg(w.s, w.b, h, t, dtype=w.dtype, norm=w.norm,
                           eps=w.eps, p_drop=0.0, fwd_plan=args.fwd_plan,
                           bwd_plan=args.bwd_plan, res_f32=res_f32)

        def fwd():
            sp.sp_norm_all_gather_fwd(cfg0, res, gamma, beta, [out], mean,
                                      rstd, stream=stream)

        def bwd():
            sp.sp_rs_norm_dropout_bwd(cfg0, dparts, None, res, gamma, None,
                                      mean, rstd, dres, None, dg, db, None,
                                      ws, stream=stream)

    for _ in range(args.warmup):
        fwd()
        bwd()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)]
           for _ in range(K)]
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)   # let the sampler start before the timed region
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    h0 = time.time()
    e0.record(stream)
    for i in range(K):
        evs[i][0].record(stream)
        fwd()
        evs[i][1].record(stream)
        bwd()
        evs[i][2].record(stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    h1 = time.time()
    if world > 1:
        dist.barrier()
    clocks.stop()
    assert sp.sp_device_error(local) == 0, "device-side wait timed out"

    fwd_ms = [evs[i][0].elapsed_time(evs[i][1]) for i in range(K)]
    bwd_ms = [evs[i][1].elapsed_time(evs[i][2]) for i in range(K)]
    total_ms = max_over_ranks(e0.elapsed_time(e1), dev)

    if args.op == "entry":
        fb, bb = entry_fwd_bytes(w), entry_bwd_bytes(w)
    else:
        fb, bb = fwd_bytes(w), bwd_bytes(w)
    step_bytes = fb + bb
    value = job_throughput(step_bytes, K, world, total_ms)
    ms_step = total_ms / K
    peak, peak_src = measured_peak()
    f_avg = statistics.mean(fwd_ms)
    b_avg = statistics.mean(bwd_ms)
    kern = {
        "fwd": {"kernel": "k_norm_ag" if args.op == "entry" else "k_fwd_tma",
                "bytes_per_launch": fb,
                "avg_ms": f_avg, "gbs": fb / (f_avg * 1e-3) / 1e9},
        "bwd": {"kernel": "k_bwd_tma + k_colreduce", "bytes_per_launch": bb,
                "avg_ms": b_avg, "gbs": bb / (b_avg * 1e-3) / 1e9},
    }
    dom = "fwd" if f_avg >= b_avg else "bwd"
    dk = kern[dom]
    traffic = recorded_traffic(f"{dom}:{args.workload}" +
                               (":entry" if args.op == "entry" else "") +
                               (":res_f32" if w.res != w.dtype else ""))
    roofline = {"bound": "hbm", "achieved": round(dk["gbs"], 1),
                "peak": peak, "unit": "GB/s",
                "frac": round(dk["gbs"] / peak, 4), "traffic": traffic,
                "kernel": dk["kernel"], "call": dom,
                "peak_source": peak_src,
                "algorithmic_bytes_per_launch": dk["bytes_per_launch"]}

    e2e = None
    cpu = None
    workloads = None
    linears = None
    attention = None
    if args.op == "boundary":
        e2e = run_e2e(args, w, cfg, sp, torch, dev, step_bytes, world)
        if world == 1 and args.workloads:
            workloads = time_workloads(args, sp, torch, dev, peak)
        if world == 1 and not args.skip_linears:
            linears = time_linears(args, sp, torch, dev)
            attention = time_ring_attention(args, sp, torch, dev)
        if rank == 0 and world == 1 and not args.skip_cpu_baseline:
            cpu = cpu_baseline(w, fb, bb, budget_s=args.cpu_seconds)

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "io_dtype": w.dtype, "data": "synthetic",
        "config": {
            "workload": (f"{w.name}: SP boundary fwd+bwd, s={w.s} b={w.b} "
                         f"h={h} t={t} emulated ranks, {w.dtype} I/O, "
                         f"{w.norm}, p={w.p_drop}, bias"
                         + (", fp32 residual stream" if w.res != w.dtype else "")
                         if args.op == "boundary" else
                         f"{w.name} shape: entry into a TP region (norm + "
                         f"all-gather) fwd+bwd, s={w.s} b={w.b} h={h} t={t}, "
                         f"{w.dtype} I/O, {w.norm}"
                         + (", fp32 residual stream" if w.res != w.dtype else "")),
            "s": w.s, "b": w.b, "h": h, "t": t,
            "global_batch": w.b * world, "seq_len": w.s,
            "parallelism": f"{world} independent replicas (t={t} ranks "
                           "emulated in one GPU's HBM each)",
            "l2": "inputs larger than L2: each step streams "
                  f"{step_bytes / 1e9:.2f} GB of distinct buffers (L2 126 MB)"},
        "tokens_per_s": round(N * world / (ms_step * 1e-3), 1),
        "pct_of_8TBs": round(100 * value / world / NOMINAL_HBM_GBS, 2),
        "pct_of_measured_peak": round(100 * value / world / peak, 2),
        "roofline": roofline,
        "kernels": kern,
        "workloads": workloads,
        "tp_linears": linears,
        "ring_attention": attention,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": 3 * K,
        "plan_hints": {"fwd": args.fwd_plan, "bwd": args.bwd_plan},
        "clocks": clocks.summary(h0, h1),
    }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def time_launches(torch, stream, fn, steps, warmup):
    """Average device time of one call of fn, from CUDA events recorded on
    the launching stream around each of `steps` calls (after `warmup`)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in evs)


def time_workloads(args, sp, torch, dev, peak):
    """Forward and backward of every workload at full size (C2 to C5), each
    timed on its own with CUDA events, plus C3's forward with the all-gather
    written as t per-rank replicas and the standalone all-gather into t
    replicas.  Inputs are resident in HBM and larger than L2."""
    import gc
    import sp_synth
    out = {}
    stream = torch.cuda.current_stream(dev)
    for name in args.workloads.split(","):
        if not name:
            continue
        w = sp_synth.WORKLOADS[name]
        N, h, t = w.rows, w.h, w.t
        dt = w.torch_dtype
        cfg = sp.make_cfg(w.s, w.b, h, t, dtype=w.dtype, norm=w.norm,
                          eps=w.eps, p_drop=w.p_drop, seed=w.drop_seed,
                          offset=w.drop_offset)
        parts = sp_synth.draw_partials(w, dev)
        bias, gamma, beta = sp_synth.draw_params(w, dev)
        if not w.has_bias:
            bias = None
        if not w.has_beta or w.norm == "rmsnorm":
            beta = None
        res = sp_synth.draw_residual(w, dev)
        with_mask = w.p_drop > 0
        rout = torch.empty((N, h), dtype=dt, device=dev)
        gath = [torch.empty((N, h), dtype=dt, device=dev)
                for _ in range(t if w.gather_replicas else 1)]
        mask = (torch.empty((N, (h + 31) // 32), dtype=torch.int32,
                            device=dev) if with_mask else None)
        mean = torch.empty(N, dtype=torch.float32, device=dev)
        rstd = torch.empty(N, dtype=torch.float32, device=dev)
        rec = {"workload": f"{name}: s={w.s} b={w.b} h={h} t={t} {w.dtype} "
                           f"{w.norm} p={w.p_drop}"
                           + (" bias" if w.has_bias else "")
                           + (" 1% x100 outliers" if w.outliers else "")}
        K = 10 if N * h > 2e8 else 40

        def entry(kernel, nbytes, ms):
            gbs = nbytes / (ms * 1e-3) / 1e9
            return {"kernel": kernel, "bytes_per_launch": nbytes,
                    "avg_ms": round(ms, 5), "gbs": round(gbs, 1),
                    "frac": round(gbs / peak, 4),
                    "pct_of_8TBs": round(100 * gbs / NOMINAL_HBM_GBS, 2)}

        def fwd(n=1):
            sp.sp_rs_bias_dropout_add_norm_fwd(cfg, parts, bias, res, gamma,
                                               beta, rout, gath[:n], mask,
                                               mean if w.norm == "layernorm"
                                               else None, rstd, stream=stream)
        ms = time_launches(torch, stream, fwd, K, 3)
        rec["fwd"] = entry("k_fwd_tma", fwd_bytes(w, 1, with_mask), ms)
        if w.gather_replicas:
            ms = time_launches(torch, stream, lambda: fwd(t), K, 3)
            rec["fwd_all_gather_replicas"] = entry(
                "k_fwd_tma (t gathered replicas)", fwd_bytes(w, t, with_mask),
                ms)
            shards = [gath[0][r * (N // t):(r + 1) * (N // t)]
                      for r in range(t)]
            ms = time_launches(torch, stream, lambda: sp.sp_all_gather(
                cfg, shards, gath[1:], stream=stream), K, 3)
            rec["all_gather"] = entry(f"k_all_gather_bulk ({t - 1} replicas)",
                                      all_gather_bytes(w, t - 1), ms)
        del parts
        gc.collect()
        dparts = sp_synth.draw_grad_partials(w, dev)
        dres = torch.empty((N, h), dtype=dt, device=dev)
        dY = torch.empty((N, h), dtype=dt, device=dev)
        dg = torch.empty(h, dtype=torch.float32, device=dev)
        db = torch.empty(h, dtype=torch.float32, device=dev) \
            if w.norm == "layernorm" else None
        dc = torch.empty(h, dtype=torch.float32, device=dev) \
            if bias is not None else None
        ws = torch.empty(sp.sp_bwd_workspace_bytes(cfg, dev.index) // 4,
                         dtype=torch.float32, device=dev)

        def bwd():
            sp.sp_rs_norm_dropout_bwd(cfg, dparts, None, rout, gamma, mask,
                                      mean if w.norm == "layernorm" else None,
                                      rstd, dres, dY, dg, db, dc, ws,
                                      stream=stream)
        ms = time_launches(torch, stream, bwd, K, 3)
        rec["bwd"] = entry("k_bwd_tma + k_colreduce", bwd_bytes(w), ms)
        out[name] = rec
        del dparts, dres, dY, rout, gath, res, ws
        gc.collect()
        torch.cuda.empty_cache()
    assert sp.sp_device_error(dev.index) == 0, "device-side wait timed out"
    return out


def time_linears(args, sp, torch, dev):
    """The tensor-parallel linears around the boundary at the C2 layer shape
    (s=2048, b=4, h=6144, t=8), the FFN down-projection f = 4h = 24576 as
    the row-parallel linear and the up-projection h -> 4h as the
    column-parallel one, synthetic bf16 inputs:

      fused      sp_linear_rs_bias_dropout_add_norm_fwd: the GEMM whose
                 accumulator reduces the t partials, with bias / dropout /
                 residual in its epilogue, then norm + all-gather
      gemm       sp_rowpar_linear_rs_fwd alone (tensor roofline)
      unfused    t GEMMs each writing its partial [N, h] to HBM, then
                 sp_rs_bias_dropout_add_norm_fwd on the t partials
      colpar     sp_ag_colpar_linear_fwd reading the t shards directly
    """
    import gc
    import sp_synth
    w = sp_synth.WORKLOADS["C2"]
    N, h, t = w.rows, w.h, w.t
    f = 4 * h
    per = f // t
    stream = torch.cuda.current_stream(dev)
    peak, peak_src = measured_tensor_peak()
    g = torch.Generator(device=dev).manual_seed(4242)
    x = (torch.randn((N, f), generator=g, device=dev) * f ** -0.5).to(torch.bfloat16)
    wt = torch.randn((h, f), generator=g, device=dev).to(torch.bfloat16)
    bias, gamma, beta = sp_synth.draw_params(w, dev)
    res = sp_synth.draw_residual(w, dev)
    rout = torch.empty((N, h), dtype=torch.bfloat16, device=dev)
    out = torch.empty((N, h), dtype=torch.bfloat16, device=dev)
    mask = torch.empty((N, (h + 31) // 32), dtype=torch.int32, device=dev)
    mean = torch.empty(N, dtype=torch.float32, device=dev)
    rstd = torch.empty(N, dtype=torch.float32, device=dev)
    cfg = sp.make_cfg(w.s, w.b, h, t, dtype="bf16", norm=w.norm, eps=w.eps,
                      p_drop=w.p_drop, seed=w.drop_seed, offset=w.drop_offset)
    flops = 2.0 * N * f * h
    K = 10

    def rec(kernel, ms, nflops=flops):
        tf = nflops / (ms * 1e-3) / 1e12
        return {"kernel": kernel, "avg_ms": round(ms, 4), "tflops": round(tf, 1),
                "frac": round(tf / peak, 4), "flops_per_launch": nflops}

    fused_ms = time_launches(torch, stream, lambda: sp.sp_linear_rs_bias_dropout_add_norm_fwd(
        cfg, f, x, wt, bias, res, gamma, beta, rout, [out], mask, mean, rstd,
        stream=stream), K, 3)
    gemm_ms = time_launches(torch, stream, lambda: sp.sp_rowpar_linear_rs_fwd(
        cfg, f, x, wt, bias, res, rout, mask, stream=stream), K, 3)
    # the unfused path: each rank's slice in its own buffers, its partial
    # written to HBM, then the boundary on the t partials
    xs = [x[:, k * per:(k + 1) * per].contiguous() for k in range(t)]
    ws = [wt[:, k * per:(k + 1) * per].contiguous() for k in range(t)]
    parts = [torch.empty((N, h), dtype=torch.bfloat16, device=dev) for _ in range(t)]
    cfg1 = sp.make_cfg(N, 1, per, 1, dtype="bf16")

    def unfused():
        for k in range(t):
            sp.sp_ag_colpar_linear_fwd(cfg1, h, [xs[k]], ws[k], parts[k], stream=stream)
        sp.sp_rs_bias_dropout_add_norm_fwd(cfg, parts, bias, res, gamma, beta, rout,
                                           [out], mask, mean, rstd, stream=stream)
    unfused_ms = time_launches(torch, stream, unfused, K, 3)
    del xs, ws, parts, x, wt
    gc.collect()
    torch.cuda.empty_cache()
    # the column-parallel up-projection from the t shards of the norm output
    fo = 4 * h
    w_in = (torch.randn((fo, h), generator=g, device=dev) * h ** -0.5).to(torch.bfloat16)
    z = torch.empty((N, fo), dtype=torch.bfloat16, device=dev)
    shards = [out[r * (N // t):(r + 1) * (N // t)] for r in range(t)]
    cfg_c = sp.make_cfg(w.s, w.b, h, t, dtype="bf16")
    col_ms = time_launches(torch, stream, lambda: sp.sp_ag_colpar_linear_fwd(
        cfg_c, fo, shards, w_in, z, stream=stream), K, 3)
    assert sp.sp_device_error(dev.index) == 0, "device-side wait timed out"
    r = {
        "workload": (f"C2 layer: s={w.s} b={w.b} h={h} t={t}; row-parallel FFN "
                     f"down-projection f={f} -> h, then the SP boundary (LN, p=0.1, "
                     f"bias); column-parallel up-projection h -> {fo}; bf16"),
        "peak_tflops": peak, "peak_source": peak_src,
        "fused": rec("k_tp_gemm2 (CTA pairs, SP epilogue) + k_norm_ag", fused_ms),
        "gemm": rec("k_tp_gemm2 (CTA pairs, SP epilogue)", gemm_ms),
        "unfused": rec(f"{t} x k_tp_gemm2 (partials to HBM) + k_fwd_tma", unfused_ms),
        "colpar": rec("k_tp_gemm2 (CTA pairs, all-gather prologue)", col_ms, 2.0 * N * h * fo),
        "fused_speedup": round(unfused_ms / fused_ms, 3),
    }
    del w_in, z, out, rout, res
    gc.collect()
    torch.cuda.empty_cache()
    return r


def time_ring_attention(args, sp, torch, dev):
    """Ring attention over t = 16 context-parallel ranks at the long-sequence
    workload's length (s = 32768, head dimension 128 = 12288 / 96), two of its
    96 heads, b = 1, synthetic bf16 q, k, v ~ N(0, 1), scale 1/sqrt(128).
    FLOPs per call: 4 s^2 d per head (Q K^T and P V)."""
    import gc
    b, heads, s, t, d = 1, 2, 32768, 16, 128
    peak, peak_src = measured_tensor_peak()
    g = torch.Generator(device=dev).manual_seed(99)
    q, k, v = (torch.randn((b, heads, s, d), generator=g, device=dev).to(torch.bfloat16)
               for _ in range(3))
    out = torch.empty_like(q)
    lse = torch.empty((b, heads, s), dtype=torch.float32, device=dev)
    cfg = sp.make_cfg(s, b, heads * d, t, dtype="bf16")
    stream = torch.cuda.current_stream(dev)
    # the workspace call: the units of the last, partly filled round of SMs
    # run split over ranges of ring steps (k_attn_merge combines them)
    nbytes = sp.sp_ring_attention_workspace_bytes(cfg, heads, dev.index)
    ws = torch.empty(nbytes // 4 + 4, device=dev) if nbytes else None
    ms = time_launches(torch, stream, lambda: sp.sp_ring_attention_fwd_ws(
        cfg, heads, d ** -0.5, q, k, v, out, lse, ws, stream=stream), 3, 3)
    assert sp.sp_device_error(dev.index) == 0, "device-side wait timed out"
    flops = 4.0 * s * s * d * heads * b
    tf = flops / (ms * 1e-3) / 1e12
    del q, k, v, out, lse, ws
    gc.collect()
    torch.cuda.empty_cache()
    return {"workload": (f"C5 attention core: s={s}, t={t} ranks of {s // t} tokens, "
                         f"head dim {d}, {heads} heads, b={b}, bf16, full attention"),
            "kernel": "k_ring_attn + k_attn_merge", "workspace_bytes": nbytes,
            "avg_ms": round(ms, 3), "tflops": round(tf, 1),
            "frac": round(tf / peak, 4), "peak_tflops": peak, "peak_source": peak_src,
            "flops_per_launch": flops}


def collective_record(nbytes, ar_ms, rs_ag_ms, world, device=None):
    """The NCCL arm on the same bytes: one all-reduce against a
    reduce-scatter plus an all-gather, each timed per call on every rank and
    taken at the slowest rank.  Per-rank wire volume of either: 2 (t-1)/t of
    the tensor ("Sequence Parallelism math", section "Why the byte count is
    identical")."""
    ar = max_over_ranks(ar_ms, device)
    rs_ag = max_over_ranks(rs_ag_ms, device)
    wire = 2.0 * (world - 1) / world * nbytes
    return {"bytes": nbytes, "all_reduce_ms": round(ar, 4), "rs_ag_ms": round(rs_ag, 4),
            "rs_ag_over_all_reduce": round(rs_ag / ar, 4) if ar > 0 else None,
            "wire_bytes_per_rank": wire,
            "all_reduce_busbw_gbs": round(wire / (ar * 1e-3) / 1e9, 1) if ar > 0 else None}


def run_ranks(args):
    """The boundary on t = N real ranks, one GPU each, through peer memory:
    rank r runs the fused forward on its token rows, pulling its rows of every
    rank's partial sum (the reduce-scatter) and pushing its normalised rows
    into every rank's gathered buffer (the all-gather); the backward pulls the
    gradient partials and pushes dY the same way, then the replicated
    parameters' gradients are all-reduced.  Beside it, NCCL's all-reduce and
    reduce-scatter + all-gather on one partial-sum tensor."""
    import datetime
    import torch
    import torch.distributed as dist
    import torch.distributed._symmetric_memory as symm_mem
    import sp_synth
    import sp_region_b200 as sp
    from sp_region_b200.ranks import peer_buffers

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    w = workload_of(args).replace(t=world)
    N, h, t = w.rows, w.h, world
    per = N // t
    r0, r1 = rank * per, (rank + 1) * per
    dt = w.torch_dtype
    cfg = sp.make_cfg(w.s, w.b, h, t, dtype=w.dtype, norm=w.norm, eps=w.eps,
                      p_drop=w.p_drop, seed=w.drop_seed, offset=w.drop_offset,
                      row_begin=r0, row_end=r1)

    def shared(x):
        buf = symm_mem.empty(tuple(x.shape), dtype=x.dtype, device=dev)
        buf.copy_(x)
        return buf
    part = shared(sp_synth.draw_partials(w, dev)[rank])
    dpart = shared(sp_synth.draw_grad_partials(w, dev)[rank])
    out = shared(torch.zeros((N, h), dtype=dt, device=dev))
    dy = shared(torch.zeros((N, h), dtype=dt, device=dev))
    parts, gathered = peer_buffers(part), peer_buffers(out)
    dparts, dys = peer_buffers(dpart), peer_buffers(dy)
    bias, gamma, beta = sp_synth.draw_params(w, dev)
    res = sp_synth.draw_residual(w, dev)[r0:r1].contiguous()
    rout = torch.empty((per, h), dtype=dt, device=dev)
    mask = torch.empty((per, (h + 31) // 32), dtype=torch.int32, device=dev)
    mean = torch.empty(per, dtype=torch.float32, device=dev)
    rstd = torch.empty(per, dtype=torch.float32, device=dev)
    dres = torch.empty((per, h), dtype=dt, device=dev)
    grads = [torch.empty(h, dtype=torch.float32, device=dev) for _ in range(3)]
    ws = torch.empty(sp.sp_bwd_workspace_bytes(cfg, local) // 4, dtype=torch.float32,
                     device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        sp.sp_rs_bias_dropout_add_norm_fwd(cfg, parts, bias, res, gamma, beta, rout,
                                           gathered, mask, mean, rstd, stream=stream)
        sp.sp_rs_norm_dropout_bwd_ag(cfg, dparts, None, rout, gamma, mask, mean, rstd,
                                     dres, dys, *grads, ws, stream=stream)
        for g_ in grads:        # replicated parameters: sum over the ranks
            dist.all_reduce(g_)

    # every rank's inputs are written before any rank's kernel reads them
    torch.cuda.synchronize(dev)
    dist.barrier()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    K = args.steps
    e0.record(stream)
    for _ in range(K):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    assert sp.sp_device_error(local) == 0, "device-side wait timed out"
    total_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    step_bytes = fwd_bytes(w) + bwd_bytes(w)
    value = step_bytes * K / (total_ms * 1e-3) / 1e9

    # NCCL on one partial-sum tensor: all-reduce vs reduce-scatter + all-gather
    x = part.clone()
    shard = torch.empty((per, h), dtype=dt, device=dev)
    KC = 20

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize(dev)
        dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(KC):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / KC
    ar_ms = timed(lambda: dist.all_reduce(x))
    rs_ag_ms = timed(lambda: (dist.reduce_scatter_tensor(shard, x),
                              dist.all_gather_into_tensor(x, shard)))
    coll = collective_record(N * h * w.elem_bytes, ar_ms, rs_ag_ms, world, dev)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(total_ms / K, 5),
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": "f32", "io_dtype": w.dtype, "data": "synthetic", "mode": "ranks",
        "config": {"workload": (f"{w.name} shape on t={t} real ranks, one GPU each: rank r "
                                f"owns token rows [r*{per}, (r+1)*{per}); partials, gathered "
                                "outputs, gradient partials and dY in symmetric memory, "
                                "reached by the kernels over peer memory"),
                   "s": w.s, "b": w.b, "h": h, "t": t, "parallelism": f"sp{t}"},
        "nccl": coll,
        "gpu_launches": 3 * K,
    }
    for b_ in (out, dy, part, dpart):
        del b_
    dist.barrier()
    dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_e2e(args, w, cfg, sp, torch, dev, step_bytes, world):
    """Same metric through the public API with host buffers: every step
    copies its inputs from pinned host memory, runs forward and backward, and
    reads every output back to pinned host memory, inside the timed region.

    Steps are pipelined the way a caller with host buffers would run them:
    inputs are double-buffered on the device, uploads run on one copy stream,
    the boundary on the compute stream and downloads on another copy stream,
    so step i+1's upload overlaps step i's compute and download (PCIe carries
    both directions at once)."""
    import sp_synth
    N, h = w.rows, w.h
    dt = w.torch_dtype
    pin = lambda x: None if x is None else x.cpu().pin_memory()
    hp = [pin(p) for p in sp_synth.draw_partials(w, dev)]
    bias, gamma, beta = sp_synth.draw_params(w, dev)
    if not w.has_bias:
        bias = None
    if not w.has_beta or w.norm == "rmsnorm":
        beta = None
    hb, hg, hbe = pin(bias), pin(gamma), pin(beta)
    hr = pin(sp_synth.draw_residual(w, dev))
    hd = [pin(p) for p in sp_synth.draw_grad_partials(w, dev)]
    ins = [*hp, hb, hg, hbe, hr, *hd]
    h2d = sum(x.numel() * x.element_size() for x in ins if x is not None)
    t = w.t
    bufs = []
    for _ in range(2):
        dev_in = [None if x is None else torch.empty_like(x, device=dev)
                  for x in ins]
        bufs.append(dev_in)
    rdt = w.res_torch_dtype
    outs_d = dict(rout=torch.empty((N, h), dtype=rdt, device=dev),
                  out=torch.empty((N, h), dtype=dt, device=dev),
                  mask=torch.empty((N, (h + 31) // 32), dtype=torch.int32,
                                   device=dev),
                  mean=torch.empty(N, dtype=torch.float32, device=dev),
                  rstd=torch.empty(N, dtype=torch.float32, device=dev),
                  dres=torch.empty((N, h), dtype=rdt, device=dev),
                  dY=torch.empty((N, h), dtype=dt, device=dev),
                  dg=torch.empty(h, dtype=torch.float32, device=dev),
                  db=torch.empty(h, dtype=torch.float32, device=dev),
                  dc=torch.empty(h, dtype=torch.float32, device=dev))
    if w.norm != "layernorm":
        outs_d["db"] = None
    if bias is None:
        outs_d["dc"] = None
    outs_h = {k: (None if v is None else
                  torch.empty_like(v, device="cpu").pin_memory())
              for k, v in outs_d.items()}
    d2h = sum(v.numel() * v.element_size() for v in outs_h.values()
              if v is not None)
    ws = torch.empty(sp.sp_bwd_workspace_bytes(cfg, dev.index) // 4,
                     dtype=torch.float32, device=dev)
    comp = torch.cuda.current_stream(dev)
    up = torch.cuda.Stream(dev)
    down = torch.cuda.Stream(dev)

    def upload(i):
        """enqueue step i's input copies; returns the event that marks them"""
        dev_in = bufs[i % 2]
        with torch.cuda.stream(up):
            # the buffer set was last read by step i-2's compute
            if i >= 2:
                up.wait_event(done_compute[i - 2])
            for d_, h_ in zip(dev_in, ins):
                if h_ is not None:
                    d_.copy_(h_, non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(up)
        return ev

    def compute(i, uploaded):
        dev_in = bufs[i % 2]
        d_parts, d_b, d_g, d_be, d_r = (dev_in[:t], dev_in[t], dev_in[t + 1],
                                        dev_in[t + 2], dev_in[t + 3])
        d_dp = dev_in[t + 4:]
        comp.wait_event(uploaded)
        if i >= 1:
            comp.wait_event(done_download[i - 1])   # outputs are reused
        o = outs_d
        sp.sp_rs_bias_dropout_add_norm_fwd(cfg, d_parts, d_b, d_r, d_g, d_be,
                                           o["rout"], [o["out"]], o["mask"],
                                           o["mean"], o["rstd"], stream=comp)
        sp.sp_rs_norm_dropout_bwd(cfg, d_dp, None, o["rout"], d_g, o["mask"],
                                  o["mean"], o["rstd"], o["dres"], o["dY"],
                                  o["dg"], o["db"], o["dc"], ws, stream=comp)
        ev = torch.cuda.Event()
        ev.record(comp)
        done_compute[i] = ev

    def download(i):
        with torch.cuda.stream(down):
            down.wait_event(done_compute[i])
            for k, v in outs_d.items():
                if v is not None:
                    outs_h[k].copy_(v, non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(down)
            done_download[i] = ev

    def run(nsteps):
        uploaded = upload(0)
        for i in range(nsteps):
            nxt = upload(i + 1) if i + 1 < nsteps else None
            compute(i, uploaded)
            download(i)
            uploaded = nxt

    done_compute, done_download = {}, {}
    run(2)
    torch.cuda.synchronize(dev)
    K = args.e2e_steps
    done_compute, done_download = {}, {}
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(up)
    run(K)
    down.wait_event(done_download[K - 1])
    e1.record(down)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1), dev)
    return {"value": round(job_throughput(step_bytes, K, world, ms), 2),
            "unit": "GB/s", "ms_per_step": round(ms / K, 3), "steps": K,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "path": "every step: pinned host -> device copies of all inputs, "
                    "fwd + bwd through the C ABI, every output copied back "
                    "to pinned host; uploads, compute and downloads on three "
                    "streams, inputs double-buffered"}


# ----------------------------------------------------------------------------
# the CPU oracle (baseline leg and reference arm)
# ----------------------------------------------------------------------------

_DRAWN = {}


def _oracle_rows(w, row0, nrows, orc, sp_synth, cfg, reuse=False):
    """Oracle forward + backward on token rows [row0, row0 + nrows), inputs
    drawn on the host with the workload's recipe (rows seeded by row0).
    reuse=True draws one sample of nrows rows per process and runs it for
    every row0 (the oracle's work per row does not depend on the values);
    only the oracle's own time is returned either way."""
    key = (repr(w), nrows)
    if reuse and key in _DRAWN:
        parts, bias, gamma, beta, res, dparts = _DRAWN[key]
    else:
        ww = w.replace(seed=w.seed + 7919 * (row0 + 1))
        parts = sp_synth.draw_partials(ww, rows=nrows)
        bias, gamma, beta = sp_synth.draw_params(w)
        res = sp_synth.draw_residual(ww, rows=nrows)
        dparts = sp_synth.draw_grad_partials(ww, rows=nrows)
        if reuse:
            _DRAWN[key] = (parts, bias, gamma, beta, res, dparts)
    ids = list(range(row0, row0 + nrows))
    t0 = time.perf_counter()
    fo = orc.fwd_rows(cfg, ids, parts, bias, res, gamma, beta)
    orc.bwd_rows(cfg, dparts, None, fo["residual_out"], gamma, fo["mask"],
                 fo["mean"], fo["rstd"])
    return time.perf_counter() - t0


def _oracle_chunk(job):
    """One job of the all-cores baseline, in a spawned worker process: the
    oracle on rows [row0, row0 + nrows) of a workload (compute time)."""
    w, row0, nrows, reuse = job
    import torch
    torch.set_num_threads(1)   # one process per core
    import oracle as orc
    import sp_synth
    return _oracle_rows(w, row0, nrows, orc, sp_synth, orc.cfg_from(w), reuse)


def _host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline_all_cores(w, fb, bb, budget_s=10.0, max_procs=64):
    """The same oracle rows spread over one process per available core
    (spawned, never forked from a process that touched the GPU).  Throughput
    counts each batch at its slowest worker's compute time."""
    import multiprocessing as mp
    procs = max(1, min(_host_cores(), max_procs))
    per_row = (fb + bb) / w.rows
    chunk = 64
    rows_done, secs, row0 = 0, 0.0, 0
    with mp.get_context("spawn").Pool(procs) as pool:
        pool.map(_oracle_chunk, [(w, 0, 1, False)] * procs)   # imports, oracle load
        while secs < budget_s and row0 < w.rows:
            jobs = []
            while len(jobs) < procs and row0 < w.rows:
                n = min(chunk, w.rows - row0)
                jobs.append((w, row0, n, False))
                row0 += n
            secs += max(pool.map(_oracle_chunk, jobs))
            rows_done += sum(j[2] for j in jobs)
    return {"value": round(per_row * rows_done / secs / 1e9, 4), "unit": "GB/s",
            "cores": procs, "kind": "oracle",
            "sample": (f"{w.name} token rows 0..{rows_done - 1} of {w.rows} in batches of "
                       f"{procs} x {chunk} rows, one process per core, "
                       f"{secs:.1f} s of critical-path oracle time"),
            "tokens_per_s": round(rows_done / secs, 2)}


def cpu_baseline(w, fb, bb, budget_s=10.0):
    import oracle as orc
    import sp_synth
    orc.build()
    cfg = orc.cfg_from(w)
    per_row = (fb + bb) / w.rows
    rows_done, secs, row0 = 0, 0.0, 0
    chunk = 64
    while secs < budget_s and row0 < w.rows:
        n = min(chunk, w.rows - row0)
        secs += _oracle_rows(w, row0, n, orc, sp_synth, cfg)
        rows_done += n
        row0 += n
    return {"value": round(per_row * rows_done / secs / 1e9, 4),
            "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": (f"{w.name} token rows 0..{rows_done - 1} of {w.rows} "
                       f"(forward + backward per row, {secs:.1f} s of "
                       "single-threaded C oracle time)"),
            "tokens_per_s": round(rows_done / secs, 2),
            "all_cores": cpu_baseline_all_cores(w, fb, bb, budget_s)}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import oracle as orc
    import sp_synth
    orc.build()
    w = workload_of(args)
    cfg = orc.cfg_from(w)
    fb, bb = fwd_bytes(w), bwd_bytes(w)
    per_row = (fb + bb) / w.rows
    procs = max(1, min(args.reference_cores or _host_cores(), 64))
    # per-step sample sized so that warm-up + timed steps take ~2 minutes;
    # with several processes a step is one batch of rows on every process,
    # timed at its slowest worker
    t_row = _oracle_rows(w, 0, 8, orc, sp_synth, cfg) / 8
    per_proc = int(max(1, min(256, 120.0 / max(1, args.steps + args.warmup)
                              / max(t_row, 1e-6))))
    per_proc = min(per_proc, max(1, w.rows // procs))
    rows = per_proc * procs

    def step_jobs(i):
        base = (i * rows) % max(1, w.rows - rows + 1)
        return [(w, base + k * per_proc, per_proc, True) for k in range(procs)]

    secs = 0.0
    if procs == 1:
        for i in range(args.warmup + args.steps):
            (wj, r0, n, reuse), = step_jobs(i)
            t = _oracle_rows(wj, r0, n, orc, sp_synth, cfg, reuse)
            if i >= args.warmup:
                secs += t
    else:
        import multiprocessing as mp
        with mp.get_context("spawn").Pool(procs) as pool:
            for i in range(args.warmup + args.steps):
                t = max(pool.map(_oracle_chunk, step_jobs(i)))
                if i >= args.warmup:
                    secs += t
    value = per_row * rows * args.steps / secs / 1e9
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "io_dtype": w.dtype, "data": "synthetic",
        "impl": "reference",
        "config": {"workload": (f"{w.name}: SP boundary fwd+bwd, s={w.s} "
                                f"b={w.b} h={w.h} t={w.t}, {w.dtype} I/O, "
                                f"{w.norm}, p={w.p_drop}, bias"
                                + (", fp32 residual stream" if w.res != w.dtype
                                   else "")),
                   "s": w.s, "b": w.b, "h": w.h, "t": w.t,
                   "sample_rows_per_step": rows},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s",
                         "cores": procs, "kind": "oracle",
                         "sample": f"{rows} token rows of {w.name} per step "
                                   f"({per_proc} on each of {procs} processes), "
                                   "forward + backward"},
        "e2e": {"value": round(value, 4), "unit": "GB/s",
                "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "tokens_per_s": round(rows * args.steps / secs, 2),
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="C2")
    ap.add_argument("--op", default="boundary", choices=["boundary", "entry"],
                    help="boundary: the exit of a TP region (reduce-scatter "
                         "+ epilogue + all-gather); entry: norm + all-gather")
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--reference-cores", type=int, default=0,
                    help="processes for --impl reference (0: every core, up to 64)")
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--mode", default="replicas", choices=["replicas", "ranks"],
                    help="replicas: N independent copies of the boundary (weak "
                         "scaling); ranks: the boundary on t = N ranks over peer "
                         "memory, with NCCL all-reduce vs reduce-scatter + "
                         "all-gather beside it")
    ap.add_argument("--skip-linears", action="store_true",
                    help="skip timing the tensor-parallel linears and the ring "
                         "attention (N = 1)")
    ap.add_argument("--workloads", default="C2,C3,C4,C5",
                    help="after the timed steps, time the forward and backward "
                         "of these workloads one by one (N = 1; '' for none)")
    ap.add_argument("--residual-f32", action="store_true",
                    help="keep the residual stream in fp32 beside bf16 I/O")
    ap.add_argument("--fwd-plan", type=int, default=0,
                    help="forward kernel plan hint (0: library's choice)")
    ap.add_argument("--bwd-plan", type=int, default=0,
                    help="backward kernel plan hint (0: library's choice)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")
    if args.impl == "reference":
        run_reference(args)
    elif args.mode == "ranks":
        run_ranks(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
