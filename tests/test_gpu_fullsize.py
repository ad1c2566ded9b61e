"""The five workloads at full size, in the launch configuration the benchmark
times (one forward call with the all-gather fused into the output write, one
backward call), compared with the CPU oracle.

C2, C3 and C4 are compared element by element against the whole oracle run;
the backward's inputs (stored residual sum, mask, statistics) are the
oracle's own forward outputs, so no oracle input comes from the CUDA path.
C5 (6.4 G partial elements) is compared on sampled token rows -- the first and
last rows, both sides of every rank boundary and random rows -- and through
properties that hold at any size.
"""
import gc
import math

import numpy as np
import pytest
import torch

import oracle
import sp_synth
from sp_synth import WORKLOADS
from _parity import (assert_close, assert_sum_close, check_forward,
                     gpu_bwd, mag_norm_out,
                     mag_residual_out, mags_backward, cfg_of)

import sp_region_b200 as sp

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    oracle.build()
    yield
    gc.collect()
    torch.cuda.empty_cache()


def _params(w, device):
    bias, gamma, beta = sp_synth.draw_params(w, device)
    if not w.has_bias:
        bias = None
    if not w.has_beta or w.norm == "rmsnorm":
        beta = None
    return bias, gamma, beta


def _device_fwd(w, parts_d, bias_d, res_d, gamma_d, beta_d, n_gathered=1):
    N, h = w.rows, w.h
    dt = w.torch_dtype
    rout = torch.empty((N, h), dtype=dt, device="cuda")
    gath = [torch.empty((N, h), dtype=dt, device="cuda")
            for _ in range(n_gathered)]
    mask = torch.empty((N, (h + 31) // 32), dtype=torch.int32, device="cuda")
    mean = torch.empty(N, dtype=torch.float32, device="cuda")
    rstd = torch.empty(N, dtype=torch.float32, device="cuda")
    sp.sp_rs_bias_dropout_add_norm_fwd(cfg_of(w), parts_d, bias_d, res_d,
                                       gamma_d, beta_d, rout, gath, mask,
                                       mean, rstd)
    torch.cuda.synchronize()
    assert sp.sp_device_error() == 0
    return rout, gath, mask, mean, rstd


def _check_full_fwd(w, n_gathered=1):
    parts = sp_synth.draw_partials(w)
    bias, gamma, beta = _params(w, "cpu")
    res = sp_synth.draw_residual(w)
    d = lambda x: None if x is None else x.cuda()
    rout, gath, mask, mean, rstd = _device_fwd(
        w, [p.cuda() for p in parts], d(bias), d(res), d(gamma), d(beta),
        n_gathered)
    ref = oracle.fwd(oracle.cfg_from(w), parts, bias, res, gamma, beta)
    got = dict(residual_out=rout.cpu(), gathered=[g.cpu() for g in gath],
               mask=mask.cpu().numpy().view(np.uint32),
               mean=mean.cpu().numpy(), rstd=rstd.cpu().numpy())
    check_forward(w, got, ref, parts, bias, res, gamma, beta, n_gathered)
    return parts, bias, res, gamma, beta, ref


def test_c2_forward_and_backward_full():
    """C2 (s=2048, b=4, h=6144, t=8, LayerNorm, p=0.1): the benchmark's
    workload, forward and backward, every element."""
    w = WORKLOADS["C2"]
    parts, bias, res, gamma, beta, ref = _check_full_fwd(w)
    del parts
    gc.collect()
    dparts = sp_synth.draw_grad_partials(w)
    cfg = oracle.cfg_from(w)
    rb = oracle.bwd(cfg, dparts, None, ref["residual_out"], gamma, ref["mask"],
                    ref["mean"], ref["rstd"])
    got = gpu_bwd(w, dparts, None, ref["residual_out"], gamma, ref["mask"],
                  ref["mean"], ref["rstd"])
    m = mags_backward(w, dparts, None, ref["residual_out"], gamma, ref["mean"],
                      ref["rstd"])
    dt = w.torch_dtype
    assert_close("dresidual_in", got["dresidual_in"], rb["dresidual_in"],
                 m["dres"], dt)
    assert_close("dY", got["dY"], rb["dY"], m["dY"], dt)
    assert_sum_close("dgamma", got["dgamma"], rb["dgamma"], m["dgamma_terms"])
    assert_sum_close("dbeta", got["dbeta"], rb["dbeta"], m["dbeta_terms"])
    assert_sum_close("dbias", got["dbias"], rb["dbias"], m["dbias_terms"])


def test_c3_rmsnorm_forward_with_replicas_full():
    """C3 (s=4096, h=8192, t=8, RMSNorm, p=0): forward plus the all-gather
    written as t per-rank replicas, every element of every replica."""
    _check_full_fwd(WORKLOADS["C3"], n_gathered=WORKLOADS["C3"].t)


def test_c3_standalone_all_gather_full():
    w = WORKLOADS["C3"]
    rows = w.rows // w.t
    x = sp_synth.draw_residual(w, "cuda")
    shards = [x[r * rows:(r + 1) * rows] for r in range(w.t)]
    outs = [torch.empty_like(x) for _ in range(w.t)]
    sp.sp_all_gather(cfg_of(w), shards, outs)
    torch.cuda.synchronize()
    for o in outs:
        assert torch.equal(o.view(torch.int16), x.view(torch.int16))


def test_c4_backward_full():
    """C4 (s=8192, b=2, h=4096, t=4): the producing forward, then the fused
    backward fed with the oracle's forward outputs; every element and the
    parameter gradients."""
    w = WORKLOADS["C4"]
    parts, bias, res, gamma, beta, ref = _check_full_fwd(w)
    del parts
    gc.collect()
    dparts = sp_synth.draw_grad_partials(w)
    cfg = oracle.cfg_from(w)
    rb = oracle.bwd(cfg, dparts, None, ref["residual_out"], gamma, ref["mask"],
                    ref["mean"], ref["rstd"])
    got = gpu_bwd(w, dparts, None, ref["residual_out"], gamma, ref["mask"],
                  ref["mean"], ref["rstd"])
    m = mags_backward(w, dparts, None, ref["residual_out"], gamma, ref["mean"],
                      ref["rstd"])
    dt = w.torch_dtype
    assert_close("dresidual_in", got["dresidual_in"], rb["dresidual_in"],
                 m["dres"], dt)
    assert_close("dY", got["dY"], rb["dY"], m["dY"], dt)
    assert_sum_close("dgamma", got["dgamma"], rb["dgamma"], m["dgamma_terms"])
    assert_sum_close("dbeta", got["dbeta"], rb["dbeta"], m["dbeta_terms"])
    assert_sum_close("dbias", got["dbias"], rb["dbias"], m["dbias_terms"])


def _sample_rows(N, t, seed, extra=24):
    per = N // t
    rows = {0, 1, N - 1}
    for r in range(1, t):
        rows.update((r * per - 1, r * per))
    rng = np.random.default_rng(seed)
    rows.update(int(x) for x in rng.integers(0, N, size=extra))
    return sorted(rows)


def test_c5_long_sequence_forward_backward_sampled():
    """C5 (s=32768, h=12288, t=16, 1 % x100 outliers): forward and backward
    on the device at full size; sampled rows against the oracle; the keep
    rate over all 402 M mask bits; dbeta against a float64 sum of the
    upstream partials; activation bytes with a = 96."""
    w = WORKLOADS["C5"]
    N, h, t = w.rows, w.h, w.t
    parts_d = sp_synth.draw_partials(w, "cuda")
    bias_d, gamma_d, beta_d = _params(w, "cuda")
    res_d = sp_synth.draw_residual(w, "cuda")
    rout, gath, mask, mean, rstd = _device_fwd(w, parts_d, bias_d, res_d,
                                               gamma_d, beta_d)
    rows = _sample_rows(N, t, seed=55)
    idx = torch.tensor(rows, device="cuda")
    cfg = oracle.cfg_from(w)
    prow = [p[idx].cpu() for p in parts_d]
    bias, gamma, beta = bias_d.cpu(), gamma_d.cpu(), beta_d.cpu()
    rrow = res_d[idx].cpu()
    ref = oracle.fwd_rows(cfg, rows, prow, bias, rrow, gamma, beta)
    dt = w.torch_dtype
    got = dict(residual_out=rout[idx].cpu(), norm_out=gath[0][idx].cpu(),
               mask=mask[idx].cpu().numpy().view(np.uint32),
               mean=mean[idx].cpu().numpy(), rstd=rstd[idx].cpu().numpy())
    check_forward(w, got, ref, prow, bias, rrow, gamma, beta)
    # keep rate over the whole mask, within 6 sigma of the binomial
    kept = int(torch.bitwise_count(mask.view(torch.int32)).sum().item()) \
        if hasattr(torch, "bitwise_count") else int(
            np.unpackbits(mask.cpu().numpy().view(np.uint8)).sum())
    n = N * h
    p = float(np.float32(w.p_drop))
    assert abs(kept - n * (1 - p)) < 6 * math.sqrt(n * p * (1 - p))
    del parts_d, gath
    gc.collect()
    torch.cuda.empty_cache()

    # backward on the device, from the device forward's outputs
    dparts_d = sp_synth.draw_grad_partials(w, "cuda")
    dres = torch.empty((N, h), dtype=dt, device="cuda")
    dY = torch.empty((N, h), dtype=dt, device="cuda")
    dg = torch.empty(h, dtype=torch.float32, device="cuda")
    db = torch.empty(h, dtype=torch.float32, device="cuda")
    dc = torch.empty(h, dtype=torch.float32, device="cuda")
    c = cfg_of(w)
    ws = torch.empty(sp.sp_bwd_workspace_bytes(c) // 4, dtype=torch.float32,
                     device="cuda")
    sp.sp_rs_norm_dropout_bwd(c, dparts_d, None, rout, gamma_d, mask, mean,
                              rstd, dres, dY, dg, db, dc, ws)
    torch.cuda.synchronize()
    assert sp.sp_device_error() == 0
    # sampled rows: the oracle's backward from the oracle's own forward rows
    drow = [d_[idx].cpu() for d_ in dparts_d]
    rb = oracle.bwd_rows(cfg, drow, None, ref["residual_out"], gamma,
                         ref["mask"], ref["mean"], ref["rstd"])
    wr = w.replace(s=len(rows), b=1, t=1)
    m = mags_backward(wr, drow, None, ref["residual_out"], gamma, ref["mean"],
                      ref["rstd"])
    assert_close("dresidual_in rows", dres[idx].cpu(), rb["dresidual_in"],
                 m["dres"], dt)
    assert_close("dY rows", dY[idx].cpu(), rb["dY"], m["dY"], dt)
    # dbeta is the sum over all tokens of the reduced upstream gradient
    dn64 = torch.zeros(h, dtype=torch.float64, device="cuda")
    absn = torch.zeros(h, dtype=torch.float64, device="cuda")
    for r0 in range(0, N, 4096):
        blk = sum(d_[r0:r0 + 4096].double() for d_ in dparts_d)
        dn64 += blk.sum(0)
        absn += blk.abs().sum(0)
    assert_sum_close("dbeta (all tokens)", db.cpu().numpy(),
                     dn64.cpu().numpy(), absn.cpu().numpy())
    # activation memory of this layer shape with a = 96 heads
    sbh = N * h
    assert sp.sp_activation_bytes(w.s, w.b, h, w.heads, t, 0, 1.0) == \
        1314 * sbh
    assert sp.sp_activation_bytes(w.s, w.b, h, w.heads, t, 2, 1.0) == \
        82.125 * sbh
