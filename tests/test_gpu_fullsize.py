"""The five workloads at full size, in the launch configuration the benchmark
times (one forward call with the all-gather fused into the output write, one
backward call), compared with the CPU oracle element by element.

The backward's inputs (stored residual sum, mask, statistics) are the
oracle's own forward outputs, so no oracle input comes from the CUDA path.
Every forward is also checked through its norm step alone: the fused kernel
fed the oracle's stored sums must give the oracle's norm output within one
I/O ulp plus the fp32 term.  C5 (6.4 G partial elements, s = 32768, h =
12288, t = 16) is compared on all 32768 rows too, its oracle runs chunk by
chunk on every host core, and its parameter gradients are the sum of the
oracle's row-chunk shares.
"""
import concurrent.futures
import os
import gc
import math

import numpy as np
import pytest
import torch

import oracle
import sp_synth
from sp_synth import WORKLOADS
from _parity import (assert_close, assert_sum_close, check_forward,
                     check_norm_step, gpu_bwd, gpu_norm_step, mags_backward,
                     cfg_of)

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
    _check_norm_step_full(w, ref["residual_out"], ref["gathered"][0],
                          ref["mean"], ref["rstd"], gamma, beta)
    return parts, bias, res, gamma, beta, ref


def _check_norm_step_full(w, x_ref, out_ref, mean_ref, rstd_ref, gamma, beta,
                          chunk=None):
    """The fused forward's norm step on the oracle's stored sums (all rows)."""
    d = lambda x: None if x is None else x.cuda()
    rout, out, mean, rstd = gpu_norm_step(w, d(x_ref), d(gamma), d(beta))
    N = x_ref.shape[0]
    chunk = chunk or N
    for r0 in range(0, N, chunk):
        r1 = min(N, r0 + chunk)
        got = dict(residual_out=rout[r0:r1].cpu(), norm_out=out[r0:r1].cpu(),
                   mean=mean[r0:r1].cpu().numpy(),
                   rstd=rstd[r0:r1].cpu().numpy())
        check_norm_step(w, got, x_ref[r0:r1], out_ref[r0:r1],
                        None if mean_ref is None else mean_ref[r0:r1],
                        rstd_ref[r0:r1], gamma, beta)


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


def _host_pool():
    """Threads for the chunked oracle: its C calls release the GIL."""
    return concurrent.futures.ThreadPoolExecutor(
        max_workers=max(1, min(16, os.cpu_count() or 1)))


def test_c5_long_sequence_forward_backward_full():
    """C5 (s=32768, h=12288, t=16, 1 % x100 outliers): forward and backward
    on the device at full size; every row against the oracle, the keep rate
    over all 402 M mask bits, dgamma / dbeta / dbias against the sum of the
    oracle's row-chunk shares, and the activation bytes with a = 96."""
    w = WORKLOADS["C5"]
    N, h, t = w.rows, w.h, w.t
    parts_d = sp_synth.draw_partials(w, "cuda")
    bias_d, gamma_d, beta_d = _params(w, "cuda")
    res_d = sp_synth.draw_residual(w, "cuda")
    rout, gath, mask, mean, rstd = _device_fwd(w, parts_d, bias_d, res_d,
                                               gamma_d, beta_d)
    cfg = oracle.cfg_from(w)
    oracle.mask_words(h)   # loads the oracle library before the threads start
    bias, gamma, beta = bias_d.cpu(), gamma_d.cpu(), beta_d.cpu()
    CH = 512
    spans = [(r0, min(N, r0 + CH)) for r0 in range(0, N, CH)]

    def fwd_chunk(span):
        r0, r1 = span
        prow = [p[r0:r1].cpu() for p in parts_d]
        rrow = res_d[r0:r1].cpu()
        ref = oracle.fwd_rows(cfg, list(range(r0, r1)), prow, bias, rrow,
                              gamma, beta)
        got = dict(residual_out=rout[r0:r1].cpu(),
                   norm_out=gath[0][r0:r1].cpu(),
                   mask=mask[r0:r1].cpu().numpy().view(np.uint32),
                   mean=mean[r0:r1].cpu().numpy(),
                   rstd=rstd[r0:r1].cpu().numpy())
        check_forward(w, got, ref, prow, bias, rrow, gamma, beta)
        return ref

    with _host_pool() as ex:
        refs = list(ex.map(fwd_chunk, spans))
    x_ref = torch.cat([r["residual_out"] for r in refs])
    out_ref = torch.cat([r["norm_out"] for r in refs])
    mask_ref = np.concatenate([r["mask"] for r in refs])
    mean_ref = np.concatenate([r["mean"] for r in refs])
    rstd_ref = np.concatenate([r["rstd"] for r in refs])
    del refs
    # keep rate over the whole mask, within 6 sigma of the binomial
    kept = int(np.unpackbits(mask_ref.view(np.uint8)).sum())
    n = N * h
    p = float(np.float32(w.p_drop))
    assert abs(kept - n * (1 - p)) < 6 * math.sqrt(n * p * (1 - p))
    del parts_d, gath, rout, mask, mean, rstd
    gc.collect()
    torch.cuda.empty_cache()
    _check_norm_step_full(w, x_ref, out_ref, mean_ref, rstd_ref, gamma, beta,
                          chunk=4096)
    del out_ref
    gc.collect()
    torch.cuda.empty_cache()

    # backward on the device, fed the oracle's forward outputs
    dparts_d = sp_synth.draw_grad_partials(w, "cuda")
    dt = w.torch_dtype
    x_d = x_ref.cuda()
    mask_d = torch.from_numpy(mask_ref.view(np.int32)).cuda()
    mean_d = torch.from_numpy(mean_ref.astype(np.float32)).cuda()
    rstd_d = torch.from_numpy(rstd_ref.astype(np.float32)).cuda()
    dres = torch.empty((N, h), dtype=dt, device="cuda")
    dY = torch.empty((N, h), dtype=dt, device="cuda")
    dg = torch.empty(h, dtype=torch.float32, device="cuda")
    db = torch.empty(h, dtype=torch.float32, device="cuda")
    dc = torch.empty(h, dtype=torch.float32, device="cuda")
    c = cfg_of(w)
    ws = torch.empty(sp.sp_bwd_workspace_bytes(c) // 4, dtype=torch.float32,
                     device="cuda")
    sp.sp_rs_norm_dropout_bwd(c, dparts_d, None, x_d, gamma_d, mask_d, mean_d,
                              rstd_d, dres, dY, dg, db, dc, ws)
    torch.cuda.synchronize()
    assert sp.sp_device_error() == 0

    def bwd_chunk(span):
        r0, r1 = span
        drow = [d_[r0:r1].cpu() for d_ in dparts_d]
        xr, mr = x_ref[r0:r1], mask_ref[r0:r1]
        mu, rs = mean_ref[r0:r1], rstd_ref[r0:r1]
        rb = oracle.bwd_rows(cfg, drow, None, xr, gamma, mr, mu, rs,
                             with_params=True)
        wr = w.replace(s=r1 - r0, b=1, t=1)
        m = mags_backward(wr, drow, None, xr, gamma, mu, rs)
        assert_close(f"dresidual_in rows {r0}..{r1}", dres[r0:r1].cpu(),
                     rb["dresidual_in"], m["dres"], dt)
        assert_close(f"dY rows {r0}..{r1}", dY[r0:r1].cpu(), rb["dY"],
                     m["dY"], dt)
        return ({k: rb[k] for k in ("dgamma", "dbeta", "dbias")},
                {k: m[k + "_terms"] for k in ("dgamma", "dbeta", "dbias")})

    with _host_pool() as ex:
        shares = list(ex.map(bwd_chunk, spans))
    for k, got in (("dgamma", dg), ("dbeta", db), ("dbias", dc)):
        ref = np.zeros(h)
        terms = np.zeros(h)
        for sh, tm in shares:          # the chunks' shares, in row order
            ref += sh[k]
            terms += tm[k]
        assert_sum_close(f"{k} (all tokens)", got.cpu().numpy(), ref, terms)
    # activation memory of this layer shape with a = 96 heads
    sbh = N * h
    assert sp.sp_activation_bytes(w.s, w.b, h, w.heads, t, 0, 1.0) == \
        1314 * sbh
    assert sp.sp_activation_bytes(w.s, w.b, h, w.heads, t, 2, 1.0) == \
        82.125 * sbh
