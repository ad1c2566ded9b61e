"""An fp32 residual stream beside bf16 partial sums, parameters and norm
outputs (sp_cfg.res_f32): residual, the stored sum, the entry's x, dR_next
and the residual gradient are fp32.  Every kernel family against the oracle:
the staged-ring kernels (exact and guarded tiling), the 2-CTA cluster split,
the general kernels, and the entry; plus t emulated ranks bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import sp_synth
from sp_synth import WORKLOADS
from _parity import (Guarded, assert_close, assert_sum_close, cfg_of,
                     check_forward, gpu_bwd, gpu_fwd, mag_norm_out,
                     mags_backward)

import sp_region_b200 as sp

pytestmark = pytest.mark.gpu

CASES = {
    # staged ring, threads tile the row exactly
    "ln_h6144_t8": dict(base="C2", s=160, b=2),
    # staged ring, guarded tail (1024 vectors over 3-vector threads)
    "rms_h8192_t8": dict(base="C3", s=128, b=1, p_drop=0.1, has_bias=True),
    # the 4-vector 544-thread plan is compiled without the fp32 residual:
    # the host picks another
    "ln_h4096_t4": dict(base="C4", s=224, b=2),
    "ln_h12288_t16": dict(base="C5", s=96, b=1, outliers=0.0),
    # rows split across a 2-CTA cluster (forward); general backward
    "ln_h24576_cluster": dict(base="C2", s=48, b=1, h=24576, t=2),
    # h not a multiple of 8: general kernels
    "ln_general_h100": dict(base="C2", s=40, b=2, h=100, t=4),
}


def _w(name):
    spec = dict(CASES[name])
    return WORKLOADS[spec.pop("base")].replace(res_dtype="f32", **spec)


def _inputs(w):
    parts = sp_synth.draw_partials(w)
    bias, gamma, beta = sp_synth.draw_params(w)
    if not w.has_bias:
        bias = None
    if not w.has_beta or w.norm == "rmsnorm":
        beta = None
    return parts, bias, sp_synth.draw_residual(w), gamma, beta


@pytest.fixture(scope="module", autouse=True)
def _needs_gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    oracle.build()


@pytest.mark.parametrize("offset", [0, 1])
@pytest.mark.parametrize("name", sorted(CASES))
def test_forward_and_backward_match_oracle(name, offset):
    """offset 1 shifts every [s,b,h] buffer off its 16-byte boundary (general
    kernels)."""
    w = _w(name)
    parts, bias, res, gamma, beta = _inputs(w)
    assert res.dtype == torch.float32 and parts[0].dtype == torch.bfloat16
    cfg = oracle.cfg_from(w)
    ref = oracle.fwd(cfg, parts, bias, res, gamma, beta)
    got = gpu_fwd(w, parts, bias, res, gamma, beta, offset_elems=offset)
    assert got["residual_out"].dtype == torch.float32
    check_forward(w, got, ref, parts, bias, res, gamma, beta)

    dparts = sp_synth.draw_grad_partials(w)
    drn = sp_synth.draw_residual_grad(w)
    want_dbeta = w.norm == "layernorm"
    rb = oracle.bwd(cfg, dparts, drn, ref["residual_out"], gamma, ref["mask"],
                    ref["mean"], ref["rstd"], with_dbeta=want_dbeta,
                    with_dbias=bias is not None)
    gb = gpu_bwd(w, dparts, drn, ref["residual_out"], gamma, ref["mask"],
                 ref["mean"], ref["rstd"], with_dbeta=want_dbeta,
                 with_dbias=bias is not None, offset_elems=offset)
    m = mags_backward(w, dparts, drn, ref["residual_out"], gamma, ref["mean"],
                      ref["rstd"])
    assert gb["dresidual_in"].dtype == torch.float32
    assert_close("dresidual_in", gb["dresidual_in"], rb["dresidual_in"],
                 m["dres"], torch.float32)
    assert_close("dY", gb["dY"], rb["dY"], m["dY"], torch.bfloat16)
    assert_sum_close("dgamma", gb["dgamma"], rb["dgamma"], m["dgamma_terms"])
    if want_dbeta:
        assert_sum_close("dbeta", gb["dbeta"], rb["dbeta"], m["dbeta_terms"])
    if bias is not None:
        assert_sum_close("dbias", gb["dbias"], rb["dbias"], m["dbias_terms"])


@pytest.mark.parametrize("plan", [0, 14])
@pytest.mark.parametrize("name", ["ln_h6144_t8", "rms_h8192_t8", "ln_general_h100"])
def test_entry_normalises_an_fp32_stream(name, plan):
    w = _w(name).replace(p_drop=0.0)
    x = sp_synth.draw_residual(w)
    bias, gamma, beta = sp_synth.draw_params(w)
    beta = beta if w.norm == "layernorm" and w.has_beta else None
    ref = oracle.norm_ag_fwd(oracle.cfg_from(w), x, gamma, beta)
    N, h = w.rows, w.h
    out = Guarded((N, h), torch.bfloat16)
    mean = Guarded((N,), torch.float32)
    rstd = Guarded((N,), torch.float32)
    sp.sp_norm_all_gather_fwd(cfg_of(w, fwd_plan=plan), x.cuda(), gamma.cuda(),
                              None if beta is None else beta.cuda(), [out.t],
                              mean.t, rstd.t)
    torch.cuda.synchronize()
    assert sp.sp_device_error() == 0
    for g in (out, mean, rstd):
        assert g.intact()
    mag = mag_norm_out(w, x, ref["mean"], ref["rstd"], gamma, beta)
    assert_close("gathered", out.t.cpu(), ref["gathered"][0], mag, torch.bfloat16)
    assert np.allclose(rstd.t.cpu().numpy(), ref["rstd"], rtol=1e-5)


def test_ranks_reproduce_the_whole_call():
    """t row-range calls give the whole call's bits, forward and backward."""
    w = _w("ln_h6144_t8")
    N, h, t = w.rows, w.h, w.t
    per = N // t
    parts, bias, res, gamma, beta = (None if x is None else
                                     (x.cuda() if torch.is_tensor(x) else
                                      [p.cuda() for p in x])
                                     for x in _inputs(w))
    mk = lambda r0=0, r1=0: sp.make_cfg(w.s, w.b, h, t, dtype=w.dtype,
                                        norm=w.norm, eps=w.eps, p_drop=w.p_drop,
                                        seed=w.drop_seed, offset=w.drop_offset,
                                        row_begin=r0, row_end=r1, res_f32=True)
    f32, bf = torch.float32, torch.bfloat16
    W = (h + 31) // 32
    rout = torch.empty(N, h, dtype=f32, device="cuda")
    gat = torch.empty(N, h, dtype=bf, device="cuda")
    mask = torch.empty(N, W, dtype=torch.int32, device="cuda")
    mean = torch.empty(N, device="cuda")
    rstd = torch.empty(N, device="cuda")
    sp.sp_rs_bias_dropout_add_norm_fwd(mk(), parts, bias, res, gamma, beta, rout,
                                       [gat], mask, mean, rstd)
    rout_r = torch.empty_like(rout)
    gat_r = torch.full_like(gat, float("nan"))
    for r in range(t):
        sl = slice(r * per, (r + 1) * per)
        sp.sp_rs_bias_dropout_add_norm_fwd(mk(r * per, (r + 1) * per), parts, bias,
                                           res[sl], gamma, beta, rout_r[sl], [gat_r],
                                           mask[sl], mean[sl], rstd[sl])
    torch.cuda.synchronize()
    assert sp.sp_device_error() == 0
    assert torch.equal(rout_r.view(torch.int32), rout.view(torch.int32))
    assert torch.equal(gat_r.view(torch.int16), gat.view(torch.int16))

    dparts = [d.cuda() for d in sp_synth.draw_grad_partials(w)]
    drn = sp_synth.draw_residual_grad(w).cuda()
    ws = torch.empty(sp.sp_bwd_workspace_bytes(mk()) // 4, device="cuda")
    g3 = lambda: [torch.empty(h, device="cuda") for _ in range(3)]
    dres = torch.empty(N, h, dtype=f32, device="cuda")
    dY = torch.empty(N, h, dtype=bf, device="cuda")
    sp.sp_rs_norm_dropout_bwd(mk(), dparts, drn, rout, gamma, mask, mean, rstd,
                              dres, dY, *g3(), ws)
    dres_r = torch.empty_like(dres)
    dY_r = torch.full_like(dY, float("nan"))
    for r in range(t):
        sl = slice(r * per, (r + 1) * per)
        sp.sp_rs_norm_dropout_bwd(mk(r * per, (r + 1) * per), dparts, drn[sl],
                                  rout[sl], gamma, mask[sl], mean[sl], rstd[sl],
                                  dres_r[sl], dY_r, *g3(), ws)
        torch.cuda.synchronize()
    assert sp.sp_device_error() == 0
    assert torch.equal(dres_r.view(torch.int32), dres.view(torch.int32))
    assert torch.equal(dY_r.view(torch.int16), dY.view(torch.int16))
