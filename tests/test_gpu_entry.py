"""Entry into a tensor-parallel region: each rank normalises its own tokens,
then the all-gather forms the input of the QKV / first FFN projection ("SP:
Partition Activations Alongside TP", section "Connect SP and TP across a
layer").  sp_norm_all_gather_fwd against the oracle, as t emulated ranks, and
its backward (the reduce-scatter of the upstream gradients, then the norm
backward: sp_rs_norm_dropout_bwd with no dropout and no dY)."""
import numpy as np
import pytest
import torch

import oracle
import sp_synth
from sp_synth import WORKLOADS
from _parity import (Guarded, assert_close, assert_sum_close, cfg_of,
                     mag_norm_out, mags_backward)

import sp_region_b200 as sp

pytestmark = pytest.mark.gpu

CASES = {
    "ln_h6144_t8": dict(base="C2", s=160, b=2),
    "rms_h8192_t8": dict(base="C3", s=152, b=1),
    "ln_h12288_t16": dict(base="C5", s=160, b=1, outliers=0.0),
    "ln_general_h100": dict(base="C2", s=40, b=2, h=100, t=4),
    "f32_ln_h512": dict(base="C2", s=64, b=3, h=512, t=2, dtype="f32"),
    # vectors per row not a multiple of the threads' share: guarded tail
    "ln_h1000_ragged": dict(base="C2", s=64, b=2, h=1000, t=4),
    "f32_rms_h520_ragged": dict(base="C3", s=48, b=2, h=520, t=2, dtype="f32"),
    "ln_h2048_no_beta": dict(base="C2", s=64, b=2, h=2048, t=4, has_beta=False),
    # many rows per consumer group (the prefetch runs across every row)
    "ln_h6144_many_rows": dict(base="C2", s=1024, b=2),
    "rms_h4096_many_rows": dict(base="C3", s=4096, b=1, h=4096, t=4),
    # one-warp consumer groups
    "ln_h1024_t2": dict(base="C2", s=512, b=1, h=1024, t=2),
}


def _w(name):
    spec = dict(CASES[name])
    return WORKLOADS[spec.pop("base")].replace(**spec)


def _params(w):
    bias, gamma, beta = sp_synth.draw_params(w)
    return gamma, (beta if w.norm == "layernorm" and w.has_beta else None)


@pytest.fixture(scope="module", autouse=True)
def _needs_gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    oracle.build()


@pytest.mark.parametrize("plan", [0, 14])
@pytest.mark.parametrize("name", sorted(CASES))
def test_entry_forward_matches_oracle(name, plan):
    """plan 0: the register-streaming entry kernel (or the general kernel for
    h not a multiple of 8); plan 14: the staged-ring forward kernel run with
    no partial sums, where the shape fits it."""
    w = _w(name)
    x = sp_synth.draw_residual(w)
    gamma, beta = _params(w)
    ref = oracle.norm_ag_fwd(oracle.cfg_from(w), x, gamma, beta, n_out=1)
    N, h = w.rows, w.h
    outs = [Guarded((N, h), w.torch_dtype) for _ in range(2)]
    mean = Guarded((N,), torch.float32)
    rstd = Guarded((N,), torch.float32)
    sp.sp_norm_all_gather_fwd(cfg_of(w, fwd_plan=plan), x.cuda(), gamma.cuda(),
                              None if beta is None else beta.cuda(),
                              [o.t for o in outs], mean.t, rstd.t)
    torch.cuda.synchronize()
    assert sp.sp_device_error() == 0
    for g in (*outs, mean, rstd):
        assert g.intact()
    mag = mag_norm_out(w, x, ref["mean"], ref["rstd"], gamma, beta)
    for o in outs:
        assert_close("gathered", o.t.cpu(), ref["gathered"][0], mag,
                     w.torch_dtype)
    assert np.allclose(rstd.t.cpu().numpy(), ref["rstd"], rtol=1e-5)
    if w.norm == "layernorm":
        rms = x.double().pow(2).mean(1).sqrt().numpy()
        assert (np.abs(mean.t.cpu().numpy() - ref["mean"]) <= 1e-5 * rms).all()


@pytest.mark.parametrize("name", ["ln_h6144_t8", "ln_general_h100", "rms_h4096_many_rows",
                                  "ln_h1000_ragged"])
def test_entry_as_ranks(name):
    """t row-range calls, each normalising its own shard and pushing into
    every rank's gathered buffer, reproduce the whole call bit for bit."""
    w = _w(name)
    N, h, t = w.rows, w.h, w.t
    per = N // t
    x = sp_synth.draw_residual(w).cuda()
    gamma, beta = _params(w)
    gamma = gamma.cuda()
    beta = None if beta is None else beta.cuda()
    whole = torch.empty((N, h), dtype=w.torch_dtype, device="cuda")
    sp.sp_norm_all_gather_fwd(cfg_of(w), x, gamma, beta, [whole])
    reps = [torch.full((N, h), float("nan"), dtype=w.torch_dtype,
                       device="cuda") for _ in range(t)]
    for r in range(t):
        c = sp.make_cfg(w.s, w.b, h, t, dtype=w.dtype, norm=w.norm, eps=w.eps,
                        row_begin=r * per, row_end=(r + 1) * per)
        sp.sp_norm_all_gather_fwd(c, x[r * per:(r + 1) * per], gamma, beta,
                                  reps)
    torch.cuda.synchronize()
    assert sp.sp_device_error() == 0
    for rep in reps:
        assert torch.equal(rep.view(torch.int16), whole.view(torch.int16))


@pytest.mark.parametrize("name", ["ln_h6144_t8", "rms_h8192_t8",
                                  "ln_general_h100", "f32_ln_h512"])
def test_entry_backward_matches_oracle(name):
    """Backward of the entry: reduce-scatter of the upstream gradient partials
    and the norm backward, with a gradient arriving on the residual stream;
    no dropout, no gradient toward partial sums."""
    w = _w(name).replace(p_drop=0.0)
    x = sp_synth.draw_residual(w)
    gamma, beta = _params(w)
    cfg = oracle.cfg_from(w)
    fo = oracle.norm_ag_fwd(cfg, x, gamma, beta)
    dparts = sp_synth.draw_grad_partials(w)
    drn = sp_synth.draw_residual_grad(w)
    ln = w.norm == "layernorm"
    rb = oracle.bwd(cfg, dparts, drn, x, gamma, None, fo["mean"], fo["rstd"],
                    with_dbeta=ln, with_dbias=False)
    N, h = w.rows, w.h
    dt = w.torch_dtype
    d = lambda v: v.cuda()
    dres = Guarded((N, h), dt)
    dg = Guarded((h,), torch.float32)
    db = Guarded((h,), torch.float32) if ln else None
    mean = (torch.from_numpy(fo["mean"].astype(np.float32)).cuda() if ln
            else None)
    rstd = torch.from_numpy(fo["rstd"].astype(np.float32)).cuda()
    c = cfg_of(w)
    ws = torch.empty(sp.sp_bwd_workspace_bytes(c) // 4, dtype=torch.float32,
                     device="cuda")
    sp.sp_rs_norm_dropout_bwd(c, [d(p) for p in dparts], d(drn), d(x),
                              d(gamma), None, mean, rstd, dres.t, None, dg.t,
                              None if db is None else db.t, None, ws)
    torch.cuda.synchronize()
    assert sp.sp_device_error() == 0
    for g in (dres, dg, db):
        if g is not None:
            assert g.intact()
    m = mags_backward(w, dparts, drn, x, gamma, fo["mean"], fo["rstd"])
    assert_close("dresidual_in", dres.t.cpu(), rb["dresidual_in"], m["dres"],
                 dt)
    assert_sum_close("dgamma", dg.t.cpu().numpy(), rb["dgamma"],
                     m["dgamma_terms"])
    if ln:
        assert_sum_close("dbeta", db.t.cpu().numpy(), rb["dbeta"],
                         m["dbeta_terms"])
