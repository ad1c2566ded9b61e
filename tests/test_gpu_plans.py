"""Every fast-kernel plan (vectors per thread, consumer groups per CTA, block
size) against the oracle.  The library takes a plan hint in sp_cfg; a hint
that does not fit a shape falls back to the automatic choice, so sweeping all
hints over several shapes runs every plan on at least one shape.  Row counts
give each consumer group several rows per CTA, so the sub-ring hand-off
between the producer and the groups is exercised in steady state."""
import functools

import numpy as np
import pytest
import torch

import oracle
import sp_synth
from sp_synth import WORKLOADS
from _parity import (assert_close, assert_sum_close, check_forward, gpu_bwd,
                     gpu_fwd, mags_backward)

import sp_region_b200 as sp

pytestmark = pytest.mark.gpu

SHAPES = {
    "h1024_t4": dict(base="C4", s=448, b=2, h=1024, t=4),
    "h6144_t8": dict(base="C2", s=232, b=4, h=6144, t=8),
    "h12288_t16": dict(base="C5", s=608, b=1, h=12288, t=16),
    "h8192_rms_t8": dict(base="C3", s=640, b=1, h=8192, t=8, p_drop=0.1,
                         has_bias=True),
    # wider than any one-CTA plan: the forward splits rows across a cluster
    "h24576_t2": dict(base="C2", s=320, b=1, h=24576, t=2),
}


def _workload(name):
    spec = dict(SHAPES[name])
    return WORKLOADS[spec.pop("base")].replace(**spec)


@functools.lru_cache(maxsize=None)
def _case(name):
    w = _workload(name)
    parts = sp_synth.draw_partials(w)
    bias, gamma, beta = sp_synth.draw_params(w)
    if not w.has_bias:
        bias = None
    if not w.has_beta or w.norm == "rmsnorm":
        beta = None
    res = sp_synth.draw_residual(w)
    cfg = oracle.cfg_from(w)
    ref = oracle.fwd(cfg, parts, bias, res, gamma, beta)
    dparts = sp_synth.draw_grad_partials(w)
    want_dbeta = w.norm == "layernorm"
    rb = oracle.bwd(cfg, dparts, None, ref["residual_out"], gamma, ref["mask"],
                    ref["mean"], ref["rstd"], with_dbeta=want_dbeta,
                    with_dbias=bias is not None)
    m = mags_backward(w, dparts, None, ref["residual_out"], gamma, ref["mean"],
                      ref["rstd"])
    return w, parts, bias, res, gamma, beta, ref, dparts, rb, m


@pytest.fixture(scope="module", autouse=True)
def _needs_gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    oracle.build()


NF, NB = sp.sp_plan_count()


@pytest.mark.parametrize("shape", sorted(SHAPES))
@pytest.mark.parametrize("plan", range(1, NF + 1))
def test_forward_plan(shape, plan):
    w, parts, bias, res, gamma, beta, ref, *_ = _case(shape)
    got = gpu_fwd(w, parts, bias, res, gamma, beta, plan=plan)
    check_forward(w, got, ref, parts, bias, res, gamma, beta)


@pytest.mark.parametrize("shape", sorted(SHAPES))
@pytest.mark.parametrize("plan", range(1, NB + 1))
def test_backward_plan(shape, plan):
    w, parts, bias, res, gamma, beta, ref, dparts, rb, m = _case(shape)
    run = lambda: gpu_bwd(w, dparts, None, ref["residual_out"], gamma,
                          ref["mask"], ref["mean"], ref["rstd"],
                          with_dbeta=rb["dbeta"] is not None,
                          with_dbias=rb["dbias"] is not None, plan=plan)
    got = run()
    # consumer groups that share accumulators take turns in a fixed order:
    # the parameter gradients are bitwise reproducible
    again = run()
    for k in ("dgamma", "dbeta", "dbias"):
        if got[k] is not None:
            assert np.array_equal(got[k], again[k]), k
    dt = w.torch_dtype
    assert_close("dresidual_in", got["dresidual_in"], rb["dresidual_in"],
                 m["dres"], dt)
    assert_close("dY", got["dY"], rb["dY"], m["dY"], dt)
    assert_sum_close("dgamma", got["dgamma"], rb["dgamma"], m["dgamma_terms"])
    if rb["dbeta"] is not None:
        assert_sum_close("dbeta", got["dbeta"], rb["dbeta"], m["dbeta_terms"])
    if rb["dbias"] is not None:
        assert_sum_close("dbias", got["dbias"], rb["dbias"], m["dbias_terms"])
