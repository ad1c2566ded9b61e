"""The backward entry point that allocates nothing.

Some callers cannot allocate device memory where they run the backward: a
memory-capped arena that owns every byte, an allocator that must not be
re-entered from inside this call, or a loop that may not synchronise (which
cudaMalloc and cudaFree can do).  sp_rs_norm_dropout_bwd_noalloc serves them
by keeping its scratch in a fixed 64 MiB array inside the library.  These
tests call it through the C ABI, twice in a row on each shape: the second
call finds the first call's leftovers in the shared array and must not
depend on them.

The no-scratch call picks the same kernel and plan as the ordinary backward
(which takes a caller-allocated workspace), so its outputs must equal that
call's bit for bit.  One shape is also checked against the CPU oracle, within
the parity tolerances.  The array holds min(rows, SMs) slices of 3*h fp32 for
the library's own plan choice: h = 8192 and h = 12288 must fit, and a shape
whose scratch exceeds 64 MiB is rejected before anything is launched.

This file is collected last, so a run that stops at the first failure has
already run every other test.
"""
import numpy as np
import pytest
import torch

import oracle
import sp_synth
from sp_synth import WORKLOADS
from _parity import assert_close, assert_sum_close, cfg_of, mags_backward

import sp_region_b200 as sp

pytestmark = pytest.mark.gpu

NOALLOC_BYTES = 64 << 20


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")


def _inputs(w):
    parts = sp_synth.draw_partials(w)
    bias, gamma, beta = sp_synth.draw_params(w)
    if not w.has_bias:
        bias = None
    if not w.has_beta or w.norm == "rmsnorm":
        beta = None
    res = sp_synth.draw_residual(w)
    oracle.build()
    ref = oracle.fwd(oracle.cfg_from(w), parts, bias, res, gamma, beta)
    dparts = sp_synth.draw_grad_partials(w)
    return bias, gamma, ref, dparts


def _outputs(w):
    N, h = w.rows, w.h
    dt = w.torch_dtype
    ln = w.norm == "layernorm"
    return dict(dres=torch.empty((N, h), dtype=dt, device="cuda"),
                dY=torch.empty((N, h), dtype=dt, device="cuda"),
                dg=torch.empty(h, dtype=torch.float32, device="cuda"),
                db=torch.empty(h, dtype=torch.float32, device="cuda")
                if ln else None,
                dc=torch.empty(h, dtype=torch.float32, device="cuda")
                if w.has_bias else None)


def _bits(x):
    return x.view(torch.int16 if x.dtype == torch.bfloat16 else torch.int32)


SHAPES = [
    ("C4_full", dict(base="C4")),
    ("C2_rows", dict(base="C2", s=256, b=2)),
    ("h8192_rmsnorm", dict(base="C3", s=1024)),
    ("h12288_outliers", dict(base="C5", s=1024)),
]


@pytest.mark.parametrize("name,over", SHAPES, ids=[n for n, _ in SHAPES])
def test_noalloc_backward_equals_the_workspace_backward(name, over):
    over = dict(over)
    w = WORKLOADS[over.pop("base")].replace(**over)
    bias, gamma, ref, dparts = _inputs(w)
    cfg = cfg_of(w)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    need = sp.sp_bwd_workspace_bytes(cfg)
    # the library's own plan choice writes one slice per CTA
    assert need == min(w.rows, sms) * 3 * w.h * 4
    assert need <= NOALLOC_BYTES

    d = lambda x: x.cuda()
    dp = [d(p) for p in dparts]
    x = d(ref["residual_out"])
    g = d(gamma)
    mask = (torch.from_numpy(ref["mask"].view(np.int32)).cuda()
            if w.p_drop > 0 else None)
    mean = (torch.from_numpy(ref["mean"].astype(np.float32)).cuda()
            if w.norm == "layernorm" else None)
    rstd = torch.from_numpy(ref["rstd"].astype(np.float32)).cuda()

    base = _outputs(w)
    ws = torch.empty(need // 4, dtype=torch.float32, device="cuda")
    ws.fill_(float("nan"))
    sp.sp_rs_norm_dropout_bwd(cfg, dp, None, x, g, mask, mean, rstd,
                              base["dres"], base["dY"], base["dg"],
                              base["db"], base["dc"], ws)
    torch.cuda.synchronize()
    assert sp.sp_device_error() == 0
    for call in range(2):
        out = _outputs(w)
        sp.sp_rs_norm_dropout_bwd_noalloc(cfg, dp, None, x, g, mask, mean,
                                          rstd, out["dres"], out["dY"],
                                          out["dg"], out["db"], out["dc"])
        torch.cuda.synchronize()
        assert sp.sp_device_error() == 0
        for k in out:
            if out[k] is not None:
                assert torch.equal(_bits(out[k]), _bits(base[k])), \
                    f"{k} differs from the workspace call (call {call})"

    if name == "C4_full":
        # and against the CPU oracle, fed the oracle's own forward outputs
        rb = oracle.bwd(oracle.cfg_from(w), dparts, None, ref["residual_out"],
                        gamma, ref["mask"], ref["mean"], ref["rstd"])
        m = mags_backward(w, dparts, None, ref["residual_out"], gamma,
                          ref["mean"], ref["rstd"])
        dt = w.torch_dtype
        assert_close("dresidual_in", out["dres"].cpu(), rb["dresidual_in"],
                     m["dres"], dt)
        assert_close("dY", out["dY"].cpu(), rb["dY"], m["dY"], dt)
        assert_sum_close("dgamma", out["dg"].cpu().numpy(), rb["dgamma"],
                         m["dgamma_terms"])
        assert_sum_close("dbeta", out["db"].cpu().numpy(), rb["dbeta"],
                         m["dbeta_terms"])
        assert_sum_close("dbias", out["dc"].cpu().numpy(), rb["dbias"],
                         m["dbias_terms"])


def test_noalloc_backward_rejects_shapes_beyond_its_scratch():
    """h = 40000 (wider than the fast kernels take: the general kernel, one
    slice per SM) over 148 rows needs 148 * 12 * 40000 = 71 MB of scratch,
    more than the fixed 64 MiB array: the call returns SP_ERR_UNSUPPORTED
    before launching anything.  The buffers are sized for the shape, so a
    launch would still be valid."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    w = WORKLOADS["C5"].replace(s=sms, b=1, t=1, h=40000, p_drop=0.0)
    cfg = cfg_of(w)
    if sp.sp_bwd_workspace_bytes(cfg) <= NOALLOC_BYTES:
        pytest.skip("this GPU has too few SMs for the shape to exceed 64 MiB")
    N, h = w.rows, w.h
    x = torch.zeros((N, h), dtype=torch.bfloat16, device="cuda")
    dp = torch.zeros((N, h), dtype=torch.bfloat16, device="cuda")
    g = torch.ones(h, dtype=torch.bfloat16, device="cuda")
    stats = torch.ones(N, dtype=torch.float32, device="cuda")
    o = _outputs(w)
    with pytest.raises(sp.SPError) as e:
        sp.sp_rs_norm_dropout_bwd_noalloc(cfg, [dp], None, x, g, None, stats,
                                          stats, o["dres"], o["dY"], o["dg"],
                                          o["db"], o["dc"])
    assert e.value.status == sp.SP_ERR_UNSUPPORTED
