"""The backward entry point that allocates nothing.

Some callers cannot allocate device memory where they run the backward: a
memory-capped arena that owns every byte, an allocator that must not be
re-entered from inside this call, or a loop that may not synchronise (which
cudaMalloc and cudaFree can do).  sp_rs_norm_dropout_bwd_noalloc serves them
by keeping its scratch in a fixed array inside the library.  These tests call
it through the C ABI and check its outputs against the ordinary backward
(which takes a caller-allocated workspace), within the same tolerances as the
oracle parity tests, on two calls in a row: the second call finds the first
call's leftovers in the shared array and must not depend on them.

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


def _inputs(w):
    parts = sp_synth.draw_partials(w)
    bias, gamma, beta = sp_synth.draw_params(w)
    res = sp_synth.draw_residual(w)
    oracle.build()
    ref = oracle.fwd(oracle.cfg_from(w), parts, bias, res, gamma, beta)
    dparts = sp_synth.draw_grad_partials(w)
    return gamma, ref, dparts


def _outputs(w):
    N, h = w.rows, w.h
    dt = w.torch_dtype
    return dict(dres=torch.empty((N, h), dtype=dt, device="cuda"),
                dY=torch.empty((N, h), dtype=dt, device="cuda"),
                dg=torch.empty(h, dtype=torch.float32, device="cuda"),
                db=torch.empty(h, dtype=torch.float32, device="cuda"),
                dc=torch.empty(h, dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("name,over", [
    ("C4_full", dict(base="C4")),
    ("C2_rows", dict(base="C2", s=256, b=2)),
])
def test_noalloc_backward_matches_the_workspace_backward(name, over):
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    over = dict(over)
    w = WORKLOADS[over.pop("base")].replace(**over)
    gamma, ref, dparts = _inputs(w)
    cfg = cfg_of(w)
    d = lambda x: x.cuda()
    dp = [d(p) for p in dparts]
    x = d(ref["residual_out"])
    g = d(gamma)
    mask = torch.from_numpy(ref["mask"].view(np.int32)).cuda()
    mean = torch.from_numpy(ref["mean"].astype(np.float32)).cuda()
    rstd = torch.from_numpy(ref["rstd"].astype(np.float32)).cuda()

    base = _outputs(w)
    ws = torch.empty(sp.sp_bwd_workspace_bytes(cfg) // 4, dtype=torch.float32,
                     device="cuda")
    sp.sp_rs_norm_dropout_bwd(cfg, dp, None, x, g, mask, mean, rstd,
                              base["dres"], base["dY"], base["dg"],
                              base["db"], base["dc"], ws)
    torch.cuda.synchronize()
    m = mags_backward(w, dparts, None, ref["residual_out"], gamma,
                      ref["mean"], ref["rstd"])
    dt = w.torch_dtype
    for call in range(2):
        out = _outputs(w)
        sp.sp_rs_norm_dropout_bwd_noalloc(cfg, dp, None, x, g, mask, mean,
                                          rstd, out["dres"], out["dY"],
                                          out["dg"], out["db"], out["dc"])
        torch.cuda.synchronize()
        assert sp.sp_device_error() == 0
        assert_close(f"dresidual_in (call {call})", out["dres"].cpu(),
                     base["dres"].cpu(), m["dres"], dt)
        assert_close(f"dY (call {call})", out["dY"].cpu(), base["dY"].cpu(),
                     m["dY"], dt)
        assert_sum_close(f"dgamma (call {call})", out["dg"].cpu().numpy(),
                         base["dg"].cpu().numpy(), m["dgamma_terms"])
        assert_sum_close(f"dbeta (call {call})", out["db"].cpu().numpy(),
                         base["db"].cpu().numpy(), m["dbeta_terms"])
        assert_sum_close(f"dbias (call {call})", out["dc"].cpu().numpy(),
                         base["dc"].cpu().numpy(), m["dbias_terms"])


def test_noalloc_backward_rejects_shapes_beyond_its_scratch():
    """592 rows of h = 12288 need 87 MB of scratch, more than the fixed 64 MiB
    array: the call returns SP_ERR_UNSUPPORTED before launching anything.
    The buffers are sized for the shape, so a launch would still be valid."""
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    w = WORKLOADS["C5"].replace(s=592, b=1, t=1, p_drop=0.0)
    cfg = cfg_of(w)
    if sp.sp_bwd_workspace_bytes(cfg) <= 64 << 20:
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
