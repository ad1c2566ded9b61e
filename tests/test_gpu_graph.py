"""A forward + backward step of the boundary captured once into a CUDA graph
and replayed.  The C-ABI calls make only host-side queries and plain kernel
launches on the caller's stream, so a step is capturable; replaying it gives
the same bits as the eager calls, and small, launch-bound steps drop their
host overhead."""
import numpy as np
import pytest
import torch

import sp_synth
from sp_synth import WORKLOADS
from _parity import cfg_of

import sp_region_b200 as sp

pytestmark = pytest.mark.gpu


def _setup(w):
    N, h = w.rows, w.h
    dt = w.torch_dtype
    d = dict(parts=[p.cuda() for p in sp_synth.draw_partials(w)],
             res=sp_synth.draw_residual(w).cuda(),
             dparts=[p.cuda() for p in sp_synth.draw_grad_partials(w)])
    bias, gamma, beta = sp_synth.draw_params(w)
    d.update(bias=bias.cuda(), gamma=gamma.cuda(), beta=beta.cuda())
    for k in ("rout", "out", "dres", "dY"):
        d[k] = torch.empty((N, h), dtype=dt, device="cuda")
    d["mask"] = torch.empty((N, (h + 31) // 32), dtype=torch.int32,
                            device="cuda")
    for k in ("mean", "rstd"):
        d[k] = torch.empty(N, dtype=torch.float32, device="cuda")
    for k in ("dg", "db", "dc"):
        d[k] = torch.empty(h, dtype=torch.float32, device="cuda")
    cfg = cfg_of(w)
    d["ws"] = torch.empty(sp.sp_bwd_workspace_bytes(cfg) // 4,
                          dtype=torch.float32, device="cuda")
    return cfg, d


def _step(cfg, d, stream):
    sp.sp_rs_bias_dropout_add_norm_fwd(cfg, d["parts"], d["bias"], d["res"],
                                       d["gamma"], d["beta"], d["rout"],
                                       [d["out"]], d["mask"], d["mean"],
                                       d["rstd"], stream=stream)
    sp.sp_rs_norm_dropout_bwd(cfg, d["dparts"], None, d["rout"], d["gamma"],
                              d["mask"], d["mean"], d["rstd"], d["dres"],
                              d["dY"], d["dg"], d["db"], d["dc"], d["ws"],
                              stream=stream)


OUTS = ("rout", "out", "mask", "mean", "rstd", "dres", "dY", "dg", "db", "dc")


@pytest.mark.parametrize("name,over", [("C2_rows", dict(base="C2", s=256, b=2)),
                                       ("small", dict(base="C2", s=16, b=1,
                                                      h=1024, t=4))])
def test_step_replays_from_a_cuda_graph(name, over):
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    over = dict(over)
    w = WORKLOADS[over.pop("base")].replace(**over)
    cfg, d = _setup(w)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        _step(cfg, d, s)          # eager: also warms the kernels up
    torch.cuda.synchronize()
    eager = {k: d[k].clone() for k in OUTS}
    for k in OUTS:
        d[k].zero_()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        _step(cfg, d, s)
    for _ in range(2):            # replay twice: the same bits each time
        for k in OUTS:
            d[k].zero_()
        g.replay()
        torch.cuda.synchronize()
        assert sp.sp_device_error() == 0
        for k in OUTS:
            a, b = d[k], eager[k]
            iv = torch.int16 if a.dtype == torch.bfloat16 else torch.int32
            assert torch.equal(a.view(iv), b.view(iv)), k
    del g
