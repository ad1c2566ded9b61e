"""sp_region_b200.ranks with the real library calls, on a one-rank NCCL group
(the one GPU here): SPBoundary's forward and backward, with their row range,
rendezvous, dY pushed by the kernel and gradient all-reduce, must give the
bits of the direct library calls.  Peer-mapped buffers (several GPUs) are not exercised."""
import socket

import pytest
import torch

import sp_synth
from sp_synth import WORKLOADS

import sp_region_b200 as sp

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture()
def one_rank_group():
    import torch.distributed as dist
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}",
                            rank=0, world_size=1,
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        yield
    finally:
        dist.destroy_process_group()


def test_one_rank_boundary_gives_the_direct_calls_bits(one_rank_group):
    from sp_region_b200.ranks import SPBoundary
    w = WORKLOADS["C2"].replace(s=96, b=2, t=1)
    N, h = w.rows, w.h
    dev = "cuda"
    parts = [p.to(dev) for p in sp_synth.draw_partials(w)]
    bias, gamma, beta = (x.to(dev) for x in sp_synth.draw_params(w))
    res = sp_synth.draw_residual(w).to(dev)
    cfg = sp.make_cfg(w.s, w.b, h, 1, dtype=w.dtype, norm=w.norm, eps=w.eps,
                      p_drop=w.p_drop, seed=w.drop_seed, offset=w.drop_offset)
    bf = dict(dtype=torch.bfloat16, device=dev)
    W = (h + 31) // 32

    def fwd_bufs():
        return dict(rout=torch.empty(N, h, **bf), out=torch.empty(N, h, **bf),
                    mask=torch.empty(N, W, dtype=torch.int32, device=dev),
                    mean=torch.empty(N, device=dev), rstd=torch.empty(N, device=dev))

    d = fwd_bufs()
    sp.sp_rs_bias_dropout_add_norm_fwd(cfg, parts, bias, res, gamma, beta, d["rout"],
                                       [d["out"]], d["mask"], d["mean"], d["rstd"])
    e = fwd_bufs()
    sb = SPBoundary(timeout_s=30.0)
    sb.forward(cfg, parts, bias, res, gamma, beta, e["rout"], [e["out"]], e["mask"],
               e["mean"], e["rstd"])
    torch.cuda.synchronize()
    assert sp.sp_device_error() == 0
    for k in ("rout", "out", "mask", "mean", "rstd"):
        assert torch.equal(d[k].view(torch.int16 if d[k].dtype == torch.bfloat16
                                     else d[k].dtype), e[k].view(
            torch.int16 if e[k].dtype == torch.bfloat16 else e[k].dtype)), k

    dparts = [p.to(dev) for p in sp_synth.draw_grad_partials(w)]
    ws = torch.empty(sp.sp_bwd_workspace_bytes(cfg) // 4, device=dev)

    def bwd_bufs():
        return dict(dres=torch.empty(N, h, **bf), dY=torch.empty(N, h, **bf),
                    dg=torch.empty(h, device=dev), db=torch.empty(h, device=dev),
                    dc=torch.empty(h, device=dev))

    a = bwd_bufs()
    sp.sp_rs_norm_dropout_bwd(cfg, dparts, None, d["rout"], gamma, d["mask"],
                              d["mean"], d["rstd"], a["dres"], a["dY"], a["dg"],
                              a["db"], a["dc"], ws)
    b = bwd_bufs()
    sb.backward(cfg, dparts, None, d["rout"], gamma, d["mask"], d["mean"], d["rstd"],
                b["dres"], [b["dY"]], b["dg"], b["db"], b["dc"], ws)
    torch.cuda.synchronize()
    assert sp.sp_device_error() == 0
    for k in ("dres", "dY"):
        assert torch.equal(a[k].view(torch.int16), b[k].view(torch.int16)), k
    for k in ("dg", "db", "dc"):
        assert torch.equal(a[k], b[k]), k
