"""The boundary as t real ranks would run it, emulated on one GPU.

Rank r calls the forward for its own token rows [r*N/t, (r+1)*N/t): it reads
its rows of every rank's partial sum (on a multi-GPU system, peers' buffers
through peer pointers), keeps its residual / stored outputs / mask /
statistics as a shard indexed from 0, and writes its normalised rows into
every rank's gathered buffer (the all-gather, pushed).  The backward does the
same with the upstream partials, pushing its dY rows into every rank's dY
buffer.  Run rank by rank on one GPU, the t
calls must reproduce the single whole-tensor call bit for bit (the dropout
counter uses the global row), and the per-rank parameter gradients must sum
to the whole call's ("Sequence Parallelism math", section "The collective
substitution"; "SP: Partition Activations Alongside TP", section "Change
layouts between SP and TP")."""
import numpy as np
import pytest
import torch

import sp_synth
from sp_synth import WORKLOADS
from _parity import assert_sum_close

import sp_region_b200 as sp

pytestmark = pytest.mark.gpu


def _cfg(w, r0=0, r1=0):
    return sp.make_cfg(w.s, w.b, w.h, w.t, dtype=w.dtype, norm=w.norm,
                       eps=w.eps, p_drop=w.p_drop, seed=w.drop_seed,
                       offset=w.drop_offset, row_begin=r0, row_end=r1)


def _empty_fwd(w, rows):
    dt = w.torch_dtype
    return dict(rout=torch.empty((rows, w.h), dtype=dt, device="cuda"),
                mask=torch.empty((rows, (w.h + 31) // 32), dtype=torch.int32,
                                 device="cuda"),
                mean=torch.empty(rows, dtype=torch.float32, device="cuda"),
                rstd=torch.empty(rows, dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("name,over", [
    ("C2_shape", dict(base="C2", s=160, b=2)),
    ("ragged_rank_rows", dict(base="C2", s=296, b=1, h=2048)),
    ("rms_t4", dict(base="C3", s=128, b=2, h=4096, t=4, p_drop=0.1,
                    has_bias=True)),
    ("general_h100", dict(base="C2", s=64, b=1, h=100, t=4)),
])
def test_ranks_reproduce_the_whole_call(name, over):
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    over = dict(over)
    w = WORKLOADS[over.pop("base")].replace(**over)
    N, h, t = w.rows, w.h, w.t
    per = N // t
    dt = w.torch_dtype
    parts = [p.cuda() for p in sp_synth.draw_partials(w)]
    bias, gamma, beta = (None if x is None else x.cuda()
                         for x in sp_synth.draw_params(w))
    if not w.has_bias:
        bias = None
    if w.norm == "rmsnorm" or not w.has_beta:
        beta = None
    res = sp_synth.draw_residual(w).cuda()

    # the whole tensor in one call
    whole = _empty_fwd(w, N)
    gat = torch.empty((N, h), dtype=dt, device="cuda")
    sp.sp_rs_bias_dropout_add_norm_fwd(_cfg(w), parts, bias, res, gamma, beta,
                                       whole["rout"], [gat], whole["mask"],
                                       whole["mean"], whole["rstd"])

    # t ranks: each its own shard, pushing into every rank's gathered buffer
    replicas = [torch.full((N, h), float("nan"), dtype=dt, device="cuda")
                for _ in range(t)]
    shards = []
    for r in range(t):
        o = _empty_fwd(w, per)
        sp.sp_rs_bias_dropout_add_norm_fwd(
            _cfg(w, r * per, (r + 1) * per), parts, bias,
            res[r * per:(r + 1) * per], gamma, beta, o["rout"], replicas,
            o["mask"], o["mean"], o["rstd"])
        shards.append(o)
    torch.cuda.synchronize()
    assert sp.sp_device_error() == 0
    bits = lambda x: x.view(torch.int16 if x.dtype == torch.bfloat16
                            else torch.int32)
    stored = ("rout", "mask", "rstd") + (("mean",) if w.norm == "layernorm"
                                         else ())   # RMSNorm writes no mean
    for k in stored:
        cat = torch.cat([o[k] for o in shards])
        assert torch.equal(bits(cat), bits(whole[k])), k
    for q in range(t):
        assert torch.equal(bits(replicas[q]), bits(gat)), q

    # backward: rank r reduce-scatters its rows of every upstream partial,
    # writes its dresidual_in shard and its rows of the gathered dY
    dparts = [d.cuda() for d in sp_synth.draw_grad_partials(w)]
    want_beta = w.norm == "layernorm"

    def grads():
        return (torch.empty(h, dtype=torch.float32, device="cuda"),
                torch.empty(h, dtype=torch.float32, device="cuda")
                if want_beta else None,
                torch.empty(h, dtype=torch.float32, device="cuda")
                if bias is not None else None)

    ws = torch.empty(sp.sp_bwd_workspace_bytes(_cfg(w)) // 4,
                     dtype=torch.float32, device="cuda")
    dres = torch.empty((N, h), dtype=dt, device="cuda")
    dY = torch.empty((N, h), dtype=dt, device="cuda")
    g0 = grads()
    sp.sp_rs_norm_dropout_bwd(_cfg(w), dparts, None, whole["rout"], gamma,
                              whole["mask"], whole["mean"], whole["rstd"],
                              dres, dY, *g0, ws)
    # every rank's dY copy, each filled by the t range calls' pushes
    dY_r = [torch.full((N, h), float("nan"), dtype=dt, device="cuda")
            for _ in range(t)]
    dres_r = []
    gsum = [np.zeros(h), np.zeros(h), np.zeros(h)]
    for r in range(t):
        sl = slice(r * per, (r + 1) * per)
        o = shards[r]
        dr = torch.empty((per, h), dtype=dt, device="cuda")
        gr = grads()
        sp.sp_rs_norm_dropout_bwd_ag(_cfg(w, r * per, (r + 1) * per), dparts,
                                     None, o["rout"], gamma, o["mask"],
                                     o["mean"], o["rstd"], dr, dY_r, *gr, ws)
        torch.cuda.synchronize()
        dres_r.append(dr)
        for q in range(3):
            if gr[q] is not None:
                gsum[q] += gr[q].cpu().double().numpy()
    assert sp.sp_device_error() == 0
    assert torch.equal(bits(torch.cat(dres_r)), bits(dres))
    for q in range(t):
        assert torch.equal(bits(dY_r[q]), bits(dY)), q
    # replicated parameters: the per-rank partial gradients sum to the whole
    dn_abs = sum(d.double().abs() for d in dparts).sum(0).cpu().numpy()
    for q in range(3):
        if g0[q] is not None:
            assert_sum_close(f"grad {q}", gsum[q], g0[q].cpu().double().numpy(),
                             dn_abs * 8.0)
