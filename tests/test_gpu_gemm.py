"""The tensor-parallel linears with the SP collectives fused into them,
through the C ABI, against the CPU oracle.

Row-parallel linear: x [rows, f] @ w [h, f]^T with the t ranks' slices of f
reduced in the tensor cores' accumulator, then bias, dropout, residual add
(sp_rowpar_linear_rs_fwd), then the norm and the all-gather
(sp_linear_rs_bias_dropout_add_norm_fwd).  Column-parallel linear: the t
sequence shards all-gathered in the GEMM's prologue (sp_ag_colpar_linear_fwd).

Small shapes cover several tiles, ragged rows, a ragged inner dimension, a
ragged last column tile, mask padding bytes, a row range, both norms, p = 0
and t = 1..8; the 22B-class layer shape (s = 2048, b = 4, h = 6144, t = 8,
FFN down-projection f = 4h) runs at full size and is compared on sampled
rows.  The tolerance adds to the boundary's bounds the fp32 accumulation of
K products in the tensor cores (see _parity.mag_linear_rout).
"""
import concurrent.futures
import gc
import os

import numpy as np
import pytest
import torch

import oracle
import sp_synth
from sp_synth import WORKLOADS
from _parity import (assert_close, check_forward, mag_linear_out,
                     mag_linear_rout)

import sp_region_b200 as sp

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    oracle.build()
    yield
    gc.collect()
    torch.cuda.empty_cache()


def _bf16(shape, seed, scale=1.0, device="cpu"):
    g = torch.Generator(device=device).manual_seed(seed)
    return (torch.randn(shape, generator=g, device=device) * scale).to(torch.bfloat16)


def _cfg(w, row_begin=0, row_end=0):
    return sp.make_cfg(w.s, w.b, w.h, w.t, dtype="bf16", norm=w.norm, eps=w.eps,
                       p_drop=w.p_drop, seed=w.drop_seed, offset=w.drop_offset,
                       row_begin=row_begin, row_end=row_end)


def _run_linear(w, f, x, wt, bias, res, gamma, beta, row_begin=0, row_end=0):
    rows = x.shape[0]
    h = w.h
    d = lambda v: None if v is None else v.cuda()
    rout = torch.empty((rows, h), dtype=torch.bfloat16, device="cuda")
    out = torch.full((w.rows, h), float("nan"), dtype=torch.bfloat16, device="cuda")
    mask = (torch.full((rows, (h + 31) // 32), -1, dtype=torch.int32, device="cuda")
            if w.p_drop > 0 else None)
    mean = torch.empty(rows, dtype=torch.float32, device="cuda")
    rstd = torch.empty(rows, dtype=torch.float32, device="cuda")
    sp.sp_linear_rs_bias_dropout_add_norm_fwd(
        _cfg(w, row_begin, row_end), f, d(x), d(wt), d(bias), d(res), d(gamma),
        d(beta), rout, [out], mask, mean if w.norm == "layernorm" else None, rstd)
    torch.cuda.synchronize()
    assert sp.sp_device_error() == 0
    r0 = row_begin
    return dict(residual_out=rout.cpu(), norm_out=out[r0:r0 + rows].cpu(),
                mask=None if mask is None else mask.cpu().numpy().view(np.uint32),
                mean=mean.cpu().numpy() if w.norm == "layernorm" else None,
                rstd=rstd.cpu().numpy())


CASES = [
    # name, rows (s*b), f, h, t, p, bias, norm
    ("one_tile_t2", 128, 256, 256, 2, 0.1, True, "layernorm"),
    ("ragged_rows_k_cols", 300, 520, 264, 4, 0.1, True, "layernorm"),
    ("two_col_tiles_rms_p0", 192, 512, 384, 4, 0.0, False, "rmsnorm"),
    ("c2_width_t8", 256, 1024, 6144, 8, 0.1, True, "layernorm"),
    ("t1", 128, 136, 128, 1, 0.25, True, "layernorm"),
    # 80 CTA-pair tiles: more than a B200's 74 clusters take in one round
    ("two_rounds_of_pair_tiles", 2048, 256, 2560, 4, 0.1, True, "layernorm"),
]


@pytest.mark.parametrize("name,rows,f,h,t,p,has_bias,norm", CASES,
                         ids=[c[0] for c in CASES])
def test_rowpar_linear_boundary_matches_oracle(name, rows, f, h, t, p, has_bias,
                                               norm):
    w = WORKLOADS["C2"].replace(s=rows, b=1, h=h, t=t, p_drop=p, norm=norm,
                                has_bias=has_bias, has_beta=norm == "layernorm",
                                eps=1e-5 if norm == "layernorm" else 1e-6)
    x = _bf16((rows, f), 101, scale=f ** -0.5)
    wt = _bf16((h, f), 102)
    bias, gamma, beta = sp_synth.draw_params(w)
    bias = bias if has_bias else None
    beta = beta if norm == "layernorm" else None
    res = sp_synth.draw_residual(w)
    got = _run_linear(w, f, x, wt, bias, res, gamma, beta)
    cfg = oracle.cfg_from(w)
    ref = oracle.linear_rs_fwd_rows(cfg, f, list(range(rows)), x, wt, bias, res,
                                    gamma, beta)
    y = oracle.rowpar_reduce(x, wt, t)
    check_forward(w, got, ref, None, bias, res, gamma, beta,
                  mag_rout=mag_linear_rout(w, x, wt, bias, res, y))
    if got["mask"] is not None:
        assert np.array_equal(got["mask"], ref["mask"])


def test_rowpar_linear_row_range_uses_global_rows():
    """A call on rows [128, 384) of 512: x, residual and the stored outputs
    hold those rows only, the dropout mask is drawn for the global rows and
    the norm output lands at the global rows of the gathered buffer."""
    w = WORKLOADS["C2"].replace(s=512, b=1, h=256, t=4, p_drop=0.1)
    f, r0, r1 = 256, 128, 384
    x = _bf16((r1 - r0, f), 111, scale=f ** -0.5)
    wt = _bf16((w.h, f), 112)
    bias, gamma, beta = sp_synth.draw_params(w)
    res = sp_synth.draw_residual(w, rows=r1 - r0)
    got = _run_linear(w, f, x, wt, bias, res, gamma, beta, r0, r1)
    ref = oracle.linear_rs_fwd_rows(oracle.cfg_from(w), f, list(range(r0, r1)),
                                    x, wt, bias, res, gamma, beta)
    y = oracle.rowpar_reduce(x, wt, w.t)
    check_forward(w, got, ref, None, bias, res, gamma, beta,
                  mag_rout=mag_linear_rout(w, x, wt, bias, res, y))
    assert np.array_equal(got["mask"], ref["mask"])


def test_rowpar_linear_rejects_what_it_does_not_take():
    w = WORKLOADS["C2"].replace(s=128, b=1, h=256, t=4)
    x = torch.zeros((128, 260), dtype=torch.bfloat16, device="cuda")
    wt = torch.zeros((256, 260), dtype=torch.bfloat16, device="cuda")
    r = torch.zeros((128, 256), dtype=torch.bfloat16, device="cuda")
    m = torch.zeros((128, 8), dtype=torch.int32, device="cuda")
    with pytest.raises(sp.SPError) as e:        # f % t != 0
        sp.sp_rowpar_linear_rs_fwd(_cfg(w), 258, x, wt, None, r, r.clone(), m)
    assert e.value.status == sp.SP_ERR_INVALID_ARG
    with pytest.raises(sp.SPError) as e:        # f % 8 != 0
        sp.sp_rowpar_linear_rs_fwd(_cfg(w), 260, x, wt, None, r, r.clone(), m)
    assert e.value.status == sp.SP_ERR_UNSUPPORTED
    wf = WORKLOADS["C1"].replace(s=128, b=1, h=256, t=4)   # fp32 I/O
    c = sp.make_cfg(wf.s, wf.b, wf.h, wf.t, dtype="f32", p_drop=0.1)
    with pytest.raises(sp.SPError) as e:
        sp.sp_rowpar_linear_rs_fwd(c, 256, x, wt, None, r, r.clone(), m)
    assert e.value.status == sp.SP_ERR_UNSUPPORTED


AG_CASES = [
    # name, N, h (inner), f_out, t
    ("t2", 256, 256, 384, 2),
    ("t4_ragged_cols", 1024, 512, 264, 4),
    ("t1_ragged_rows_k", 300, 520, 128, 1),
    ("t8", 1024, 1024, 512, 8),
    ("two_rounds_of_pair_tiles", 2048, 256, 2560, 4),
]


@pytest.mark.parametrize("name,N,h,f_out,t", AG_CASES, ids=[c[0] for c in AG_CASES])
def test_ag_colpar_linear_matches_oracle(name, N, h, f_out, t):
    per = N // t
    shards = [_bf16((per, h), 200 + r) for r in range(t)]
    wt = _bf16((f_out, h), 300, scale=h ** -0.5)
    out = torch.full((N, f_out), float("nan"), dtype=torch.bfloat16, device="cuda")
    cfg = sp.make_cfg(N, 1, h, t, dtype="bf16")
    sp.sp_ag_colpar_linear_fwd(cfg, f_out, [s_.cuda() for s_ in shards], wt.cuda(), out)
    torch.cuda.synchronize()
    assert sp.sp_device_error() == 0
    ref = oracle.ag_colpar_fwd(shards, wt)
    assert_close("column-parallel out", out.cpu(), ref,
                 mag_linear_out(torch.cat(shards), wt), torch.bfloat16)


def test_ag_colpar_linear_rejects_tiles_across_shards():
    t, N, h = 4, 4 * 96, 128          # 96 rows per shard: a 128-row tile spans two
    shards = [torch.zeros((N // t, h), dtype=torch.bfloat16, device="cuda")
              for _ in range(t)]
    wt = torch.zeros((128, h), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((N, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sp.SPError) as e:
        sp.sp_ag_colpar_linear_fwd(sp.make_cfg(N, 1, h, t), 128, shards, wt, out)
    assert e.value.status == sp.SP_ERR_UNSUPPORTED


def _sample_rows(N, t, seed, extra=12):
    per = N // t
    rows = {0, N - 1}
    for r in range(1, t):
        rows.update((r * per - 1, r * per))
    rng = np.random.default_rng(seed)
    rows.update(int(v) for v in rng.integers(0, N, size=extra))
    return sorted(rows)


def _pool():
    return concurrent.futures.ThreadPoolExecutor(
        max_workers=max(1, min(16, os.cpu_count() or 1)))


def test_c2_layer_ffn_down_projection_full_size_sampled():
    """The 22B-class layer shape: s = 2048, b = 4, h = 6144, t = 8, the FFN
    down-projection's inner dimension f = 4h = 24576 (each rank's slice 3072).
    The fused forward runs at full size; sampled rows (both ends, both sides
    of every rank boundary, random) are compared with the oracle, which
    reduces the eight 3072-wide partials of each sampled row in double."""
    w = WORKLOADS["C2"]
    N, h, t = w.rows, w.h, w.t
    f = 4 * h
    x = _bf16((N, f), 401, scale=f ** -0.5, device="cuda")
    wt = _bf16((h, f), 402, device="cuda")
    bias, gamma, beta = sp_synth.draw_params(w, "cuda")
    res = sp_synth.draw_residual(w, "cuda")
    rout = torch.empty((N, h), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((N, h), dtype=torch.bfloat16, device="cuda")
    mask = torch.empty((N, (h + 31) // 32), dtype=torch.int32, device="cuda")
    mean = torch.empty(N, dtype=torch.float32, device="cuda")
    rstd = torch.empty(N, dtype=torch.float32, device="cuda")
    sp.sp_linear_rs_bias_dropout_add_norm_fwd(_cfg(w), f, x, wt, bias, res, gamma,
                                              beta, rout, [out], mask, mean, rstd)
    torch.cuda.synchronize()
    assert sp.sp_device_error() == 0
    rows = _sample_rows(N, t, seed=77)
    idx = torch.tensor(rows, device="cuda")
    xr, wt_c = x[idx].cpu(), wt.cpu()
    bias_c, gamma_c, beta_c, rr = bias.cpu(), gamma.cpu(), beta.cpu(), res[idx].cpu()
    cfg = oracle.cfg_from(w)
    oracle.mask_words(h)   # loads the oracle library before the threads start

    def one(i):
        return oracle.linear_rs_fwd_rows(cfg, f, [rows[i]], xr[i:i + 1], wt_c,
                                         bias_c, rr[i:i + 1], gamma_c, beta_c)
    with _pool() as ex:
        refs = list(ex.map(one, range(len(rows))))
    ref = dict(residual_out=torch.cat([r["residual_out"] for r in refs]),
               norm_out=torch.cat([r["norm_out"] for r in refs]),
               mask=np.concatenate([r["mask"] for r in refs]),
               mean=np.concatenate([r["mean"] for r in refs]),
               rstd=np.concatenate([r["rstd"] for r in refs]))
    got = dict(residual_out=rout[idx].cpu(), norm_out=out[idx].cpu(),
               mask=mask[idx].cpu().numpy().view(np.uint32),
               mean=mean[idx].cpu().numpy(), rstd=rstd[idx].cpu().numpy())
    with _pool() as ex:
        y = np.concatenate(list(ex.map(
            lambda i: oracle.rowpar_reduce(xr[i:i + 1], wt_c, t), range(len(rows)))))
    check_forward(w, got, ref, None, bias_c, rr, gamma_c, beta_c,
                  mag_rout=mag_linear_rout(w, xr, wt_c, bias_c, rr, y))
    assert np.array_equal(got["mask"], ref["mask"])
