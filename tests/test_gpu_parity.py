"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Small cases compare every element and cover several CTAs per launch, ragged
row tails (rows not a multiple of the grid), ragged vector tails (h/8 not a
multiple of the consumer thread count), both dtypes, both norms, the general
kernel (h % 8 != 0, misaligned pointers), t = 1 and t = 64, replicas, and the
optional outputs.  The five workloads at full size run in the launch
configuration the benchmark times and are compared on sampled token rows,
plus properties that hold at any size.
"""
import numpy as np
import pytest
import torch

import oracle
import sp_synth
from sp_synth import WORKLOADS
from _parity import (assert_close, assert_sum_close, check_forward,
                     gpu_bwd, gpu_fwd,
                     mag_norm_out, mag_residual_out, mags_backward,
                     unpack_mask, cfg_of, Guarded)

import sp_region_b200 as sp

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _needs_gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    oracle.build()


def _inputs(w, device="cpu"):
    parts = sp_synth.draw_partials(w, device)
    bias, gamma, beta = sp_synth.draw_params(w, device)
    res = sp_synth.draw_residual(w, device)
    if not w.has_bias:
        bias = None
    if not w.has_beta or w.norm == "rmsnorm":
        beta = None
    return parts, bias, res, gamma, beta


def _check_fwd(w, got, ref, parts, bias, res, gamma, beta, n_gathered=1):
    check_forward(w, got, ref, parts, bias, res, gamma, beta, n_gathered)


FWD_CASES = {
    # name: workload overrides
    "C1_worked_f32": dict(base="C1"),
    "bf16_ln_h6144_t8_ragged_rows": dict(base="C2", s=200, b=3),
    "bf16_ln_h1000_t3_ragged_vectors": dict(base="C2", s=111, b=3, h=1000, t=3),
    "bf16_rms_h8192_t8_p0": dict(base="C3", s=304, b=1),
    "bf16_ln_h12288_t16_outliers": dict(base="C5", s=160, b=1),
    "bf16_ln_h16384_t2": dict(base="C2", s=64, b=1, h=16384, t=2),
    "bf16_ln_h32768_cluster": dict(base="C2", s=80, b=2, h=32768, t=2),
    "bf16_ln_h4096_t4": dict(base="C4", s=300, b=2),
    "f32_ln_h512_t2": dict(base="C2", s=64, b=3, h=512, t=2, dtype="f32"),
    "f32_rms_h2048_t4": dict(base="C3", s=96, b=1, h=2048, t=4, dtype="f32"),
    "bf16_general_h100": dict(base="C2", s=40, b=2, h=100, t=4),
    "f32_general_h36": dict(base="C1", s=30, b=1, h=36, t=3),
    "bf16_t1": dict(base="C2", s=70, b=1, h=256, t=1),
    "bf16_t64_h64": dict(base="C2", s=128, b=1, h=64, t=64),
    "bf16_h8_one_vector": dict(base="C2", s=16, b=1, h=8, t=2),
    "bf16_single_row": dict(base="C2", s=1, b=1, h=6144, t=1),
    "bf16_rms_bias_p01": dict(base="C3", s=64, b=2, h=1536, t=4,
                                 p_drop=0.1, has_bias=True),
    "bf16_seed_offset": dict(base="C2", s=32, b=1, h=768, t=2,
                             drop_seed=0xFEEDFACECAFEBEEF,
                             drop_offset=(7 << 32) + 3),
}


def _workload(spec):
    spec = dict(spec)
    w = WORKLOADS[spec.pop("base")]
    return w.replace(**spec)


@pytest.mark.parametrize("name", sorted(FWD_CASES))
def test_forward_matches_oracle(name):
    w = _workload(FWD_CASES[name])
    parts, bias, res, gamma, beta = _inputs(w)
    ref = oracle.fwd(oracle.cfg_from(w), parts, bias, res, gamma, beta)
    got = gpu_fwd(w, parts, bias, res, gamma, beta)
    _check_fwd(w, got, ref, parts, bias, res, gamma, beta)


def test_forward_worked_value_nine():
    """The worked layout's token t0, feature 0 reduces 4 + 5 = 9 on rank 0;
    with p = 0, no bias and a zero residual the stored sum is exactly 9."""
    w = WORKLOADS["C1"].replace(p_drop=0.0)
    parts, bias, res, gamma, beta = _inputs(w)
    got = gpu_fwd(w, parts, None, torch.zeros_like(res), gamma, beta)
    assert float(got["residual_out"][0, 0]) == 9.0


def test_forward_replicas_and_optional_outputs():
    w = WORKLOADS["C3"].replace(s=64, b=2, h=1024, t=4)
    parts, bias, res, gamma, beta = _inputs(w)
    ref = oracle.fwd(oracle.cfg_from(w), parts, bias, res, gamma, beta)
    got = gpu_fwd(w, parts, bias, res, gamma, beta, n_gathered=w.t)
    _check_fwd(w, got, ref, parts, bias, res, gamma, beta, n_gathered=w.t)
    for q in range(1, w.t):
        assert torch.equal(got["gathered"][q], got["gathered"][0])
    got2 = gpu_fwd(w, parts, bias, res, gamma, beta, with_mask=False,
                   with_stats=False)
    assert torch.equal(got2["gathered"][0], got["gathered"][0])


def test_forward_in_place_residual():
    w = WORKLOADS["C2"].replace(s=48, b=2, h=2048, t=4)
    parts, bias, res, gamma, beta = _inputs(w)
    ref = oracle.fwd(oracle.cfg_from(w), parts, bias, res, gamma, beta)
    got = gpu_fwd(w, parts, bias, res, gamma, beta, inplace=True)
    _check_fwd(w, got, ref, parts, bias, res, gamma, beta)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_forward_misaligned_pointers_take_the_general_kernel(dtype):
    w = WORKLOADS["C2"].replace(s=32, b=2, h=1024, t=4, dtype=dtype)
    parts, bias, res, gamma, beta = _inputs(w)
    ref = oracle.fwd(oracle.cfg_from(w), parts, bias, res, gamma, beta)
    got = gpu_fwd(w, parts, bias, res, gamma, beta, offset_elems=1)
    _check_fwd(w, got, ref, parts, bias, res, gamma, beta)


@pytest.mark.parametrize("norm", ["layernorm", "rmsnorm"])
def test_forward_is_independent_of_t(norm):
    """Bit-identical outputs for t in {1, 2, 4, 8, 16} when the partials add
    exactly (dyadic atoms grouped per t)."""
    base = WORKLOADS["C2"].replace(s=64, b=1, h=6144, norm=norm,
                                    has_beta=norm == "layernorm")
    atoms = sp_synth.dyadic_atoms(base.rows, base.h, seed=5)
    outs = []
    for t in (1, 2, 4, 8, 16):
        w = base.replace(t=t)
        parts = sp_synth.group_atoms(atoms, t, w.torch_dtype)
        _, bias, res, gamma, beta = _inputs(w)
        outs.append(gpu_fwd(w, parts, bias, res, gamma, beta))
    for o in outs[1:]:
        assert torch.equal(o["residual_out"], outs[0]["residual_out"])
        assert torch.equal(o["gathered"][0], outs[0]["gathered"][0])
        assert np.array_equal(o["mask"], outs[0]["mask"])
        assert np.array_equal(o["rstd"], outs[0]["rstd"])


def test_forward_run_twice_bitwise():
    w = WORKLOADS["C2"].replace(s=160, b=2, h=6144, t=8)
    parts, bias, res, gamma, beta = _inputs(w)
    a = gpu_fwd(w, parts, bias, res, gamma, beta)
    b = gpu_fwd(w, parts, bias, res, gamma, beta)
    assert torch.equal(a["residual_out"], b["residual_out"])
    assert torch.equal(a["gathered"][0], b["gathered"][0])
    assert np.array_equal(a["mask"], b["mask"])


# ----------------------------------------------------------------------------
# all-gather
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,h,t,n_out", [("bf16", 6144, 8, 1),
                                             ("bf16", 8192, 8, 8),
                                             ("f32", 36, 3, 2),
                                             ("bf16", 100, 4, 3)])
def test_all_gather_matches_oracle(dtype, h, t, n_out):
    w = WORKLOADS["C3"].replace(s=8 * t, b=3, h=h, t=t, dtype=dtype)
    rows = w.rows // t
    shards = [sp_synth.draw_residual(w.replace(seed=40 + r), rows=rows)
              for r in range(t)]
    ref = oracle.all_gather([s_.double().numpy() for s_ in shards])
    dsh = [s_.cuda() for s_ in shards]
    outs = [Guarded((w.rows, h), w.torch_dtype) for _ in range(n_out)]
    sp.sp_all_gather(cfg_of(w), dsh, [o.t for o in outs])
    torch.cuda.synchronize()
    for o in outs:
        assert o.intact()
        assert np.array_equal(o.t.double().cpu().numpy(), ref)


# ----------------------------------------------------------------------------
# backward
# ----------------------------------------------------------------------------

BWD_CASES = {
    "bf16_ln_h4096_t4": dict(base="C4", s=300, b=2),
    "bf16_ln_h6144_t8_drnext": dict(base="C2", s=160, b=2, drnext=True),
    "bf16_ln_h12288_t16": dict(base="C5", s=160, b=1),
    "bf16_rms_h8192_p0_nomask": dict(base="C3", s=152, b=1, nomask=True),
    "bf16_ln_h1000_ragged": dict(base="C2", s=111, b=3, h=1000, t=3),
    "bf16_general_h100": dict(base="C2", s=40, b=2, h=100, t=4, drnext=True),
    # h % 4 != 0: the column sums take their one-column-per-lane form
    "bf16_general_h90": dict(base="C2", s=48, b=2, h=90, t=3, drnext=True),
    "f32_general_h30": dict(base="C1", s=30, b=1, h=30, t=3),
    "f32_ln_h512": dict(base="C2", s=64, b=3, h=512, t=2, dtype="f32"),
    "f32_general_worked": dict(base="C1", drnext=True),
    "bf16_ln_no_dbias_dbeta": dict(base="C4", s=64, b=1, h=2048,
                                   no_param_grads=True),
    "bf16_ln_h16384_t2": dict(base="C2", s=64, b=1, h=16384, t=2),
    "bf16_ln_h32768_cluster": dict(base="C2", s=80, b=2, h=32768, t=2),
    "bf16_t64_h64": dict(base="C2", s=128, b=1, h=64, t=64),
}


def _run_bwd_case(spec, offset_elems=0):
    spec = dict(spec)
    drn_on = spec.pop("drnext", False)
    nomask = spec.pop("nomask", False)
    no_pg = spec.pop("no_param_grads", False)
    w = _workload(spec)
    parts, bias, res, gamma, beta = _inputs(w)
    cfg = oracle.cfg_from(w)
    fo = oracle.fwd(cfg, parts, bias, res, gamma, beta)
    dparts = sp_synth.draw_grad_partials(w)
    drn = sp_synth.draw_residual_grad(w) if drn_on else None
    mask = None if nomask else fo["mask"]
    want_dbeta = (w.norm == "layernorm") and not no_pg
    want_dbias = (bias is not None) and not no_pg
    ref = oracle.bwd(cfg, dparts, drn, fo["residual_out"], gamma, mask,
                     fo["mean"], fo["rstd"], with_dbeta=want_dbeta,
                     with_dbias=want_dbias)
    got = gpu_bwd(w, dparts, drn, fo["residual_out"], gamma, mask,
                  fo["mean"], fo["rstd"], with_dbeta=want_dbeta,
                  with_dbias=want_dbias, offset_elems=offset_elems)
    m = mags_backward(w, dparts, drn, fo["residual_out"], gamma, fo["mean"],
                      fo["rstd"])
    dt = w.torch_dtype
    assert_close("dresidual_in", got["dresidual_in"], ref["dresidual_in"],
                 m["dres"], dt)
    assert_close("dY", got["dY"], ref["dY"], m["dY"], dt)
    assert_sum_close("dgamma", got["dgamma"], ref["dgamma"],
                     m["dgamma_terms"])
    if want_dbeta:
        assert_sum_close("dbeta", got["dbeta"], ref["dbeta"], m["dbeta_terms"])
    if want_dbias:
        assert_sum_close("dbias", got["dbias"], ref["dbias"], m["dbias_terms"])
    return got


@pytest.mark.parametrize("name", sorted(BWD_CASES))
def test_backward_matches_oracle(name):
    _run_bwd_case(BWD_CASES[name])


def test_backward_misaligned_pointers():
    _run_bwd_case(dict(base="C4", s=32, b=2, h=1024, t=4, drnext=True),
                  offset_elems=1)


def test_backward_run_twice_bitwise():
    a = _run_bwd_case(BWD_CASES["bf16_ln_h6144_t8_drnext"])
    b = _run_bwd_case(BWD_CASES["bf16_ln_h6144_t8_drnext"])
    for k in ("dresidual_in", "dY"):
        assert torch.equal(a[k], b[k])
    for k in ("dgamma", "dbeta", "dbias"):
        assert np.array_equal(a[k], b[k])


# ----------------------------------------------------------------------------
# failure detection: a bounded device wait that runs out reports, not hangs
# ----------------------------------------------------------------------------

def test_bounded_wait_reports_timeout():
    sp.sp_device_error(clear=True)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    sp.sp_debug_wait_timeout(20_000_000, status)   # 20 ms
    torch.cuda.synchronize()
    assert int(status.item()) == 1
    assert sp.sp_device_error(clear=True) == 9
    assert sp.sp_device_error(clear=False) == 0
    # the context is still usable
    x = torch.ones(16, device="cuda")
    assert float(x.sum()) == 16.0
