"""The GPU parity checker itself, on CPU: it must accept the oracle's own
outputs, accept a stored residual sum one ulp from the oracle's when the norm
output follows that sum, and reject a norm output that does not."""
import numpy as np
import pytest
import torch

import oracle
import sp_synth
from _parity import check_forward


def _case(norm):
    w = sp_synth.WORKLOADS["C2"].replace(s=32, b=2, h=256, t=4, norm=norm,
                                          has_beta=norm == "layernorm")
    parts = sp_synth.draw_partials(w)
    res = sp_synth.draw_residual(w)
    bias, gamma, beta = sp_synth.draw_params(w)
    ref = oracle.fwd(oracle.cfg_from(w), parts, bias, res, gamma, beta)
    return w, parts, bias, res, gamma, beta, ref


def _as_got(ref):
    return dict(residual_out=ref["residual_out"].clone(),
                gathered=[ref["gathered"][0].clone()], mask=ref["mask"].copy(),
                mean=None if ref["mean"] is None else ref["mean"].astype(np.float32),
                rstd=ref["rstd"].astype(np.float32))


def _nudge_row(w, got, gamma, beta, row):
    """Move one stored sum of `row` by one bf16 ulp and renormalise that row
    with the oracle, as a kernel whose fp32 sum rounded a near-tie the other
    way would."""
    x = got["residual_out"]
    bits = x[row, 3:4].view(torch.int16)
    x[row, 3:4] = (bits + 1).view(torch.bfloat16)
    cfg = oracle.cfg_from(w, s=1, b=1, t=1)
    alt = oracle.norm_ag_fwd(cfg, x[row:row + 1].contiguous(), gamma, beta)
    got["gathered"][0][row] = alt["gathered"][0][0]
    got["rstd"][row] = alt["rstd"][0]
    if got["mean"] is not None:
        got["mean"][row] = alt["mean"][0]


@pytest.mark.parametrize("norm", ["layernorm", "rmsnorm"])
def test_checker_accepts_the_oracle(norm):
    w, parts, bias, res, gamma, beta, ref = _case(norm)
    check_forward(w, _as_got(ref), ref, parts, bias, res, gamma, beta)


@pytest.mark.parametrize("norm", ["layernorm", "rmsnorm"])
def test_checker_follows_a_stored_sum_one_ulp_away(norm):
    w, parts, bias, res, gamma, beta, ref = _case(norm)
    got = _as_got(ref)
    _nudge_row(w, got, gamma, beta, 5)
    check_forward(w, got, ref, parts, bias, res, gamma, beta)


def test_checker_rejects_a_norm_output_two_ulps_off():
    w, parts, bias, res, gamma, beta, ref = _case("layernorm")
    got = _as_got(ref)
    o = got["gathered"][0]
    bits = o[7, 11:12].view(torch.int16)
    o[7, 11:12] = (bits + 2).view(torch.bfloat16)
    with pytest.raises(AssertionError, match="gathered"):
        check_forward(w, got, ref, parts, bias, res, gamma, beta)

