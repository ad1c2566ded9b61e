"""Ring attention over t context-parallel ranks (sp_ring_attention_fwd)
through the C ABI, against the CPU oracle ("Sequence Parallelism math",
section "Context parallelism and ring attention").

Tolerance.  The kernel's scores are fp32 sums of d = 128 products
accumulated in tensor memory, |ds| <= (d/16 + 16) 2^-23 scale sum_c |q_c k_c|.
The probabilities enter the second product as bf16 (relative error up to
2^-9, plus exp2's few ulps), while the normaliser l sums them in fp32, and
the output accumulates over all s keys in fp32.  So an output element passes
when

  |out - ref| <= ulp_bf16(ref) + (2^-8 + 2 max|ds| + (s/16 + 16) 2^-23) W,

W = sum_j softmax_j |v_j| (the attention-weighted mean of |v|, float64),
and the log-sum-exp when |lse - ref| <= 2 max|ds| + 1e-5 (1 + |ref|).
"""
import concurrent.futures
import gc
import math
import os

import numpy as np
import pytest
import torch

import oracle
from _parity import ulp_io

import sp_region_b200 as sp

pytestmark = pytest.mark.gpu

D = 128


@pytest.fixture(autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    oracle.build()
    yield
    gc.collect()
    torch.cuda.empty_cache()


def _qkv(b, heads, s, seed, device="cpu", k_ramp=None):
    g = torch.Generator(device=device).manual_seed(seed)
    q, k, v = (torch.randn((b, heads, s, D), generator=g, device=device)
               for _ in range(3))
    if k_ramp is not None:
        # key magnitude rising (or falling) along the sequence, so later ring
        # steps raise (or never raise) the running maximum
        k = k * k_ramp(torch.arange(s, device=device, dtype=torch.float32))[:, None]
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def _run(b, heads, s, t, scale, q, k, v):
    cfg = sp.make_cfg(s, b, heads * D, t, dtype="bf16")
    out = torch.full((b, heads, s, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((b, heads, s), float("nan"), dtype=torch.float32, device="cuda")
    sp.sp_ring_attention_fwd(cfg, heads, scale, q.cuda(), k.cuda(), v.cuda(), out, lse)
    torch.cuda.synchronize()
    assert sp.sp_device_error() == 0
    return out.cpu(), lse.cpu()


def _check(out, lse, ref, ref_lse, q, k, v, scale):
    """q, k, v, out, ref [n, s_q, D] (per head); lse, ref_lse [n, s_q]."""
    qd, kd, vd = q.double(), k.double(), v.double()
    sc = (qd @ kd.transpose(-1, -2)) * scale
    w = torch.softmax(sc, -1)
    W = (w @ vd.abs()).numpy()
    mag = (qd.abs() @ kd.abs().transpose(-1, -2)) * scale
    ds = ((D / 16 + 16) * 2.0 ** -23 * mag).amax(-1).numpy()[..., None]
    s_keys = k.shape[-2]
    r = ref.double().numpy()
    g = out.double().numpy()
    tol = ulp_io(r, torch.bfloat16) + (2.0 ** -8 + 2 * ds + (s_keys / 16 + 16) * 2.0 ** -23) * W
    bad = ~(np.abs(g - r) <= tol)
    assert not bad.any(), (f"out: {int(bad.sum())} of {bad.size} outside; first "
                           f"{np.argwhere(bad)[:3].tolist()}")
    lt = 2 * ds[..., 0] + 1e-5 * (1 + np.abs(ref_lse))
    bad = ~(np.abs(np.asarray(lse, np.float64) - ref_lse) <= lt)
    assert not bad.any(), f"lse: {int(bad.sum())} of {bad.size} outside"


CASES = [
    # name, b, heads, s, t
    ("t1", 1, 1, 256, 1),
    ("one_tile_per_rank", 1, 2, 256, 2),
    ("two_tiles_per_rank", 1, 2, 512, 2),
    ("t4_batch2", 2, 1, 1024, 4),
    ("t8", 1, 1, 1024, 8),
]


@pytest.mark.parametrize("name,b,heads,s,t", CASES, ids=[c[0] for c in CASES])
def test_ring_attention_matches_oracle(name, b, heads, s, t):
    q, k, v = _qkv(b, heads, s, 7)
    scale = D ** -0.5
    out, lse = _run(b, heads, s, t, scale, q, k, v)
    flat = lambda x: x.reshape(b * heads, s, *x.shape[3:])
    ref, ref_lse = oracle.ring_attention(flat(q), flat(k), flat(v), t, scale)
    _check(flat(out), flat(lse).numpy(), ref, ref_lse, flat(q), flat(k), flat(v), scale)


@pytest.mark.parametrize("ramp", ["rising", "falling"])
def test_ring_attention_rescales_when_the_maximum_moves(ramp):
    """Key magnitudes rising along the sequence make later ring steps raise
    every query's running maximum (the accumulated output is rescaled at
    each); falling ones never do after the first steps."""
    b, heads, s, t = 1, 1, 1024, 4
    f = (lambda x: 0.25 + 2.0 * x / s) if ramp == "rising" else (lambda x: 2.25 - 2.0 * x / s)
    q, k, v = _qkv(b, heads, s, 8, k_ramp=f)
    scale = D ** -0.5
    out, lse = _run(b, heads, s, t, scale, q, k, v)
    ref, ref_lse = oracle.ring_attention(q[0], k[0], v[0], t, scale)
    _check(out[0], lse[0].numpy(), ref, ref_lse, q[0], k[0], v[0], scale)


def test_ring_attention_rejects_what_it_does_not_take():
    q = torch.zeros((1, 1, 384, D), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    with pytest.raises(sp.SPError) as e:         # s / t = 192 is not a tile multiple
        sp.sp_ring_attention_fwd(sp.make_cfg(384, 1, D, 2), 1, 0.1, q, q, q, o)
    assert e.value.status == sp.SP_ERR_UNSUPPORTED
    with pytest.raises(sp.SPError) as e:         # head dimension 64
        sp.sp_ring_attention_fwd(sp.make_cfg(384, 1, 64, 1), 1, 0.1, q, q, q, o)
    assert e.value.status == sp.SP_ERR_UNSUPPORTED


def test_ring_attention_long_sequence_sampled():
    """The long-sequence workload's attention core: s = 32768, t = 16 ranks
    (2048 tokens each), two heads of dimension 128, at full size on the
    device; sampled query rows (both ends, both sides of every rank
    boundary, random) against the oracle."""
    b, heads, s, t = 1, 2, 32768, 16
    q, k, v = _qkv(b, heads, s, 9, device="cuda")
    scale = D ** -0.5
    cfg = sp.make_cfg(s, b, heads * D, t, dtype="bf16")
    out = torch.empty_like(q)
    lse = torch.empty((b, heads, s), dtype=torch.float32, device="cuda")
    sp.sp_ring_attention_fwd(cfg, heads, scale, q, k, v, out, lse)
    torch.cuda.synchronize()
    assert sp.sp_device_error() == 0
    per = s // t
    rows = {0, s - 1}
    for r in range(1, t):
        rows.update((r * per - 1, r * per))
    rows.update(int(x) for x in np.random.default_rng(3).integers(0, s, size=8))
    rows = sorted(rows)
    oracle.mask_words(8)   # loads the oracle library before the threads start

    def one(hd):
        qc, kc, vc = q[0, hd, rows].cpu(), k[0, hd].cpu(), v[0, hd].cpu()
        ref, ref_lse = oracle.ring_attention_rows(qc, rows, kc, vc, t, scale)
        return hd, qc, kc, vc, ref, ref_lse
    with concurrent.futures.ThreadPoolExecutor(heads) as ex:
        results = list(ex.map(one, range(heads)))
    for hd, qc, kc, vc, ref, ref_lse in results:
        _check(out[0, hd, rows].cpu()[None], lse[0, hd, rows].cpu().numpy()[None],
               ref[None], ref_lse[None], qc[None], kc[None], vc[None], scale)
