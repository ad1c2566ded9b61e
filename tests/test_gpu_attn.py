"""Ring attention over t context-parallel ranks (sp_ring_attention_fwd)
through the C ABI, against the CPU oracle ("Sequence Parallelism math",
section "Context parallelism and ring attention").

Tolerance.  The kernel's scores are fp32 sums of d = 128 products
accumulated in tensor memory, |ds| <= (d/16 + 16) 2^-23 scale sum_c |q_c k_c|.
The probabilities enter the second product as bf16 (relative error up to
2^-9, plus exp2's few ulps; one pair in 8 comes from a cubic whose relative
error is at most 7.5e-5), while the normaliser l sums them in fp32 (so l is
off by at most 7.5e-5 relative), and the output accumulates over all s keys
in fp32.  So an output element passes when

  |out - ref| <= ulp_bf16(ref) + (2^-8 + 2 max|ds| + (s/16 + 16) 2^-23) W,

W = sum_j softmax_j |v_j| (the attention-weighted mean of |v|, float64;
2^-8 covers 2^-9 + 2 * 7.5e-5), and the log-sum-exp when
|lse - ref| <= 2 max|ds| + 1e-5 (1 + |ref|) + 7.5e-5.
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
EXP2_POLY_REL = 7.5e-5   # the kernel's cubic for 2^f, f in [-1/2, 1/2]: max relative error


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


def _run_ws(b, heads, s, t, scale, q, k, v):
    """The workspace call: the units of the last round of SMs split into
    ranges of ring steps and merged."""
    cfg = sp.make_cfg(s, b, heads * D, t, dtype="bf16")
    out = torch.full((b, heads, s, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((b, heads, s), float("nan"), dtype=torch.float32, device="cuda")
    nbytes = sp.sp_ring_attention_workspace_bytes(cfg, heads)
    ws = torch.full((nbytes // 4 + 4,), float("nan"), device="cuda") if nbytes else None
    sp.sp_ring_attention_fwd_ws(cfg, heads, scale, q.cuda(), k.cuda(), v.cuda(), out, lse, ws)
    torch.cuda.synchronize()
    assert sp.sp_device_error() == 0
    return out.cpu(), lse.cpu(), nbytes


def _plan_units(b, heads, s, t):
    """The units the call runs (QT query tiles of one head each) and how many
    of them are split, as the library plans them for this GPU."""
    per = s // t
    qt = 2 if per % 256 == 0 else 1
    units = b * heads * (s // (qt * 128))
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return qt, units, units % sms


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
    lt = 2 * ds[..., 0] + 1e-5 * (1 + np.abs(ref_lse)) + EXP2_POLY_REL
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


@pytest.mark.parametrize("call", ["plain", "ws"])
def test_ring_attention_long_sequence_sampled(call):
    """The long-sequence workload's attention core: s = 32768, t = 16 ranks
    (2048 tokens each), two heads of dimension 128, at full size on the
    device; sampled query rows (both ends, both sides of every rank
    boundary, random) against the oracle.  With the workspace call (the one
    the benchmark times) the second head's rows from 5120 on belong to the
    units split over the last round of SMs."""
    b, heads, s, t = 1, 2, 32768, 16
    q, k, v = _qkv(b, heads, s, 9, device="cuda")
    scale = D ** -0.5
    cfg = sp.make_cfg(s, b, heads * D, t, dtype="bf16")
    out = torch.empty_like(q)
    lse = torch.empty((b, heads, s), dtype=torch.float32, device="cuda")
    if call == "plain":
        sp.sp_ring_attention_fwd(cfg, heads, scale, q, k, v, out, lse)
    else:
        nbytes = sp.sp_ring_attention_workspace_bytes(cfg, heads)
        ws = torch.empty(nbytes // 4 + 4, device="cuda") if nbytes else None
        sp.sp_ring_attention_fwd_ws(cfg, heads, scale, q, k, v, out, lse, ws)
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


SPLIT_CASES = CASES + [
    # every unit in the last (only) round: 8 units of two query tiles, each
    # cut into 4 ranges of 4 key tiles
    ("split4_s2048_t4", 1, 1, 2048, 4),
    ("split4_s2048_t8", 1, 1, 2048, 8),
]


@pytest.mark.parametrize("name,b,heads,s,t", SPLIT_CASES, ids=[c[0] for c in SPLIT_CASES])
def test_ring_attention_ws_matches_oracle(name, b, heads, s, t):
    """The split-and-merge call against the oracle, at the same tolerance:
    the merge applies the online-softmax update once per range."""
    q, k, v = _qkv(b, heads, s, 7)
    scale = D ** -0.5
    out, lse, nbytes = _run_ws(b, heads, s, t, scale, q, k, v)
    n_tiles = s // 128
    _, units, rem = _plan_units(b, heads, s, t)
    if rem and n_tiles >= 8:
        assert nbytes > 0, "a partly filled round with 8+ key tiles is split"
    flat = lambda x: x.reshape(b * heads, s, *x.shape[3:])
    ref, ref_lse = oracle.ring_attention(flat(q), flat(k), flat(v), t, scale)
    _check(flat(out), flat(lse).numpy(), ref, ref_lse, flat(q), flat(k), flat(v), scale)


def test_ring_attention_ws_whole_and_split_units():
    """160 units on 148 SMs: the first full round runs whole units (outputs
    bit-identical to the unsplit call), the 12 of the last round are split 8
    ways; every row of the split units and sampled rows of whole ones against
    the oracle."""
    b, heads, s, t = 1, 10, 4096, 4
    qt, units, rem = _plan_units(b, heads, s, t)
    q, k, v = _qkv(b, heads, s, 11, device="cuda")
    scale = D ** -0.5
    ref_out, ref_lse_gpu = _run(b, heads, s, t, scale, q, k, v)
    out, lse, nbytes = _run_ws(b, heads, s, t, scale, q, k, v)
    rows_per_unit, nx = qt * 128, s // (qt * 128)
    full = units - rem if nbytes else units
    if nbytes:
        assert rem > 0
    # whole units: the same kernel path, the same bits
    for u in range(full):
        hd, r0 = u // nx, (u % nx) * rows_per_unit
        assert torch.equal(out[0, hd, r0:r0 + rows_per_unit], ref_out[0, hd, r0:r0 + rows_per_unit])
        assert torch.equal(lse[0, hd, r0:r0 + rows_per_unit], ref_lse_gpu[0, hd, r0:r0 + rows_per_unit])
    # split units (and three sampled rows of each head's first unit)
    by_head = {}
    for u in range(full, units):
        hd, r0 = u // nx, (u % nx) * rows_per_unit
        by_head.setdefault(hd, set()).update(range(r0, r0 + rows_per_unit))
    for hd in range(heads):
        by_head.setdefault(hd, set()).update((0, 77, rows_per_unit - 1))
    oracle.mask_words(8)   # loads the oracle library before the threads start

    def one(hd):
        rows = sorted(by_head[hd])
        qc, kc, vc = q[0, hd, rows].cpu(), k[0, hd].cpu(), v[0, hd].cpu()
        r, rl = oracle.ring_attention_rows(qc, rows, kc, vc, t, scale)
        return hd, rows, qc, kc, vc, r, rl
    with concurrent.futures.ThreadPoolExecutor(min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(one, sorted(by_head)))
    for hd, rows, qc, kc, vc, r, rl in results:
        _check(out[0, hd, rows][None], lse[0, hd, rows].numpy()[None], r[None], rl[None],
               qc[None], kc[None], vc[None], scale)


def test_ring_attention_ws_rejects_a_short_workspace():
    b, heads, s, t = 1, 1, 2048, 4
    cfg = sp.make_cfg(s, b, heads * D, t, dtype="bf16")
    nbytes = sp.sp_ring_attention_workspace_bytes(cfg, heads)
    assert nbytes > 0
    q = torch.zeros((b, heads, s, D), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    for ws in (None, torch.empty(nbytes // 4 - 4, device="cuda")):
        with pytest.raises(sp.SPError) as e:
            sp.sp_ring_attention_fwd_ws(cfg, heads, 0.1, q, q, q, o, None, ws)
        assert e.value.status == sp.SP_ERR_INVALID_ARG
    # the shapes the plain call rejects, this one rejects too
    with pytest.raises(sp.SPError) as e:
        sp.sp_ring_attention_workspace_bytes(sp.make_cfg(384, 1, D, 2), 1)
    assert e.value.status == sp.SP_ERR_UNSUPPORTED


def test_ring_attention_ws_without_lse():
    """The workspace call with no log-sum-exp output: the split units' merge
    skips it and writes the same output bits as with it."""
    b, heads, s, t = 1, 10, 4096, 4   # 160 units: whole and split ones
    q, k, v = _qkv(b, heads, s, 12, device="cuda")
    cfg = sp.make_cfg(s, b, heads * D, t, dtype="bf16")
    nbytes = sp.sp_ring_attention_workspace_bytes(cfg, heads)
    ws = torch.empty(nbytes // 4 + 4, device="cuda") if nbytes else None
    out1 = torch.empty_like(q)
    lse = torch.empty((b, heads, s), dtype=torch.float32, device="cuda")
    sp.sp_ring_attention_fwd_ws(cfg, heads, D ** -0.5, q, k, v, out1, lse, ws)
    out2 = torch.full_like(q, float("nan"))
    sp.sp_ring_attention_fwd_ws(cfg, heads, D ** -0.5, q, k, v, out2, None, ws)
    torch.cuda.synchronize()
    assert sp.sp_device_error() == 0
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
