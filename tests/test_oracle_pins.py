"""Pins of the CPU oracle to things other than itself.

Each test checks the oracle against a value the pages print, a closed form, a
library routine, an invariant the method guarantees, or brute force.  They run
without a GPU.
"""
import ctypes
import ctypes.util
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import sp_synth
from _golden import load

pytestmark = pytest.mark.filterwarnings("ignore")


# ----------------------------------------------------------------------------
# Philox4x32-10 against cuRAND's host-side Philox4_32_10 generator
# ----------------------------------------------------------------------------

def _curand():
    for cand in ("/usr/local/cuda/lib64/libcurand.so",
                 ctypes.util.find_library("curand")):
        if cand and os.path.exists(cand):
            return ctypes.CDLL(cand)
    return None


def _curand_blocks(lib, seed, nwords):
    g = ctypes.c_void_p()
    assert lib.curandCreateGeneratorHost(ctypes.byref(g), 161) == 0
    try:
        assert lib.curandSetPseudoRandomGeneratorSeed(
            g, ctypes.c_ulonglong(seed)) == 0
        out = np.zeros(nwords, dtype=np.uint32)
        assert lib.curandGenerate(g, out.ctypes.data_as(ctypes.c_void_p),
                                  ctypes.c_size_t(nwords)) == 0
    finally:
        lib.curandDestroyGenerator(g)
    return out


def test_philox_matches_curand_host_generator(orc):
    """cuRAND's host Philox4_32_10 generator (CPU code, a library routine)
    writes output block m = Philox(counter=(m // 65536, 0, m % 65536, 0),
    key=(seed lo, seed hi)).  Comparing block by block exercises the round
    function, both key words and the key schedule, and two counter words."""
    lib = _curand()
    if lib is None:
        pytest.skip("libcurand not present")
    blocks = [0, 1, 2, 3, 17, 255, 4096, 65535, 65536, 65537, 65536 * 2 + 9]
    for seed in (0, 1, 0xDEADBEEF, 0x0123456789ABCDEF, 2**64 - 1):
        out = _curand_blocks(lib, seed, 4 * (max(blocks) + 1))
        key = [seed & 0xFFFFFFFF, seed >> 32]
        for m in blocks:
            ref = [int(v) for v in out[4 * m:4 * m + 4]]
            got = orc.philox([m // 65536, 0, m % 65536, 0], key)
            assert got == ref, (seed, m)


def test_philox_counter_words_all_matter(orc):
    """Every counter word and key word changes the output (a dropped word in
    the round function would leave one of them without effect)."""
    base = orc.philox([1, 2, 3, 4], [5, 6])
    for i in range(4):
        c = [1, 2, 3, 4]
        c[i] ^= 1
        assert orc.philox(c, [5, 6]) != base
    for i in range(2):
        k = [5, 6]
        k[i] ^= 1
        assert orc.philox([1, 2, 3, 4], k) != base


# ----------------------------------------------------------------------------
# rounding to the I/O dtype
# ----------------------------------------------------------------------------

def _rand_f32_bits(n, seed):
    rng = np.random.default_rng(seed)
    bits = rng.integers(0, 2**32, size=n, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    return x[np.isfinite(x)]


def test_bf16_rounding_matches_torch(orc):
    """torch's float32 -> bfloat16 conversion is round-to-nearest-even; every
    float32 is exactly a double, so the two must agree bit for bit, including
    exact ties (low 16 bits = 0x8000) and subnormals."""
    x = _rand_f32_bits(20000, 1)
    rng = np.random.default_rng(2)
    ties = (rng.integers(0, 2**16, size=4000).astype(np.uint32) << 16
            | np.uint32(0x8000)).view(np.float32)
    ties = ties[np.isfinite(ties)]
    sub = (rng.integers(1, 2**23, size=2000).astype(np.uint32)).view(np.float32)
    vals = np.concatenate([x, ties, sub, np.float32([65504.0, 3.3895314e38,
                                                     -3.3895314e38, 1e-40])])
    ref = torch.from_numpy(vals.copy()).to(torch.bfloat16).to(torch.float64)
    got = np.array([orc.round_to(float(v), "bf16") for v in vals])
    r = ref.numpy()
    same = (got == r) | (np.isnan(got) & np.isnan(r))
    assert same.all(), vals[~same][:5]


def test_f32_rounding_matches_numpy_cast(orc):
    """numpy's float64 -> float32 cast is IEEE round-to-nearest-even."""
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(5000) * 10.0 ** rng.integers(
        -40, 38, size=5000), [1.0 + 2.0 ** -24, 1.0 + 3 * 2.0 ** -24,
                              2.0 ** -149 * 1.5, 3.4028235677973366e38]])
    got = np.array([orc.round_to(float(v), "f32") for v in x])
    ref = x.astype(np.float32).astype(np.float64)
    assert (got == ref).all()


def test_bf16_hand_ties(orc):
    """Ties from the definition: 1 + 2^-8 is halfway between 1 and 1 + 2^-7
    and goes to the even significand (1); 1 + 3*2^-8 goes up to 1 + 2^-6."""
    assert orc.round_to(1.0 + 2.0 ** -8, "bf16") == 1.0
    assert orc.round_to(1.0 + 3 * 2.0 ** -8, "bf16") == 1.0 + 2.0 ** -6
    assert orc.round_to(-(1.0 + 2.0 ** -8 + 2.0 ** -30), "bf16") == \
        -(1.0 + 2.0 ** -7)


# ----------------------------------------------------------------------------
# dropout
# ----------------------------------------------------------------------------

def test_drop_threshold_closed_form(orc):
    assert orc.drop_threshold(0.0) == 0
    assert orc.drop_threshold(0.5) == 2 ** 31
    assert orc.drop_threshold(0.25) == 2 ** 30
    assert orc.drop_threshold(0.1) == math.floor(
        float(np.float32(0.1)) * 2 ** 32)


def test_keep_rate_binomial(orc):
    """The keep rate over many draws is within 6 sigma of (1 - p)."""
    w = sp_synth.WORKLOADS["C1"].replace(s=64, b=2, h=512, t=2)
    cfg = orc.cfg_from(w)
    parts = sp_synth.draw_partials(w)
    bias, gamma, beta = sp_synth.draw_params(w)
    res = sp_synth.draw_residual(w)
    out = orc.fwd(cfg, parts, bias, res, gamma, beta)
    bits = np.unpackbits(out["mask"].view(np.uint8)).sum()
    n = w.rows * w.h
    p = float(np.float32(w.p_drop))
    mu, sd = n * (1 - p), math.sqrt(n * p * (1 - p))
    assert abs(bits - mu) < 6 * sd


def test_inverted_dropout_preserves_the_expectation(orc):
    """Inverted dropout keeps E[z] = y: with a constant reduced sum c, zero
    bias and zero residual, the mean of the stored sums over many elements is
    c within 6 sigma of the binomial noise."""
    w = sp_synth.WORKLOADS["C1"].replace(s=64, b=2, h=512, t=2, p_drop=0.4)
    cfg = orc.cfg_from(w)
    c = 0.5
    parts = [torch.full((w.rows, w.h), c / 2), torch.full((w.rows, w.h),
                                                          c / 2)]
    out = orc.fwd(cfg, parts, torch.zeros(w.h), torch.zeros((w.rows, w.h)),
                  torch.ones(w.h), torch.zeros(w.h))
    z = out["residual_out"].double()
    n = z.numel()
    p = float(np.float32(w.p_drop))
    sd = c / (1 - p) * math.sqrt(p * (1 - p) / n)
    assert abs(float(z.mean()) - c) < 6 * sd
    kept = z[z != 0]
    assert torch.allclose(kept, torch.full_like(kept, c / (1 - p)),
                          rtol=1e-7)


def test_keep_words_follow_curand_stream_on_row_zero(orc):
    """Row 0 with offset 0 uses counter (j >> 2, 0, 0, 0), which cuRAND's host
    Philox4_32_10 generator emits as block (j >> 2) * 65536; feature j takes
    word j & 3 of it and is kept iff that word is >= floor(p * 2^32)."""
    lib = _curand()
    if lib is None:
        pytest.skip("libcurand not present")
    h = 24
    seed = 0x5EED
    words = _curand_blocks(lib, seed, 4 * ((h // 4 - 1) * 65536 + 1))
    p = 0.3
    thr = orc.drop_threshold(p)
    for j in range(h):
        u = int(words[4 * 65536 * (j >> 2) + (j & 3)])
        assert orc.keep(seed, 0, 0, j, p) == (u >= thr), j


def test_mask_marks_exactly_the_zeroed_outputs(orc):
    """With zero residual and zero bias, an element of the stored residual
    sum is zero exactly where dropout removed it; the packed bit j of row n is
    bit (j & 31) of word n*W + (j >> 5), least significant bit first."""
    w = sp_synth.WORKLOADS["C1"].replace(s=6, b=1, h=70, t=3, p_drop=0.3)
    cfg = orc.cfg_from(w)
    parts = [p + 2.0 for p in sp_synth.draw_partials(w)]   # sums never 0
    zeros = torch.zeros((w.rows, w.h))
    out = orc.fwd(cfg, parts, torch.zeros(w.h), zeros, torch.ones(w.h),
                  torch.zeros(w.h))
    rout = out["residual_out"].numpy()
    mask = out["mask"]
    W = (w.h + 31) // 32
    assert mask.shape == (w.rows, W)
    for n in range(w.rows):
        for j in range(w.h):
            bit = (int(mask[n, j >> 5]) >> (j & 31)) & 1
            assert bit == (rout[n, j] != 0.0)
        # padding bits of the last word are zero
        assert int(mask[n, W - 1]) >> (w.h - 32 * (W - 1)) == 0


def test_p_zero_is_identity(orc):
    """p = 0 keeps everything and scales by exactly 1: the stored residual sum
    is the rounded sum of residual, bias and the reduced partials, computed
    here in float64 by torch."""
    w = sp_synth.WORKLOADS["C1"].replace(s=8, b=2, h=40, t=4, p_drop=0.0)
    cfg = orc.cfg_from(w)
    parts = sp_synth.draw_partials(w)
    bias, gamma, beta = sp_synth.draw_params(w)
    res = sp_synth.draw_residual(w)
    out = orc.fwd(cfg, parts, bias, res, gamma, beta)
    assert (np.unpackbits(out["mask"].view(np.uint8)).reshape(
        w.rows, -1)[:, :w.h].all())
    tot = torch.stack([p.double() for p in parts]).sum(0)
    ref = (res.double() + (tot + bias.double())).float()
    assert torch.equal(out["residual_out"], ref)


# ----------------------------------------------------------------------------
# reduce-scatter / all-gather
# ----------------------------------------------------------------------------

def test_worked_layout_4_plus_5(orc):
    """The 4 x 4, two-GPU layout: rank 0 owns t0, t1 and rank 1 owns t2, t3;
    token t0's first feature reduces 4 + 5 to 9 on rank 0."""
    g = load("worked_layout_2gpu.txt")
    w = sp_synth.WORKLOADS["C1"]
    assert (w.s * w.b, w.h, w.t) == (g["tokens"], g["features"], g["gpus"])
    parts = sp_synth.draw_partials(w)
    assert float(parts[0][0, 0]) == g["t0_f0_partial_gpu0"]
    assert float(parts[1][0, 0]) == g["t0_f0_partial_gpu1"]
    rs0 = orc.reduce_scatter(parts, 0)
    rs1 = orc.reduce_scatter(parts, 1)
    assert rs0.shape == (2, 4) and rs1.shape == (2, 4)
    assert rs0[0, 0] == g["t0_f0_reduced"]
    ar = orc.all_reduce(parts)
    # rank r's shard holds exactly its tokens, whole feature vectors
    for r, toks in ((0, g["gpu0_tokens"]), (1, g["gpu1_tokens"])):
        shard = rs0 if r == 0 else rs1
        for i, tok in enumerate(toks):
            assert np.array_equal(shard[i], ar[int(tok)])


@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_rs_then_ag_equals_all_reduce(orc, t):
    """All-gather of the reduce-scatter shards is the all-reduce, bit for
    bit (same summation order)."""
    w = sp_synth.WORKLOADS["C2"].replace(s=16, b=3, h=24, t=t)
    parts = sp_synth.draw_partials(w)
    shards = [orc.reduce_scatter(parts, r) for r in range(t)]
    assert np.array_equal(orc.all_gather(shards), orc.all_reduce(parts))


def test_ring_volume_worked_example(orc):
    g = load("ring_volume_t8.txt")
    t = int(g["t"])
    assert orc.ring_bytes(t, "all_reduce", 1.0) == g["all_reduce"]
    assert orc.ring_bytes(t, "all_gather", 1.0) == g["all_gather"]
    assert orc.ring_bytes(t, "reduce_scatter", 1.0) == g["reduce_scatter"]
    assert 2 * orc.ring_bytes(t, "all_reduce", 1.0) == g["per_layer_tp"]
    assert (2 * orc.ring_bytes(t, "all_gather", 1.0)
            + 2 * orc.ring_bytes(t, "reduce_scatter", 1.0)) == g["per_layer_sp"]


# ----------------------------------------------------------------------------
# t-invariance
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("norm", ["layernorm", "rmsnorm"])
def test_outputs_do_not_depend_on_t(orc, norm):
    """The norm and the dropout act on each token alone, so the result is the
    same for every sharding degree when the partial sums add exactly."""
    base = sp_synth.WORKLOADS["C2"].replace(s=16, b=2, h=48, norm=norm,
                                             has_beta=norm == "layernorm")
    atoms = sp_synth.dyadic_atoms(base.rows, base.h, seed=11)
    ref = None
    for t in (1, 2, 4, 8, 16):
        w = base.replace(t=t)
        parts = sp_synth.group_atoms(atoms, t, w.torch_dtype)
        bias, gamma, beta = sp_synth.draw_params(w)
        res = sp_synth.draw_residual(w)
        out = orc.fwd(orc.cfg_from(w), parts, bias, res, gamma, beta)
        cur = (out["residual_out"], out["gathered"][0], out["mask"],
               out["rstd"])
        if ref is None:
            ref = cur
        else:
            assert torch.equal(cur[0], ref[0])
            assert torch.equal(cur[1], ref[1])
            assert np.array_equal(cur[2], ref[2])
            assert np.array_equal(cur[3], ref[3])


# ----------------------------------------------------------------------------
# norms against torch (library) in float64
# ----------------------------------------------------------------------------

def _ulp_bf16(x):
    x = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(x, 2.0 ** -126)))
    return 2.0 ** (e - 7)


@pytest.mark.parametrize("norm", ["layernorm", "rmsnorm"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_norm_matches_torch_functional(orc, norm, dtype):
    w = sp_synth.WORKLOADS["C2"].replace(s=12, b=2, h=96, t=4, norm=norm,
                                          dtype=dtype,
                                          has_beta=norm == "layernorm")
    cfg = orc.cfg_from(w)
    parts = sp_synth.draw_partials(w)
    bias, gamma, beta = sp_synth.draw_params(w)
    res = sp_synth.draw_residual(w)
    out = orc.fwd(cfg, parts, bias, res, gamma, beta)
    x = out["residual_out"].double()
    eps = float(np.float32(w.eps))
    if norm == "layernorm":
        ref = F.layer_norm(x, (w.h,), gamma.double(), beta.double(), eps)
        var, mean = torch.var_mean(x, dim=1, unbiased=False)
        assert np.allclose(out["mean"], mean.numpy(), rtol=1e-13, atol=1e-13)
        assert np.allclose(out["rstd"], (1 / torch.sqrt(var + eps)).numpy(),
                           rtol=1e-12)
    else:
        ref = F.rms_norm(x, (w.h,), gamma.double(), eps)
        ms = (x * x).mean(1)
        assert np.allclose(out["rstd"], (1 / torch.sqrt(ms + eps)).numpy(),
                           rtol=1e-12)
    got = out["gathered"][0].double().numpy()
    r = ref.numpy()
    if dtype == "f32":
        assert np.allclose(got, r, rtol=2 ** -23, atol=1e-30)
    else:
        assert (np.abs(got - r) <= _ulp_bf16(r) * 0.5 + 1e-300).all()


def test_layernorm_constant_row_gives_beta(orc):
    w = sp_synth.WORKLOADS["C1"].replace(s=2, b=1, h=16, t=1, p_drop=0.0)
    cfg = orc.cfg_from(w)
    parts = [torch.full((2, 16), 0.75)]
    bias, gamma, beta = sp_synth.draw_params(w)
    out = orc.fwd(cfg, parts, torch.zeros(16), torch.zeros((2, 16)), gamma,
                  beta)
    assert torch.equal(out["gathered"][0][0], beta)
    assert out["mean"][0] == 0.75


def test_rmsnorm_constant_row_closed_form(orc):
    w = sp_synth.WORKLOADS["C3"].replace(s=1, b=1, h=8, t=1, dtype="f32")
    cfg = orc.cfg_from(w)
    c = 0.375
    gamma = torch.linspace(0.5, 2.0, 8)
    out = orc.fwd(cfg, [torch.full((1, 8), c)], None, torch.zeros((1, 8)),
                  gamma, None)
    eps = float(np.float32(w.eps))
    ref = c / math.sqrt(c * c + eps) * gamma.double()
    assert np.allclose(out["gathered"][0][0].double().numpy(), ref.numpy(),
                       rtol=2 ** -23)


def test_layernorm_moments_with_unit_affine(orc):
    """With gamma = 1 and beta = 0 the normalised row has mean 0 and variance
    var / (var + eps)."""
    w = sp_synth.WORKLOADS["C1"].replace(s=4, b=1, h=256, t=2, p_drop=0.0)
    cfg = orc.cfg_from(w)
    parts = sp_synth.draw_partials(w)
    res = sp_synth.draw_residual(w)
    out = orc.fwd(cfg, parts, torch.zeros(w.h), res, torch.ones(w.h),
                  torch.zeros(w.h))
    o = out["gathered"][0].double()
    x = out["residual_out"].double()
    var = x.var(1, unbiased=False)
    eps = float(np.float32(w.eps))
    assert torch.allclose(o.mean(1), torch.zeros(4, dtype=torch.float64),
                          atol=1e-6)
    assert torch.allclose(o.var(1, unbiased=False), var / (var + eps),
                          rtol=1e-6)


# ----------------------------------------------------------------------------
# backward against torch autograd (float64) and finite differences
# ----------------------------------------------------------------------------

def _torch_reference_grads(w, parts_y, bias, x, gamma, beta, mask_bits, dn,
                           drnext):
    """Reverse-mode through bias, dropout, residual add and the norm, by
    torch autograd in float64, evaluated at the stored residual sum x."""
    h = w.h
    keep = torch.from_numpy(np.unpackbits(
        mask_bits.view(np.uint8), bitorder="little").reshape(
            w.rows, -1)[:, :h].astype(np.float64))
    scale = 1.0 / (1.0 - float(np.float32(w.p_drop)))
    y = parts_y.clone().requires_grad_(True)
    bvar = (bias.double().clone().requires_grad_(True) if bias is not None
            else torch.zeros(h, dtype=torch.float64))
    g = gamma.double().clone().requires_grad_(True)
    be = (beta.double().clone().requires_grad_(True) if beta is not None
          else None)
    z = (y + bvar) * keep * scale
    resid = (x.double() - z.detach()).requires_grad_(True)
    r = resid + z
    eps = float(np.float32(w.eps))
    if w.norm == "layernorm":
        o = F.layer_norm(r, (h,), g, be, eps)
    else:
        o = F.rms_norm(r, (h,), g, eps)
    L = (o * dn).sum()
    if drnext is not None:
        L = L + (r * drnext.double()).sum()
    L.backward()
    return dict(dresidual_in=resid.grad, dY=y.grad, dgamma=g.grad,
                dbeta=None if be is None else be.grad,
                dbias=bvar.grad if bias is not None else None)


@pytest.mark.parametrize("norm", ["layernorm", "rmsnorm"])
@pytest.mark.parametrize("with_drnext", [False, True])
def test_backward_matches_torch_autograd(orc, norm, with_drnext):
    w = sp_synth.WORKLOADS["C2"].replace(s=8, b=2, h=40, t=4, norm=norm,
                                          dtype="f32", p_drop=0.25,
                                          has_beta=norm == "layernorm")
    cfg = orc.cfg_from(w)
    parts = sp_synth.draw_partials(w)
    bias, gamma, beta = sp_synth.draw_params(w)
    res = sp_synth.draw_residual(w)
    fo = orc.fwd(cfg, parts, bias, res, gamma, beta)
    dparts = sp_synth.draw_grad_partials(w)
    drn = sp_synth.draw_residual_grad(w) if with_drnext else None
    bo = orc.bwd(cfg, dparts, drn, fo["residual_out"], gamma, fo["mask"],
                 fo["mean"], fo["rstd"], with_dbeta=beta is not None)
    dn = torch.stack([d.double() for d in dparts]).sum(0)
    y = torch.stack([p.double() for p in parts]).sum(0)
    ref = _torch_reference_grads(w, y, bias, fo["residual_out"], gamma, beta,
                                 fo["mask"], dn, drn)
    for k in ("dresidual_in", "dY"):
        assert torch.allclose(bo[k].double(), ref[k], rtol=1e-6, atol=1e-6), k
    for k in ("dgamma", "dbeta", "dbias"):
        if ref[k] is None:
            continue
        assert np.allclose(bo[k], ref[k].numpy(), rtol=1e-10, atol=1e-10), k


def test_backward_finite_differences(orc):
    """Central differences of L = sum(dn * norm_out) + sum(drnext * r) in
    double, on a tiny fp32 problem with the dropout mask held fixed."""
    w = sp_synth.WORKLOADS["C1"].replace(s=2, b=2, h=8, t=2, p_drop=0.3)
    cfg = orc.cfg_from(w)
    parts = sp_synth.draw_partials(w)
    bias, gamma, beta = sp_synth.draw_params(w)
    res = sp_synth.draw_residual(w)
    fo = orc.fwd(cfg, parts, bias, res, gamma, beta)
    dparts = sp_synth.draw_grad_partials(w)
    drn = sp_synth.draw_residual_grad(w)
    bo = orc.bwd(cfg, dparts, drn, fo["residual_out"], gamma, fo["mask"],
                 fo["mean"], fo["rstd"])
    dn = torch.stack([d.double() for d in dparts]).sum(0)
    keep = np.unpackbits(fo["mask"].view(np.uint8), bitorder="little")
    keep = keep.reshape(w.rows, -1)[:, :w.h].astype(np.float64)
    scale = 1.0 / (1.0 - float(np.float32(w.p_drop)))
    y0 = torch.stack([p.double() for p in parts]).sum(0).numpy()
    x0 = fo["residual_out"].double().numpy()
    resid0 = x0 - (y0 + bias.double().numpy()) * keep * scale
    gam = gamma.double().numpy()
    bet = beta.double().numpy()
    eps = float(np.float32(w.eps))

    def loss(y, resid, gm, bt, bs):
        r = resid + (y + bs) * keep * scale
        mu = r.mean(1, keepdims=True)
        var = ((r - mu) ** 2).mean(1, keepdims=True)
        o = (r - mu) / np.sqrt(var + eps) * gm + bt
        return float((o * dn.numpy()).sum() + (r * drn.double().numpy()).sum())

    hstep = 1e-6
    args = [y0, resid0, gam, bet, bias.double().numpy()]
    names = ["dY", "dresidual_in", "dgamma", "dbeta", "dbias"]
    for ai, name in enumerate(names):
        base = args[ai]
        num = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            a_p = [a.copy() for a in args]
            a_m = [a.copy() for a in args]
            a_p[ai][idx] += hstep
            a_m[ai][idx] -= hstep
            num[idx] = (loss(*a_p) - loss(*a_m)) / (2 * hstep)
        got = bo[name]
        got = got.double().numpy() if isinstance(got, torch.Tensor) else got
        assert np.allclose(got, num, rtol=1e-5, atol=1e-5), name


def test_backward_layernorm_invariants(orc):
    """LayerNorm's input gradient sums to zero over each row (shift
    invariance) and is orthogonal to the normalised row (scale invariance,
    up to eps); with p = 0 and no residual-stream gradient the gathered
    gradient equals the residual gradient."""
    w = sp_synth.WORKLOADS["C2"].replace(s=8, b=1, h=64, t=2, dtype="f32",
                                          p_drop=0.0)
    cfg = orc.cfg_from(w)
    parts = sp_synth.draw_partials(w)
    bias, gamma, beta = sp_synth.draw_params(w)
    res = sp_synth.draw_residual(w)
    fo = orc.fwd(cfg, parts, bias, res, gamma, beta)
    dparts = sp_synth.draw_grad_partials(w)
    bo = orc.bwd(cfg, dparts, None, fo["residual_out"], gamma, fo["mask"],
                 fo["mean"], fo["rstd"])
    dx = bo["dresidual_in"].double()
    x = fo["residual_out"].double()
    xhat = (x - torch.from_numpy(fo["mean"])[:, None]) * torch.from_numpy(
        fo["rstd"])[:, None]
    assert torch.allclose(dx.sum(1), torch.zeros(8, dtype=torch.float64),
                          atol=1e-5)
    assert torch.allclose((dx * xhat).sum(1),
                          torch.zeros(8, dtype=torch.float64), atol=1e-3)
    assert torch.equal(bo["dY"], bo["dresidual_in"])


def test_backward_rows_agrees_with_full(orc):
    w = sp_synth.WORKLOADS["C2"].replace(s=8, b=2, h=32, t=4)
    cfg = orc.cfg_from(w)
    parts = sp_synth.draw_partials(w)
    bias, gamma, beta = sp_synth.draw_params(w)
    res = sp_synth.draw_residual(w)
    fo = orc.fwd(cfg, parts, bias, res, gamma, beta)
    dparts = sp_synth.draw_grad_partials(w)
    bo = orc.bwd(cfg, dparts, None, fo["residual_out"], gamma, fo["mask"],
                 fo["mean"], fo["rstd"])
    rows = [0, 5, 15]
    br = orc.bwd_rows(cfg, [d[rows] for d in dparts], None,
                      fo["residual_out"][rows], gamma, fo["mask"][rows],
                      fo["mean"][rows], fo["rstd"][rows])
    assert torch.equal(br["dresidual_in"], bo["dresidual_in"][rows])
    assert torch.equal(br["dY"], bo["dY"][rows])
    fr = orc.fwd_rows(cfg, rows, [p[rows] for p in parts], bias, res[rows],
                      gamma, beta)
    assert torch.equal(fr["residual_out"], fo["residual_out"][rows])
    assert torch.equal(fr["norm_out"], fo["gathered"][0][rows])
    assert np.array_equal(fr["mask"], fo["mask"][rows])


@pytest.mark.parametrize("norm", ["layernorm", "rmsnorm"])
def test_backward_rows_parameter_shares_match_autograd(orc, norm):
    """The rows' shares of dgamma / dbeta / dbias: each chunk's share equals
    torch autograd's parameter gradient of the loss over that chunk's rows
    alone, and the shares of a partition of all rows add up to autograd's
    full gradient (float64)."""
    w = sp_synth.WORKLOADS["C2"].replace(s=12, b=2, h=48, t=4, norm=norm,
                                          dtype="f32", p_drop=0.25,
                                          has_beta=norm == "layernorm")
    cfg = orc.cfg_from(w)
    parts = sp_synth.draw_partials(w)
    bias, gamma, beta = sp_synth.draw_params(w)
    res = sp_synth.draw_residual(w)
    fo = orc.fwd(cfg, parts, bias, res, gamma, beta)
    dparts = sp_synth.draw_grad_partials(w)
    dn = torch.stack([d.double() for d in dparts]).sum(0)
    y = torch.stack([p.double() for p in parts]).sum(0)
    chunks = [list(range(0, 7)), list(range(7, 8)), list(range(8, 24))]
    total = {k: np.zeros(w.h) for k in ("dgamma", "dbeta", "dbias")}
    for rows in chunks:
        sh = orc.bwd_rows(cfg, [d[rows] for d in dparts], None,
                          fo["residual_out"][rows], gamma, fo["mask"][rows],
                          None if fo["mean"] is None else fo["mean"][rows],
                          fo["rstd"][rows], with_params=True)
        only = torch.zeros_like(dn)
        only[rows] = dn[rows]      # the loss restricted to this chunk
        ref = _torch_reference_grads(w, y, bias, fo["residual_out"], gamma,
                                     beta, fo["mask"], only, None)
        for k in total:
            if ref[k] is None:
                continue
            assert np.allclose(sh[k], ref[k].numpy(), rtol=1e-10,
                               atol=1e-12), (k, rows)
            total[k] += sh[k]
    full = _torch_reference_grads(w, y, bias, fo["residual_out"], gamma, beta,
                                  fo["mask"], dn, None)
    for k in total:
        if full[k] is not None:
            assert np.allclose(total[k], full[k].numpy(), rtol=1e-10,
                               atol=1e-12), k


# ----------------------------------------------------------------------------
# activation-memory closed forms
# ----------------------------------------------------------------------------

def test_activation_worked_example(orc):
    g = load("activation_worked_example.txt")
    s, b, h, a, t = (int(g[k]) for k in ("s", "b", "h", "a", "t"))
    bpe = g["bytes_per_elem"]
    sbh = s * b * h
    assert 5 * a * s / h == g["attn_coeff"]
    assert f"{sbh:.{int(g['sbh_sig']) - 1}e}" == f"{g['sbh']:.3e}"
    tp = orc.activation_bytes(s, b, h, a, t, 1, bpe)
    tpsp = orc.activation_bytes(s, b, h, a, t, 2, bpe)
    assert tp / (sbh * bpe) == g["tp_coeff"]
    assert tpsp / (sbh * bpe) == g["tpsp_coeff"]
    assert round(tp / 1e9, 2) == g["tp_gb"]
    assert round(tpsp / 1e9, 2) == g["tpsp_gb"]
    assert round(100 * (1 - tpsp / tp)) == g["reduction_pct"]
    assert round((tp - tpsp) / 1e9, 2) == g["saved_gb_per_layer"]
    assert abs(g["layers"] * (tp - tpsp) / 1e9 - g["saved_gb_stack"]) < 5


def test_activation_identities(orc):
    for (s, b, h, a) in [(2048, 4, 12288, 96), (32768, 1, 12288, 96),
                         (4096, 2, 8192, 64)]:
        sbh = s * b * h
        full = orc.activation_bytes(s, b, h, a, 1, 0, 1.0)
        # t = 1 collapses every formula to the single-device one
        assert orc.activation_bytes(s, b, h, a, 1, 1, 1.0) == full
        assert orc.activation_bytes(s, b, h, a, 1, 2, 1.0) == full
        for t in (2, 4, 8, 16):
            tp = orc.activation_bytes(s, b, h, a, t, 1, 1.0)
            sp = orc.activation_bytes(s, b, h, a, t, 2, 1.0)
            assert math.isclose(sp, full / t, rel_tol=1e-15)
            # the gap is the replicated 10*sbh band, now divided by t
            assert math.isclose(tp - sp, 10 * sbh * (1 - 1 / t),
                                rel_tol=1e-12)


def test_activation_long_sequence_coefficients(orc):
    """s = 32768, h = 12288, a = 96: 5as/h = 1280, so A_layer = 1314 sbh,
    A_TP = 91.5 sbh and A_TP+SP = 82.125 sbh at t = 16."""
    s, b, h, a, t = 32768, 1, 12288, 96, 16
    sbh = s * b * h
    assert orc.activation_bytes(s, b, h, a, t, 0, 1.0) == 1314 * sbh
    assert orc.activation_bytes(s, b, h, a, t, 1, 1.0) == 91.5 * sbh
    assert orc.activation_bytes(s, b, h, a, t, 2, 1.0) == 82.125 * sbh


# ----------------------------------------------------------------------------
# entry into a TP region: norm of the shard, then all-gather
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("norm", ["layernorm", "rmsnorm"])
def test_entry_norm_matches_torch_and_gathers_in_rank_order(orc, norm):
    """Each rank normalises its own tokens, then the shards are gathered in
    rank order: the gathered tensor is the library norm of the whole x."""
    w = sp_synth.WORKLOADS["C2"].replace(s=16, b=2, h=64, t=4, norm=norm,
                                          dtype="f32")
    cfg = orc.cfg_from(w)
    x = sp_synth.draw_residual(w)
    bias, gamma, beta = sp_synth.draw_params(w)
    beta = beta if norm == "layernorm" else None
    out = orc.norm_ag_fwd(cfg, x, gamma, beta, n_out=2)
    eps = float(np.float32(w.eps))
    if norm == "layernorm":
        ref = F.layer_norm(x.double(), (w.h,), gamma.double(), beta.double(),
                           eps)
    else:
        ref = F.rms_norm(x.double(), (w.h,), gamma.double(), eps)
    for q in range(2):
        assert np.allclose(out["gathered"][q].double().numpy(), ref.numpy(),
                           rtol=2 ** -23, atol=1e-30)
    # the same as the exit's norm with nothing to reduce: zero partials, no
    # bias, p = 0, the residual is x
    fo = orc.fwd(orc.cfg_from(w, p_drop=0.0), [torch.zeros_like(x)] * w.t, None, x,
                 gamma, beta)
    assert torch.equal(fo["gathered"][0], out["gathered"][0])


@pytest.mark.parametrize("norm", ["layernorm", "rmsnorm"])
def test_entry_statistics_match_torch_var_mean(orc, norm):
    """The entry's per-token statistics at t = 4, indexed by global token row:
    mean and biased variance from torch.var_mean in float64, rstd =
    1/sqrt(var + eps) (LayerNorm) or 1/sqrt(mean(x^2) + eps) (RMSNorm)."""
    w = sp_synth.WORKLOADS["C2"].replace(s=16, b=2, h=72, t=4, norm=norm,
                                          dtype="bf16")
    cfg = orc.cfg_from(w)
    x = sp_synth.draw_residual(w)
    # rows of very different scale, so a statistic stored at the wrong row
    # cannot pass by chance
    x = (x.float() * torch.arange(1, w.rows + 1,
                                  dtype=torch.float32)[:, None]).to(x.dtype)
    bias, gamma, beta = sp_synth.draw_params(w)
    beta = beta if norm == "layernorm" else None
    out = orc.norm_ag_fwd(cfg, x, gamma, beta)
    xd = x.double()
    eps = float(np.float32(w.eps))
    if norm == "layernorm":
        var, mu = torch.var_mean(xd, dim=1, unbiased=False)
        assert np.allclose(out["mean"], mu.numpy(), rtol=1e-13, atol=1e-13)
        rstd = 1.0 / torch.sqrt(var + eps)
    else:
        assert out["mean"] is None
        rstd = 1.0 / torch.sqrt(xd.pow(2).mean(1) + eps)
    assert np.allclose(out["rstd"], rstd.numpy(), rtol=1e-13, atol=0)


# ----------------------------------------------------------------------------
# fp32 residual stream beside bf16 partial sums, parameters and norm outputs
# ----------------------------------------------------------------------------

def _mixed(norm="layernorm", **over):
    d = dict(s=12, b=2, h=96, t=4, norm=norm, dtype="bf16", res_dtype="f32",
             p_drop=0.25, has_bias=True, has_beta=norm == "layernorm")
    d.update(over)
    return sp_synth.WORKLOADS["C2"].replace(**d)


def _keep_matrix(orc, w):
    p = float(np.float32(w.p_drop))
    return np.array([[orc.keep(w.drop_seed, w.drop_offset, n, j, p)
                      for j in range(w.h)] for n in range(w.rows)])


@pytest.mark.parametrize("norm", ["layernorm", "rmsnorm"])
def test_fp32_residual_stream_forward(orc, norm):
    """The stored sum is the fp32 rounding of residual + dropout(sum of
    partials + bias), formed in float64 here by torch; the norm output is
    the library norm of that fp32 tensor, rounded to bf16."""
    w = _mixed(norm)
    cfg = orc.cfg_from(w)
    parts = sp_synth.draw_partials(w)
    bias, gamma, beta = sp_synth.draw_params(w)
    beta = beta if norm == "layernorm" else None
    res = sp_synth.draw_residual(w)
    assert res.dtype == torch.float32 and parts[0].dtype == torch.bfloat16
    out = orc.fwd(cfg, parts, bias, res, gamma, beta)
    y = torch.stack([p.double() for p in parts]).sum(0) + bias.double()
    scale = 1.0 / (1.0 - float(np.float32(w.p_drop)))
    keep = torch.from_numpy(_keep_matrix(orc, w))
    z = torch.where(keep, y * scale, torch.zeros_like(y))
    want = (res.double() + z).float()
    assert out["residual_out"].dtype == torch.float32
    assert torch.equal(out["residual_out"], want)
    # the pin has power: bf16 storage of the sum would differ
    assert not torch.equal(want.bfloat16().float(), want)
    eps = float(np.float32(w.eps))
    x = want.double()
    if norm == "layernorm":
        ref = F.layer_norm(x, (w.h,), gamma.double(), beta.double(), eps)
    else:
        ref = F.rms_norm(x, (w.h,), gamma.double(), eps)
    got = out["gathered"][0]
    assert got.dtype == torch.bfloat16
    r = ref.numpy()
    assert (np.abs(got.double().numpy() - r) <= _ulp_bf16(r) * 0.5 + 1e-12 * np.abs(r)).all()


def test_fp32_residual_stream_backward(orc):
    """Reverse mode against torch autograd in float64: the residual gradient
    (with one arriving on the stream) is stored in fp32, dY in bf16."""
    w = _mixed()
    cfg = orc.cfg_from(w)
    parts = sp_synth.draw_partials(w)
    bias, gamma, beta = sp_synth.draw_params(w)
    res = sp_synth.draw_residual(w)
    fo = orc.fwd(cfg, parts, bias, res, gamma, beta)
    dparts = sp_synth.draw_grad_partials(w)
    drn = sp_synth.draw_residual_grad(w)
    assert drn.dtype == torch.float32
    bo = orc.bwd(cfg, dparts, drn, fo["residual_out"], gamma, fo["mask"],
                 fo["mean"], fo["rstd"])
    dn = torch.stack([d.double() for d in dparts]).sum(0)
    y = torch.stack([p.double() for p in parts]).sum(0)
    ref = _torch_reference_grads(w, y, bias, fo["residual_out"], gamma, beta,
                                 fo["mask"], dn, drn)
    assert bo["dresidual_in"].dtype == torch.float32
    assert torch.equal(bo["dresidual_in"], ref["dresidual_in"].float())
    r = ref["dY"].numpy()
    assert (np.abs(bo["dY"].double().numpy() - r) <= _ulp_bf16(r) * 0.5 + 1e-12 * np.abs(r)).all()
    for k in ("dgamma", "dbeta", "dbias"):
        assert np.allclose(bo[k], ref[k].numpy(), rtol=1e-10, atol=1e-10), k


def test_fp32_residual_stream_entry(orc):
    """The entry normalises an fp32 residual stream into bf16 outputs."""
    w = _mixed(p_drop=0.0, has_bias=False, s=16, h=64)
    x = sp_synth.draw_residual(w)
    bias, gamma, beta = sp_synth.draw_params(w)
    out = orc.norm_ag_fwd(orc.cfg_from(w), x, gamma, beta)
    ref = F.layer_norm(x.double(), (w.h,), gamma.double(), beta.double(),
                       float(np.float32(w.eps))).numpy()
    got = out["gathered"][0].double().numpy()
    assert (np.abs(got - ref) <= _ulp_bf16(ref) * 0.5 + 1e-12 * np.abs(ref)).all()


# ----------------------------------------------------------------------------
# tensor-parallel linears: the row-parallel reduction and the all-gathered
# column-parallel linear
# ----------------------------------------------------------------------------

def _bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_rowpar_reduce_matches_torch_matmul(orc, t):
    """The t ranks' partials summed equal the whole product x @ w^T, against
    torch.matmul in float64."""
    x, w = _bf16((5, 64), 11), _bf16((24, 64), 12)
    y = orc.rowpar_reduce(x, w, t)
    ref = (x.double() @ w.double().T).numpy()
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_rowpar_reduce_hand_worked_2x2(orc):
    """x = [[1, 2], [3, 4]], w = [[5, 6], [7, 8]] on t = 2 ranks: rank 0's
    partial is x[:, 0] w[:, 0]^T = [[5, 7], [15, 21]], rank 1's is
    [[12, 16], [24, 32]]; their sum is x w^T = [[17, 23], [39, 53]]."""
    x = torch.tensor([[1.0, 2.0], [3.0, 4.0]]).to(torch.bfloat16)
    w = torch.tensor([[5.0, 6.0], [7.0, 8.0]]).to(torch.bfloat16)
    assert np.array_equal(orc.rowpar_reduce(x[:, :1], w[:, :1], 1), [[5, 7], [15, 21]])
    assert np.array_equal(orc.rowpar_reduce(x[:, 1:], w[:, 1:], 1), [[12, 16], [24, 32]])
    assert np.array_equal(orc.rowpar_reduce(x, w, 2), [[17, 23], [39, 53]])


def test_rowpar_reduce_does_not_depend_on_t(orc):
    """Small integer inputs make every partial and every sum exact, so the
    split of the inner dimension over t ranks cannot change the result."""
    g = torch.Generator().manual_seed(5)
    x = torch.randint(-3, 4, (6, 64), generator=g).to(torch.bfloat16)
    w = torch.randint(-3, 4, (10, 64), generator=g).to(torch.bfloat16)
    ys = [orc.rowpar_reduce(x, w, t) for t in (1, 2, 4, 8)]
    for y in ys[1:]:
        assert np.array_equal(y, ys[0])


@pytest.mark.parametrize("norm", ["layernorm", "rmsnorm"])
def test_linear_rs_equals_the_boundary_on_exact_partials(orc, norm):
    """With inputs whose every rank partial is exact in bf16 (integers of at
    most 64 in magnitude), the row-parallel linear followed by the SP region
    gives exactly what the boundary gives on those partials stored as t
    buffers: stored sum, norm output, mask and statistics, bit for bit."""
    w_ = sp_synth.WORKLOADS["C2"].replace(s=8, b=2, h=48, t=4, norm=norm,
                                           p_drop=0.25,
                                           has_beta=norm == "layernorm")
    f, t = 64, w_.t
    g = torch.Generator().manual_seed(9)
    x = torch.randint(-2, 3, (w_.rows, f), generator=g).to(torch.bfloat16)
    w = torch.randint(-2, 3, (w_.h, f), generator=g).to(torch.bfloat16)
    bias, gamma, beta = sp_synth.draw_params(w_)
    beta = beta if norm == "layernorm" else None
    res = sp_synth.draw_residual(w_)
    cfg = orc.cfg_from(w_)
    per = f // t
    parts = [(x[:, k * per:(k + 1) * per].double() @
              w[:, k * per:(k + 1) * per].double().T).to(torch.bfloat16)
             for k in range(t)]
    for p_ in parts:
        assert p_.double().abs().max() <= 64
    ref = orc.fwd(cfg, parts, bias, res, gamma, beta)
    got = orc.linear_rs_fwd_rows(cfg, f, list(range(w_.rows)), x, w, bias, res,
                                 gamma, beta)
    assert torch.equal(got["residual_out"], ref["residual_out"])
    assert torch.equal(got["norm_out"], ref["gathered"][0])
    assert np.array_equal(got["mask"], ref["mask"])
    assert np.array_equal(got["rstd"], ref["rstd"])
    if norm == "layernorm":
        assert np.array_equal(got["mean"], ref["mean"])


@pytest.mark.parametrize("t", [1, 2, 4])
def test_ag_colpar_is_the_correctly_rounded_product_of_the_gathered_input(orc, t):
    """The shards are gathered in rank order and multiplied by w^T: every
    output is the float64 product (torch.matmul) rounded once to bf16, so it
    lies within half a bf16 ulp of it; and reversing the shard order changes
    the rows."""
    shards = [_bf16((6, 40), 20 + r) for r in range(t)]
    w = _bf16((24, 40), 30)
    out = orc.ag_colpar_fwd(shards, w).double().numpy()
    ref = (torch.cat(shards).double() @ w.double().T).numpy()
    e = np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126)))
    assert (np.abs(out - ref) <= 2.0 ** (e - 8) * (1 + 1e-12)).all()
    if t > 1:
        rev = orc.ag_colpar_fwd(shards[::-1], w).double().numpy()
        assert not np.array_equal(rev, out)


# ----------------------------------------------------------------------------
# context parallelism: ring attention with an online softmax
# ----------------------------------------------------------------------------

def _attn_ref(q, k, v, scale):
    """softmax(q k^T * scale) v and the log-sum-exp, float64 (torch)."""
    sc = (q.double() @ k.double().transpose(-1, -2)) * scale
    return torch.softmax(sc, -1) @ v.double(), torch.logsumexp(sc, -1)


@pytest.mark.parametrize("t", [1, 2, 4, 8])
def test_ring_attention_equals_plain_attention(orc, t):
    """After the t ring steps the online softmax has reached the plain
    softmax attention over all keys: the output is its bf16 rounding and the
    log-sum-exp matches torch.logsumexp (float64)."""
    bh, s, d = 2, 32, 16
    q, k, v = (_bf16((bh, s, d), 40 + i) for i in range(3))
    scale = d ** -0.5
    out, lse = orc.ring_attention(q, k, v, t, scale)
    ref, ref_lse = _attn_ref(q, k, v, scale)
    e = np.floor(np.log2(np.maximum(np.abs(ref.numpy()), 2.0 ** -126)))
    assert (np.abs(out.double().numpy() - ref.numpy()) <= 2.0 ** (e - 8) * 1.001 + 1e-12).all()
    assert np.allclose(lse, ref_lse.numpy(), rtol=1e-12, atol=1e-12)


def test_ring_attention_special_cases(orc):
    """All scores equal (q = 0): every query averages all values.  One key
    far above the rest: the output is that key's value (to the bf16 ulp)."""
    bh, s, d, t = 1, 16, 8, 4
    k, v = _bf16((bh, s, d), 50), _bf16((bh, s, d), 51)
    q = torch.zeros((bh, s, d), dtype=torch.bfloat16)
    out, lse = orc.ring_attention(q, k, v, t, 1.0)
    mean = v.double().mean(1, keepdim=True).expand(bh, s, d)
    assert torch.allclose(out.double(), mean, rtol=2 ** -8, atol=1e-6)
    assert np.allclose(lse, np.log(s))
    k2 = torch.zeros((bh, s, d), dtype=torch.bfloat16)
    k2[0, 11] = 8.0                      # key 11 in rank 2's block
    q2 = torch.ones((bh, s, d), dtype=torch.bfloat16)
    out2, _ = orc.ring_attention(q2, k2, v, t, 1.0)
    assert torch.equal(out2[0], v[0, 11].expand(s, d))


def test_ring_attention_rows_agree_with_the_whole(orc):
    bh, s, d, t = 1, 64, 16, 4
    q, k, v = (_bf16((bh, s, d), 60 + i) for i in range(3))
    out, lse = orc.ring_attention(q, k, v, t, 0.25)
    rows = [0, 15, 16, 47, 63]
    o2, l2 = orc.ring_attention_rows(q[0, rows], rows, k[0], v[0], t, 0.25)
    assert torch.equal(o2, out[0, rows])
    assert np.array_equal(l2, lse[0, rows])
