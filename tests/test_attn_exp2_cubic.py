"""The ring-attention kernel computes one exponential pair in 8 with a cubic
for 2^f on [-1/2, 1/2] (plus an exponent-field shift for the integer part).
The GPU tests widen the log-sum-exp tolerance by that cubic's relative
error bound; this pins the bound to the coefficients the kernel source holds,
evaluated the kernel's way in fp32 (Horner, then 2^n into the exponent), on
a dense grid over the whole input range the kernel admits."""
import os
import re

import numpy as np

from test_gpu_attn import EXP2_POLY_REL

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "sp_region_b200", "csrc", "sp_attn.cuh")


def _coefficients():
    text = open(SRC).read()
    body = text[text.index("F2 exp2_poly2(F2 x)"):]
    body = body[:body.index("\n}\n")]
    hexes = re.findall(r"f2\((0x[0-9a-fA-F.]+p[-+]?\d+)f\)", body)
    assert len(hexes) == 4, hexes
    return [np.float32(float.fromhex(h)) for h in hexes]


def _cubic_exp2(x, c):
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)              # 1.5 * 2^23: round to nearest
    sh = (x + magic).astype(np.float32)
    n = (sh - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = (c[0].astype(np.float64) * f + c[1]).astype(np.float32)
    p = (p.astype(np.float64) * f + c[2]).astype(np.float32)
    p = (p.astype(np.float64) * f + c[3]).astype(np.float32)
    bits = (p.view(np.int32).astype(np.int64) + (sh.view(np.int32).astype(np.int64) << 23))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_cubic_meets_the_bound_the_tolerance_uses():
    c = _coefficients()
    # probabilities are 2^(s * scale - m) with m the maximum in use: inputs
    # run from far below zero up to the 8 (log2) the lazy rescale allows
    x = np.concatenate([np.linspace(-125.0, 8.0, 4_000_001),
                        np.arange(-125, 9, dtype=np.float64) + 0.5]).astype(np.float32)
    got = _cubic_exp2(x, c).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() <= EXP2_POLY_REL, rel.max()
    assert np.all(got > 0) and np.all(np.isfinite(got))


def test_cubic_clamps_far_below_zero():
    c = _coefficients()
    got = _cubic_exp2(np.array([-1e4, -300.0, -126.0], dtype=np.float32), c)
    # the clamp keeps the exponent field positive: a tiny positive number,
    # negligible against a row sum of at least 1
    assert np.all(got > 0) and np.all(got < 1e-37)
