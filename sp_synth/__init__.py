"""Seeded synthetic inputs for the sequence-parallel boundary workloads.

This module is shared by the tests, ``bench.py`` and the oracle's callers.  It
draws random tensors and nothing else: it contains none of the boundary's
arithmetic (no reduction, dropout, residual add or normalisation), so the CUDA
path and the CPU oracle stay independent of each other.

Workloads
---------
The five workloads are the token-row problems of a Megatron sequence-parallel
boundary ("Sequence Parallelism math", section "The move: split the
LayerNorm/dropout band along the sequence"; "SP: Partition Activations
Alongside TP", section "Normalize and add residuals by token"):

====  =====  ===  =====  ==  =====  =====  ====================================
name  s      b    h      t   dtype  norm   notes
====  =====  ===  =====  ==  =====  =====  ====================================
C1    4      1    4      2   f32    LN     worked 4-token x 4-feature layout
C2    2048   4    6144   8   bf16   LN     22B-class layer shape, p = 0.1
C3    4096   1    8192   8   bf16   RMS    p = 0, no bias / beta
C4    8192   2    4096   4   bf16   LN     backward workload, p = 0.1
C5    32768  1    12288  16  bf16   LN     1 % outliers x100, p = 0.1, a = 96
====  =====  ===  =====  ==  =====  =====  ====================================

Recipe (every draw is fp32, then rounded to nearest-even into the I/O dtype):

* partial sums ``P_k ~ N(0, 1/t)`` (variance 1/t, so the reduced sum is about
  N(0, 1)); C1 uses U(-1, 1).  For C5 each partial element is, independently
  with probability 0.01 (its own Bernoulli draw), multiplied by 100 before
  rounding.
* residual ``~ N(0, 1)`` (C1: U(-1, 1)).
* bias and beta ``~ N(0, 0.02)`` read as standard deviation 0.02; gamma
  ``~ 1 + N(0, 0.02)``.  C1 draws all three from U(-1, 1).
* backward upstream partials ``dP_k ~ N(0, 1/t)``.
* C1 plants the two partial-sum values the worked layout prints for token t0,
  feature 0: 4 on GPU 0 and 5 on GPU 1, whose reduction is 9 ("SP: Partition
  Activations Alongside TP", section "Change layouts between SP and TP").

Each tensor has its own generator seeded from ``(config seed, tensor id)`` so
that a tensor's values do not depend on which other tensors were drawn.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import torch

# ----------------------------------------------------------------------------
# workload table
# ----------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    s: int
    b: int
    h: int
    t: int
    dtype: str           # "f32" or "bf16"
    norm: str            # "layernorm" or "rmsnorm"
    eps: float
    p_drop: float
    has_bias: bool
    has_beta: bool
    dist: str            # "uniform" (C1) or "normal"
    outliers: float      # probability of a x100 outlier per partial element
    seed: int            # base seed of every tensor draw
    drop_seed: int = 0   # Philox key of the dropout mask
    drop_offset: int = 0
    heads: int = 0       # attention heads for the activation-memory check
    backward: bool = False
    gather_replicas: bool = False  # also gather into t per-rank replicas
    # dtype of the residual stream (residual in, stored sum, dR_next and the
    # residual gradient): "" for the I/O dtype, or "f32" (an fp32 residual
    # stream beside bf16 partial sums, parameters and norm outputs)
    res_dtype: str = ""

    @property
    def rows(self) -> int:
        return self.s * self.b

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def res(self) -> str:
        """dtype of the residual stream"""
        return self.res_dtype or self.dtype

    @property
    def res_torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.res == "f32" else torch.bfloat16

    @property
    def res_elem_bytes(self) -> int:
        return 4 if self.res == "f32" else 2

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    "C1": Workload("C1", s=4, b=1, h=4, t=2, dtype="f32", norm="layernorm",
                   eps=1e-5, p_drop=0.1, has_bias=True, has_beta=True,
                   dist="uniform", outliers=0.0, seed=1),
    "C2": Workload("C2", s=2048, b=4, h=6144, t=8, dtype="bf16",
                   norm="layernorm", eps=1e-5, p_drop=0.1, has_bias=True,
                   has_beta=True, dist="normal", outliers=0.0, seed=2,
                   backward=True),
    "C3": Workload("C3", s=4096, b=1, h=8192, t=8, dtype="bf16",
                   norm="rmsnorm", eps=1e-6, p_drop=0.0, has_bias=False,
                   has_beta=False, dist="normal", outliers=0.0, seed=3,
                   gather_replicas=True),
    "C4": Workload("C4", s=8192, b=2, h=4096, t=4, dtype="bf16",
                   norm="layernorm", eps=1e-5, p_drop=0.1, has_bias=True,
                   has_beta=True, dist="normal", outliers=0.0, seed=4,
                   backward=True),
    "C5": Workload("C5", s=32768, b=1, h=12288, t=16, dtype="bf16",
                   norm="layernorm", eps=1e-5, p_drop=0.1, has_bias=True,
                   has_beta=True, dist="normal", outliers=0.01, seed=5,
                   heads=96, backward=True),
}

# tensor ids for seeding
_ID_PARTIAL = 100      # + k
_ID_OUTLIER = 300      # + k
_ID_RESIDUAL = 1
_ID_BIAS = 2
_ID_GAMMA = 3
_ID_BETA = 4
_ID_DPARTIAL = 500     # + k
_ID_DRNEXT = 5


def _gen(seed: int, tid: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1_000_003 + tid)
    return g


def _draw(shape, dist: str, scale: float, shift: float, seed: int, tid: int,
          device, out_dtype: torch.dtype) -> torch.Tensor:
    g = _gen(seed, tid, device)
    if dist == "uniform":
        x = torch.rand(shape, generator=g, device=device, dtype=torch.float32)
        x = x.mul_(2.0).sub_(1.0)
    else:
        x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        x = x.mul_(scale)
    if shift:
        x = x.add_(shift)
    return x.to(out_dtype)


def draw_partials(w: Workload, device="cpu", rows: Optional[int] = None,
                  tid_base: int = _ID_PARTIAL) -> List[torch.Tensor]:
    """t partial-sum tensors, each ``[rows, h]`` (``rows`` defaults to s*b).

    The ``[s, b, h]`` layout with h fastest is stored flattened as
    ``[s*b, h]``; token row n = s_idx * b + b_idx.
    """
    n = w.rows if rows is None else rows
    std = (1.0 / w.t) ** 0.5
    out = []
    for k in range(w.t):
        g = _gen(w.seed, tid_base + k, device)
        if w.dist == "uniform":
            x = torch.rand((n, w.h), generator=g, device=device,
                           dtype=torch.float32).mul_(2.0).sub_(1.0)
        else:
            x = torch.randn((n, w.h), generator=g, device=device,
                            dtype=torch.float32).mul_(std)
        if w.outliers > 0.0:
            go = _gen(w.seed, _ID_OUTLIER + k, device)
            hit = torch.rand((n, w.h), generator=go, device=device,
                             dtype=torch.float32) < w.outliers
            x = torch.where(hit, x * 100.0, x)
        out.append(x.to(w.torch_dtype))
    if w.name == "C1" and tid_base == _ID_PARTIAL and n > 0:
        # the worked layout's token t0, feature 0: 4 on GPU 0 plus 5 on GPU 1
        out[0][0, 0] = 4.0
        out[1][0, 0] = 5.0
    return out


def draw_residual(w: Workload, device="cpu", rows: Optional[int] = None):
    n = w.rows if rows is None else rows
    return _draw((n, w.h), w.dist, 1.0, 0.0, w.seed, _ID_RESIDUAL, device,
                 w.res_torch_dtype)


def draw_params(w: Workload, device="cpu"):
    """(bias, gamma, beta); absent ones are None."""
    bias = (_draw((w.h,), w.dist, 0.02, 0.0, w.seed, _ID_BIAS, device,
                  w.torch_dtype) if w.has_bias else None)
    if w.dist == "uniform":
        gamma = _draw((w.h,), "uniform", 1.0, 0.0, w.seed, _ID_GAMMA, device,
                      w.torch_dtype)
    else:
        gamma = _draw((w.h,), "normal", 0.02, 1.0, w.seed, _ID_GAMMA, device,
                      w.torch_dtype)
    beta = (_draw((w.h,), w.dist, 0.02, 0.0, w.seed, _ID_BETA, device,
                  w.torch_dtype) if w.has_beta else None)
    return bias, gamma, beta


def draw_grad_partials(w: Workload, device="cpu", rows: Optional[int] = None):
    """t upstream-gradient partials dP_k ``[rows, h]`` ~ N(0, 1/t)."""
    n = w.rows if rows is None else rows
    std = (1.0 / w.t) ** 0.5
    out = []
    for k in range(w.t):
        g = _gen(w.seed, _ID_DPARTIAL + k, device)
        if w.dist == "uniform":
            x = torch.rand((n, w.h), generator=g, device=device,
                           dtype=torch.float32).mul_(2.0).sub_(1.0)
        else:
            x = torch.randn((n, w.h), generator=g, device=device,
                            dtype=torch.float32).mul_(std)
        out.append(x.to(w.torch_dtype))
    return out


def draw_residual_grad(w: Workload, device="cpu", rows: Optional[int] = None):
    """Optional gradient arriving on the residual stream from later layers."""
    n = w.rows if rows is None else rows
    return _draw((n, w.h), w.dist, 1.0, 0.0, w.seed, _ID_DRNEXT, device,
                 w.res_torch_dtype)


def dyadic_atoms(rows: int, h: int, seed: int, n_atoms: int = 16,
                 device="cpu") -> List[torch.Tensor]:
    """n_atoms tensors whose entries are multiples of 1/8 in [-1, 1].

    Grouping the atoms into t pieces (``group_atoms``) gives partial sums that
    are multiples of 1/8 with magnitude at most n_atoms, so every piece is
    exact in bf16 and in fp32, and every fp32 sum of pieces is exact whatever
    the order.  The same atoms grouped for different t therefore describe the
    same reduced tensor, bit for bit.
    """
    g = _gen(seed, 900, device)
    return [torch.randint(-8, 9, (rows, h), generator=g, device=device)
            .to(torch.float32) / 8.0 for _ in range(n_atoms)]


def group_atoms(atoms: List[torch.Tensor], t: int,
                dtype: torch.dtype) -> List[torch.Tensor]:
    """Split the atoms into t contiguous groups; piece k is group k's total."""
    n = len(atoms)
    if n % t:
        raise ValueError("t must divide the number of atoms")
    per = n // t
    pieces = []
    for k in range(t):
        acc = torch.zeros_like(atoms[0])
        for a in atoms[k * per:(k + 1) * per]:
            acc = acc + a
        pieces.append(acc.to(dtype))
    return pieces


def bf16_bits_to_f64(x: torch.Tensor):
    """Exact widening of a bf16/f32 tensor to a float64 numpy array."""
    return x.detach().to("cpu").to(torch.float64).numpy()
