"""CPU oracle of the sequence-parallel boundary (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (``sp_region_b200``)
never imports, links or runs anything here, and this package never imports the
product: the two share nothing but the seeded input generators in ``sp_synth``.

The arithmetic lives in ``sp_oracle.c`` (plain scalar C, double precision);
this module only builds it with gcc and marshals tensors through ctypes.
Inputs are CPU tensors in the I/O dtype (float32 or bfloat16), outputs are
tensors in the I/O dtype plus float64 numpy arrays for the statistics and the
parameter gradients.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import List, Optional, Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sp_oracle.c")
_LIB = os.path.join(_HERE, "liborc.so")

F32, BF16 = 0, 1
LAYERNORM, RMSNORM = 0, 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE double, no contraction into FMA).

    ``SP_ORACLE_LIB`` names an already built library to load instead; the
    mutation tests use it to run the pins against deliberately broken copies.
    """
    override = os.environ.get("SP_ORACLE_LIB")
    if override:
        return override
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-o", _LIB + ".tmp", _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(_LIB + ".tmp", _LIB)
    return _LIB


class Cfg(ctypes.Structure):
    _fields_ = [("s", ctypes.c_int64), ("b", ctypes.c_int64),
                ("h", ctypes.c_int64), ("t", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("norm", ctypes.c_int32),
                ("eps", ctypes.c_float), ("p_drop", ctypes.c_float),
                ("seed", ctypes.c_uint64), ("offset", ctypes.c_uint64),
                ("res_dtype", ctypes.c_int32)]


_lib_handle = None


def _lib():
    global _lib_handle
    if _lib_handle is None:
        _lib_handle = ctypes.CDLL(build())
        L = _lib_handle
        vp, i64, i32, dp = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                            ctypes.c_void_p)
        L.orc_philox4x32_10.argtypes = [vp, vp, vp]
        L.orc_round.argtypes = [ctypes.c_double, ctypes.c_int]
        L.orc_round.restype = ctypes.c_double
        L.orc_drop_threshold.argtypes = [ctypes.c_float]
        L.orc_drop_threshold.restype = ctypes.c_uint32
        L.orc_keep.argtypes = [ctypes.c_uint64, ctypes.c_uint64, i64, i64,
                               ctypes.c_float]
        L.orc_keep.restype = ctypes.c_int
        L.orc_mask_words.argtypes = [i64]
        L.orc_mask_words.restype = i64
        L.orc_all_reduce.argtypes = [ctypes.c_int, i64, ctypes.c_int, vp, dp]
        L.orc_reduce_scatter.argtypes = [ctypes.c_int, i64, i64, ctypes.c_int,
                                         vp, ctypes.c_int, dp]
        L.orc_all_gather.argtypes = [ctypes.c_int, i64, i64, vp, dp]
        L.orc_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int,
                              vp, dp, dp]
        L.orc_fwd.restype = ctypes.c_int
        L.orc_fwd_rows.argtypes = [vp, i64, vp, vp, vp, vp, vp, vp, vp, vp,
                                   vp, dp, dp]
        L.orc_fwd_rows.restype = ctypes.c_int
        L.orc_norm_ag_fwd.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int, dp, dp]
        L.orc_norm_ag_fwd.restype = ctypes.c_int
        L.orc_bwd.argtypes = [vp, vp, vp, vp, vp, vp, dp, dp, vp, vp, dp, dp,
                              dp]
        L.orc_bwd.restype = ctypes.c_int
        L.orc_bwd_rows.argtypes = [vp, i64, vp, vp, vp, vp, vp, dp, dp, vp, vp,
                                   dp, dp, dp]
        L.orc_bwd_rows.restype = ctypes.c_int
        L.orc_rowpar_reduce.argtypes = [i64, i64, i64, ctypes.c_int, vp, vp, dp]
        L.orc_linear_rs_fwd_rows.argtypes = [vp, i64, i64, vp, vp, vp, vp, vp, vp,
                                             vp, vp, vp, vp, dp, dp]
        L.orc_linear_rs_fwd_rows.restype = ctypes.c_int
        L.orc_ag_colpar_fwd.argtypes = [ctypes.c_int, i64, i64, i64, vp, vp, vp]
        L.orc_ag_colpar_fwd.restype = ctypes.c_int
        L.orc_ring_attention.argtypes = [i64, i64, i64, ctypes.c_int, ctypes.c_double,
                                         vp, vp, vp, vp, dp]
        L.orc_ring_attention.restype = ctypes.c_int
        L.orc_ring_attention_rows.argtypes = [i64, i64, ctypes.c_int, ctypes.c_double,
                                              vp, vp, i64, vp, vp, vp, dp]
        L.orc_ring_attention_rows.restype = ctypes.c_int
        L.orc_activation_bytes.argtypes = [i64, i64, i64, i64, i32, i32,
                                           ctypes.c_double]
        L.orc_activation_bytes.restype = ctypes.c_double
        L.orc_ring_bytes.argtypes = [i32, i32, ctypes.c_double]
        L.orc_ring_bytes.restype = ctypes.c_double
    return _lib_handle


# ----------------------------------------------------------------------------
# marshalling helpers
# ----------------------------------------------------------------------------

def _dtype_code(dt) -> int:
    if dt in ("f32", torch.float32):
        return F32
    if dt in ("bf16", torch.bfloat16):
        return BF16
    raise ValueError(f"unsupported dtype {dt}")


def _torch_dtype(code: int) -> torch.dtype:
    return torch.float32 if code == F32 else torch.bfloat16


def make_cfg(s, b, h, t, dtype, norm, eps, p_drop, seed=0, offset=0,
             res_dtype=None) -> Cfg:
    """res_dtype: dtype of the residual stream tensors (None or "": dtype)."""
    return Cfg(s=s, b=b, h=h, t=t, dtype=_dtype_code(dtype),
               norm=LAYERNORM if norm in ("layernorm", LAYERNORM) else RMSNORM,
               eps=eps, p_drop=p_drop, seed=seed, offset=offset,
               res_dtype=_dtype_code(res_dtype or dtype))


def cfg_from(w, **over) -> Cfg:
    """Oracle configuration from a workload description (``sp_synth``)."""
    d = dict(s=w.s, b=w.b, h=w.h, t=w.t, dtype=w.dtype, norm=w.norm,
             eps=w.eps, p_drop=w.p_drop, seed=w.drop_seed,
             offset=w.drop_offset, res_dtype=w.res)
    d.update(over)
    return make_cfg(**d)


def _cpu(x: Optional[torch.Tensor], dt_code: int) -> Optional[torch.Tensor]:
    if x is None:
        return None
    x = x.detach().to("cpu").contiguous()
    if x.dtype != _torch_dtype(dt_code):
        raise TypeError(f"expected {_torch_dtype(dt_code)}, got {x.dtype}")
    return x


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.data_ptr()
    return x.ctypes.data


def _ptr_array(ts: Sequence) -> ctypes.Array:
    arr = (ctypes.c_void_p * len(ts))()
    for i, x in enumerate(ts):
        arr[i] = _ptr(x)
    return arr


# ----------------------------------------------------------------------------
# primitives
# ----------------------------------------------------------------------------

def philox(ctr: Sequence[int], key: Sequence[int]) -> List[int]:
    c = np.array(ctr, dtype=np.uint32)
    k = np.array(key, dtype=np.uint32)
    o = np.zeros(4, dtype=np.uint32)
    _lib().orc_philox4x32_10(c.ctypes.data, k.ctypes.data, o.ctypes.data)
    return [int(v) for v in o]


def round_to(x: float, dtype) -> float:
    return _lib().orc_round(float(x), _dtype_code(dtype))


def drop_threshold(p: float) -> int:
    return int(_lib().orc_drop_threshold(p))


def keep(seed: int, offset: int, n: int, j: int, p: float) -> bool:
    return bool(_lib().orc_keep(seed, offset, n, j, p))


def mask_words(h: int) -> int:
    return int(_lib().orc_mask_words(h))


def all_reduce(parts: Sequence[torch.Tensor]) -> np.ndarray:
    dt = _dtype_code(parts[0].dtype)
    ps = [_cpu(p, dt) for p in parts]
    out = np.zeros(ps[0].numel(), dtype=np.float64)
    _lib().orc_all_reduce(len(ps), ps[0].numel(), dt, _ptr_array(ps),
                          out.ctypes.data)
    return out.reshape(tuple(ps[0].shape))


def reduce_scatter(parts: Sequence[torch.Tensor], rank: int) -> np.ndarray:
    """parts: t tensors [rows, h]; returns rank's [rows/t, h] float64."""
    dt = _dtype_code(parts[0].dtype)
    ps = [_cpu(p, dt) for p in parts]
    rows, h = ps[0].shape
    t = len(ps)
    out = np.zeros((rows // t, h), dtype=np.float64)
    _lib().orc_reduce_scatter(t, rows, h, dt, _ptr_array(ps), rank,
                              out.ctypes.data)
    return out


def all_gather(shards: Sequence[np.ndarray]) -> np.ndarray:
    sh = [np.ascontiguousarray(s, dtype=np.float64) for s in shards]
    rows, h = sh[0].shape
    out = np.zeros((rows * len(sh), h), dtype=np.float64)
    _lib().orc_all_gather(len(sh), rows, h, _ptr_array(sh), out.ctypes.data)
    return out


def activation_bytes(s, b, h, a, t, mode, bytes_per_elem) -> float:
    return float(_lib().orc_activation_bytes(s, b, h, a, t, mode,
                                             bytes_per_elem))


def ring_bytes(t: int, kind: str, V: float) -> float:
    k = {"reduce_scatter": 0, "all_gather": 1, "all_reduce": 2}[kind]
    return float(_lib().orc_ring_bytes(t, k, V))


# ----------------------------------------------------------------------------
# the boundary
# ----------------------------------------------------------------------------

def fwd(cfg: Cfg, parts, bias, residual, gamma, beta, n_out: int = 1,
        want_mask: bool = True) -> dict:
    """Forward on all t emulated ranks.  Tensors are [s*b, h] / [h]."""
    dt, rdt = cfg.dtype, cfg.res_dtype
    tdt = _torch_dtype(dt)
    ps = [_cpu(p, dt) for p in parts]
    bias, gamma, beta = (_cpu(x, dt) for x in (bias, gamma, beta))
    residual = _cpu(residual, rdt)
    N, h = cfg.s * cfg.b, cfg.h
    rout = torch.empty((N, h), dtype=_torch_dtype(rdt))
    gathered = [torch.empty((N, h), dtype=tdt) for _ in range(n_out)]
    mask = (np.zeros((N, mask_words(h)), dtype=np.uint32) if want_mask
            else None)
    mean = np.zeros(N, dtype=np.float64)
    rstd = np.zeros(N, dtype=np.float64)
    rc = _lib().orc_fwd(ctypes.byref(cfg), _ptr_array(ps), _ptr(bias),
                        _ptr(residual), _ptr(gamma), _ptr(beta), _ptr(rout),
                        _ptr_array(gathered), n_out, _ptr(mask),
                        mean.ctypes.data, rstd.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle forward rejected the configuration ({rc})")
    return dict(residual_out=rout, gathered=gathered, mask=mask,
                mean=mean if cfg.norm == LAYERNORM else None, rstd=rstd)


def fwd_rows(cfg: Cfg, row_ids, part_rows, bias, residual_rows, gamma,
             beta) -> dict:
    """Forward on selected global token rows; inputs are [nrows, h]."""
    dt, rdt = cfg.dtype, cfg.res_dtype
    tdt = _torch_dtype(dt)
    ids = np.ascontiguousarray(np.asarray(row_ids, dtype=np.int64))
    ps = [_cpu(p, dt) for p in part_rows]
    bias, gamma, beta = (_cpu(x, dt) for x in (bias, gamma, beta))
    residual_rows = _cpu(residual_rows, rdt)
    n, h = len(ids), cfg.h
    rout = torch.empty((n, h), dtype=_torch_dtype(rdt))
    out = torch.empty((n, h), dtype=tdt)
    mask = np.zeros((n, mask_words(h)), dtype=np.uint32)
    mean = np.zeros(n, dtype=np.float64)
    rstd = np.zeros(n, dtype=np.float64)
    rc = _lib().orc_fwd_rows(ctypes.byref(cfg), n, ids.ctypes.data,
                             _ptr_array(ps), _ptr(bias), _ptr(residual_rows),
                             _ptr(gamma), _ptr(beta), _ptr(rout), _ptr(out),
                             mask.ctypes.data, mean.ctypes.data,
                             rstd.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle forward rejected the configuration ({rc})")
    return dict(residual_out=rout, norm_out=out, mask=mask,
                mean=mean if cfg.norm == LAYERNORM else None, rstd=rstd)


def norm_ag_fwd(cfg: Cfg, x, gamma, beta, n_out: int = 1) -> dict:
    """Entry into a TP region: per-rank norm of x's shard, then all-gather."""
    dt = cfg.dtype
    tdt = _torch_dtype(dt)
    gamma, beta = (_cpu(v, dt) for v in (gamma, beta))
    x = _cpu(x, cfg.res_dtype)
    N, h = cfg.s * cfg.b, cfg.h
    gathered = [torch.empty((N, h), dtype=tdt) for _ in range(n_out)]
    mean = np.zeros(N)
    rstd = np.zeros(N)
    rc = _lib().orc_norm_ag_fwd(ctypes.byref(cfg), _ptr(x), _ptr(gamma),
                                _ptr(beta), _ptr_array(gathered), n_out,
                                mean.ctypes.data, rstd.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle entry forward rejected the configuration ({rc})")
    return dict(gathered=gathered,
                mean=mean if cfg.norm == LAYERNORM else None, rstd=rstd)


def bwd(cfg: Cfg, dparts, drnext, x, gamma, mask, mean, rstd,
        with_dbeta: bool = True, with_dbias: bool = True) -> dict:
    """Backward on all t emulated ranks (mask None: nothing was dropped)."""
    dt, rdt = cfg.dtype, cfg.res_dtype
    tdt = _torch_dtype(dt)
    ps = [_cpu(p, dt) for p in dparts]
    gamma = _cpu(gamma, dt)
    drnext, x = (_cpu(v, rdt) for v in (drnext, x))
    N, h = cfg.s * cfg.b, cfg.h
    mask = None if mask is None else np.ascontiguousarray(mask, np.uint32)
    mean = (np.zeros(N) if mean is None
            else np.ascontiguousarray(mean, np.float64))
    rstd = np.ascontiguousarray(rstd, np.float64)
    dres = torch.empty((N, h), dtype=_torch_dtype(rdt))
    dY = torch.empty((N, h), dtype=tdt)
    dg = np.zeros(h)
    db = np.zeros(h) if with_dbeta else None
    dc = np.zeros(h) if with_dbias else None
    rc = _lib().orc_bwd(ctypes.byref(cfg), _ptr_array(ps), _ptr(drnext),
                        _ptr(x), _ptr(gamma), _ptr(mask), mean.ctypes.data,
                        rstd.ctypes.data, _ptr(dres), _ptr(dY), dg.ctypes.data,
                        _ptr(db), _ptr(dc))
    if rc != 0:
        raise ValueError(f"oracle backward rejected the configuration ({rc})")
    return dict(dresidual_in=dres, dY=dY, dgamma=dg, dbeta=db, dbias=dc)


def bwd_rows(cfg: Cfg, dpart_rows, drnext_rows, x_rows, gamma, mask_rows,
             mean, rstd, with_params: bool = False) -> dict:
    """Backward on selected rows.  with_params: also return the rows' share
    of dgamma / dbeta / dbias (float64 sums over these rows; summing the
    shares of a partition of all tokens gives the full gradients)."""
    dt, rdt = cfg.dtype, cfg.res_dtype
    tdt = _torch_dtype(dt)
    ps = [_cpu(p, dt) for p in dpart_rows]
    gamma = _cpu(gamma, dt)
    drnext_rows, x_rows = (_cpu(v, rdt) for v in (drnext_rows, x_rows))
    n, h = x_rows.shape
    mask_rows = (None if mask_rows is None
                 else np.ascontiguousarray(mask_rows, np.uint32))
    mean = (np.zeros(n) if mean is None
            else np.ascontiguousarray(mean, np.float64))
    rstd = np.ascontiguousarray(rstd, np.float64)
    dres = torch.empty((n, h), dtype=_torch_dtype(rdt))
    dY = torch.empty((n, h), dtype=tdt)
    pg = [np.zeros(h) for _ in range(3)] if with_params else [None] * 3
    rc = _lib().orc_bwd_rows(ctypes.byref(cfg), n, _ptr_array(ps),
                             _ptr(drnext_rows), _ptr(x_rows), _ptr(gamma),
                             _ptr(mask_rows), mean.ctypes.data,
                             rstd.ctypes.data, _ptr(dres), _ptr(dY),
                             *(_ptr(g) for g in pg))
    if rc != 0:
        raise ValueError(f"oracle backward rejected the configuration ({rc})")
    out = dict(dresidual_in=dres, dY=dY)
    if with_params:
        out.update(dgamma=pg[0], dbeta=pg[1], dbias=pg[2])
    return out


# ----------------------------------------------------------------------------
# tensor-parallel linears on t emulated ranks
# ----------------------------------------------------------------------------

def rowpar_reduce(x, w, t: int) -> np.ndarray:
    """Row-parallel linear: the t ranks' partials x[:, slice k] @ w[:, slice
    k]^T summed k ascending, in float64.  x [rows, f], w [h, f] bf16."""
    x, w = _cpu(x, BF16), _cpu(w, BF16)
    rows, f = x.shape
    h = w.shape[0]
    y = np.zeros((rows, h))
    _lib().orc_rowpar_reduce(rows, f, h, t, _ptr(x), _ptr(w), y.ctypes.data)
    return y


def linear_rs_fwd_rows(cfg: Cfg, f: int, row_ids, x_rows, w, bias, residual_rows,
                       gamma, beta) -> dict:
    """The row-parallel linear, then the SP region, on selected global token
    rows (x_rows [nrows, f], residual_rows [nrows, h])."""
    ids = np.ascontiguousarray(np.asarray(row_ids, dtype=np.int64))
    x_rows, w = _cpu(x_rows, BF16), _cpu(w, BF16)
    bias, gamma, beta = (_cpu(v, cfg.dtype) for v in (bias, gamma, beta))
    residual_rows = _cpu(residual_rows, cfg.res_dtype)
    n, h = len(ids), cfg.h
    rout = torch.empty((n, h), dtype=_torch_dtype(cfg.res_dtype))
    out = torch.empty((n, h), dtype=_torch_dtype(cfg.dtype))
    mask = np.zeros((n, mask_words(h)), dtype=np.uint32)
    mean = np.zeros(n)
    rstd = np.zeros(n)
    rc = _lib().orc_linear_rs_fwd_rows(
        ctypes.byref(cfg), f, n, ids.ctypes.data, _ptr(x_rows), _ptr(w), _ptr(bias),
        _ptr(residual_rows), _ptr(gamma), _ptr(beta), _ptr(rout), _ptr(out),
        mask.ctypes.data, mean.ctypes.data, rstd.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle linear forward rejected the configuration ({rc})")
    return dict(residual_out=rout, norm_out=out, mask=mask,
                mean=mean if cfg.norm == LAYERNORM else None, rstd=rstd)


def ag_colpar_fwd(shards, w) -> torch.Tensor:
    """All-gather of the t shards, then the column-parallel linear X @ w^T
    rounded to bf16 (shards [rows/t, h] each, w [f_out, h])."""
    sh = [_cpu(x, BF16) for x in shards]
    w = _cpu(w, BF16)
    t, (per, h), f_out = len(sh), sh[0].shape, w.shape[0]
    out = torch.empty((t * per, f_out), dtype=torch.bfloat16)
    rc = _lib().orc_ag_colpar_fwd(t, per, h, f_out, _ptr_array(sh), _ptr(w), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle column-parallel forward rejected the shapes ({rc})")
    return out


# ----------------------------------------------------------------------------
# context parallelism: ring attention
# ----------------------------------------------------------------------------

def ring_attention(q, k, v, t: int, scale: float):
    """Ring attention over t ranks; q, k, v [bh, s, d] bf16.  Returns
    (out [bh, s, d] bf16, lse [bh, s] float64)."""
    q, k, v = (_cpu(x, BF16) for x in (q, k, v))
    bh, s, d = q.shape
    out = torch.empty((bh, s, d), dtype=torch.bfloat16)
    lse = np.zeros((bh, s))
    rc = _lib().orc_ring_attention(bh, s, d, t, scale, _ptr(q), _ptr(k), _ptr(v),
                                   _ptr(out), lse.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle ring attention rejected the shapes ({rc})")
    return out, lse


def ring_attention_rows(q_rows, rows, k, v, t: int, scale: float):
    """Ring attention of one head on selected query rows: q_rows [n, d]
    (the queries of tokens rows[i]), k, v [s, d]."""
    q_rows, k, v = (_cpu(x, BF16) for x in (q_rows, k, v))
    ids = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    s, d = k.shape
    out = torch.empty((len(ids), d), dtype=torch.bfloat16)
    lse = np.zeros(len(ids))
    rc = _lib().orc_ring_attention_rows(s, d, t, scale, _ptr(q_rows), ids.ctypes.data,
                                        len(ids), _ptr(k), _ptr(v), _ptr(out),
                                        lse.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle ring attention rejected the shapes ({rc})")
    return out, lse
