"""Python binding of the B200 sequence-parallel boundary library.

A thin ctypes layer over ``libsp_region.so`` (C ABI in ``include/sp_region.h``):
it turns tensors into device pointers and a ``sp_cfg`` struct and calls the
entry point of the same name.  Every step of the boundary runs in the
library's CUDA kernels; there is no other implementation and no fallback.  If
the library is missing or cannot be loaded, importing this package raises.

The functions take torch CUDA tensors laid out as the header describes
(``[s, b, h]`` stored as ``[s*b, h]`` rows, h fastest) and enqueue work on
``stream`` (default: torch's current stream of the tensors' device).  They
raise ``SPError`` when the library rejects a call.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsp_region.so")

SP_OK, SP_ERR_INVALID_ARG, SP_ERR_UNSUPPORTED, SP_ERR_CUDA, \
    SP_ERR_DEVICE_TIMEOUT = range(5)
SP_F32, SP_BF16 = 0, 1
SP_LAYERNORM, SP_RMSNORM = 0, 1
SP_MAX_T = 64

# every symbol include/sp_region.h declares
EXPORTS = ("sp_rs_bias_dropout_add_norm_fwd", "sp_all_gather",
           "sp_rs_norm_dropout_bwd", "sp_bwd_workspace_bytes",
           "sp_activation_bytes", "sp_status_string", "sp_device_error",
           "sp_debug_wait_timeout", "sp_plan_count",
           "sp_rs_norm_dropout_bwd_noalloc", "sp_norm_all_gather_fwd",
           "sp_rowpar_linear_rs_fwd", "sp_linear_rs_bias_dropout_add_norm_fwd",
           "sp_ag_colpar_linear_fwd", "sp_rs_norm_dropout_bwd_ag",
           "sp_ring_attention_fwd", "sp_ring_attention_fwd_ws",
           "sp_ring_attention_workspace_bytes")


class SPError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {_status_string(status)} ({status})")


class sp_cfg(ctypes.Structure):
    _fields_ = [("s", ctypes.c_int64), ("b", ctypes.c_int64),
                ("h", ctypes.c_int64), ("t", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("norm", ctypes.c_int32),
                ("eps", ctypes.c_float), ("p_drop", ctypes.c_float),
                ("seed", ctypes.c_uint64), ("offset", ctypes.c_uint64),
                ("fwd_plan", ctypes.c_int32), ("bwd_plan", ctypes.c_int32),
                ("row_begin", ctypes.c_int64), ("row_end", ctypes.c_int64),
                ("res_f32", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python sp_region_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    cfgp = ctypes.POINTER(sp_cfg)
    lib.sp_rs_bias_dropout_add_norm_fwd.argtypes = [
        cfgp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp]
    lib.sp_all_gather.argtypes = [cfgp, vp, vp, i32, vp]
    lib.sp_norm_all_gather_fwd.argtypes = [cfgp, vp, vp, vp, vp, i32, vp, vp,
                                           vp]
    lib.sp_rs_norm_dropout_bwd.argtypes = [
        cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
        ctypes.c_size_t, vp]
    lib.sp_bwd_workspace_bytes.argtypes = [cfgp, i32,
                                           ctypes.POINTER(ctypes.c_size_t)]
    lib.sp_activation_bytes.argtypes = [i64, i64, i64, i64, i32, i32,
                                        ctypes.c_double,
                                        ctypes.POINTER(ctypes.c_double)]
    lib.sp_status_string.argtypes = [ctypes.c_int]
    lib.sp_status_string.restype = ctypes.c_char_p
    lib.sp_device_error.argtypes = [i32, ctypes.POINTER(i32), i32]
    lib.sp_debug_wait_timeout.argtypes = [i64, vp, vp]
    lib.sp_plan_count.argtypes = [ctypes.POINTER(i32), ctypes.POINTER(i32)]
    lib.sp_rs_norm_dropout_bwd_noalloc.argtypes = [
        cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    lib.sp_rs_norm_dropout_bwd_ag.argtypes = [
        cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp,
        ctypes.c_size_t, vp]
    lib.sp_rowpar_linear_rs_fwd.argtypes = [cfgp, i64, vp, vp, vp, vp, vp, vp, vp]
    lib.sp_linear_rs_bias_dropout_add_norm_fwd.argtypes = [
        cfgp, i64, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp]
    lib.sp_ag_colpar_linear_fwd.argtypes = [cfgp, i64, vp, vp, vp, vp]
    lib.sp_ring_attention_fwd.argtypes = [cfgp, i32, ctypes.c_float, vp, vp, vp,
                                          vp, vp, vp]
    lib.sp_ring_attention_fwd_ws.argtypes = [cfgp, i32, ctypes.c_float, vp, vp,
                                             vp, vp, vp, vp, ctypes.c_size_t,
                                             vp]
    lib.sp_ring_attention_workspace_bytes.argtypes = [
        cfgp, i32, i32, ctypes.POINTER(ctypes.c_size_t)]
    for f in EXPORTS:
        getattr(lib, f).restype = (ctypes.c_char_p if f == "sp_status_string"
                                   else ctypes.c_int)
    return lib


_lib = _load()


def _status_string(status: int) -> str:
    return _lib.sp_status_string(status).decode()


def _check(fn: str, status: int) -> None:
    if status != SP_OK:
        raise SPError(fn, status)


def make_cfg(s: int, b: int, h: int, t: int, dtype="bf16",
             norm="layernorm", eps: float = 1e-5, p_drop: float = 0.0,
             seed: int = 0, offset: int = 0, fwd_plan: int = 0,
             bwd_plan: int = 0, row_begin: int = 0,
             row_end: int = 0, res_f32: bool = False) -> sp_cfg:
    """res_f32: the residual stream (residual, residual_out, the entry's x,
    dR_next, dresidual_in) is fp32 beside bf16 partials and outputs."""
    dt = {"f32": SP_F32, "bf16": SP_BF16, torch.float32: SP_F32,
          torch.bfloat16: SP_BF16}[dtype]
    nm = {"layernorm": SP_LAYERNORM, "rmsnorm": SP_RMSNORM}[norm]
    return sp_cfg(s=s, b=b, h=h, t=t, dtype=dt, norm=nm, eps=eps,
                  p_drop=p_drop, seed=seed, offset=offset, fwd_plan=fwd_plan,
                  bwd_plan=bwd_plan, row_begin=row_begin, row_end=row_end,
                  res_f32=1 if res_f32 else 0)


def _p(x: Optional[torch.Tensor]) -> Optional[int]:
    return None if x is None else x.data_ptr()


def _ptrs(ts: Sequence[torch.Tensor]):
    arr = (ctypes.c_void_p * len(ts))()
    for i, x in enumerate(ts):
        arr[i] = x.data_ptr()
    return arr


def _stream(stream, like: torch.Tensor) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(like.device)
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def sp_rs_bias_dropout_add_norm_fwd(cfg: sp_cfg, partials, bias, residual,
                                    gamma, beta, residual_out, gathered,
                                    mask_bits=None, mean=None, rstd=None,
                                    stream=None) -> None:
    """Forward: reduce-scatter + bias + dropout + residual + norm, with the
    all-gather written to every tensor in ``gathered``."""
    gathered = list(gathered)
    _check("sp_rs_bias_dropout_add_norm_fwd",
           _lib.sp_rs_bias_dropout_add_norm_fwd(
               ctypes.byref(cfg), _ptrs(partials), _p(bias), _p(residual),
               _p(gamma), _p(beta), _p(residual_out), _ptrs(gathered),
               len(gathered), _p(mask_bits), _p(mean), _p(rstd),
               _stream(stream, residual)))


def sp_norm_all_gather_fwd(cfg: sp_cfg, x, gamma, beta, gathered, mean=None,
                           rstd=None, stream=None) -> None:
    """Entry into a TP region: per-token norm of x, all-gathered into every
    tensor in ``gathered``."""
    gathered = list(gathered)
    _check("sp_norm_all_gather_fwd",
           _lib.sp_norm_all_gather_fwd(
               ctypes.byref(cfg), _p(x), _p(gamma), _p(beta), _ptrs(gathered),
               len(gathered), _p(mean), _p(rstd), _stream(stream, x)))


def sp_all_gather(cfg: sp_cfg, shards, outs, stream=None) -> None:
    """All-gather of t sequence shards into every tensor in ``outs``."""
    outs = list(outs)
    _check("sp_all_gather",
           _lib.sp_all_gather(ctypes.byref(cfg), _ptrs(shards), _ptrs(outs),
                              len(outs), _stream(stream, shards[0])))


def sp_bwd_workspace_bytes(cfg: sp_cfg, device=None) -> int:
    dev = torch.cuda.current_device() if device is None else int(device)
    n = ctypes.c_size_t(0)
    _check("sp_bwd_workspace_bytes",
           _lib.sp_bwd_workspace_bytes(ctypes.byref(cfg), dev,
                                       ctypes.byref(n)))
    return int(n.value)


def sp_rs_norm_dropout_bwd(cfg: sp_cfg, dn_partials, dR_next, residual_out,
                           gamma, mask_bits, mean, rstd, dresidual_in, dY,
                           dgamma, dbeta, dbias, workspace,
                           stream=None) -> None:
    """Backward: reduce-scatter of dn + norm / residual / dropout backward,
    dY all-gathered, parameter gradients summed over all tokens."""
    _check("sp_rs_norm_dropout_bwd",
           _lib.sp_rs_norm_dropout_bwd(
               ctypes.byref(cfg), _ptrs(dn_partials), _p(dR_next),
               _p(residual_out), _p(gamma), _p(mask_bits), _p(mean), _p(rstd),
               _p(dresidual_in), _p(dY), _p(dgamma), _p(dbeta), _p(dbias),
               _p(workspace), workspace.numel() * workspace.element_size(),
               _stream(stream, residual_out)))


def sp_rs_norm_dropout_bwd_ag(cfg: sp_cfg, dn_partials, dR_next, residual_out,
                              gamma, mask_bits, mean, rstd, dresidual_in, dY,
                              dgamma, dbeta, dbias, workspace,
                              stream=None) -> None:
    """The backward with every row of dY written to each buffer in ``dY``
    (every rank's copy: the all-gather done by the kernel's stores)."""
    dY = list(dY)
    _check("sp_rs_norm_dropout_bwd_ag",
           _lib.sp_rs_norm_dropout_bwd_ag(
               ctypes.byref(cfg), _ptrs(dn_partials), _p(dR_next),
               _p(residual_out), _p(gamma), _p(mask_bits), _p(mean), _p(rstd),
               _p(dresidual_in), _ptrs(dY), len(dY), _p(dgamma), _p(dbeta),
               _p(dbias), _p(workspace),
               workspace.numel() * workspace.element_size(),
               _stream(stream, residual_out)))


def sp_rs_norm_dropout_bwd_noalloc(cfg: sp_cfg, dn_partials, dR_next,
                                   residual_out, gamma, mask_bits, mean, rstd,
                                   dresidual_in, dY, dgamma, dbeta, dbias,
                                   stream=None) -> None:
    """The backward with its scratch in the library's fixed 64 MiB device
    array instead of a caller buffer, for callers that cannot allocate device
    memory at this point.  Calls that overlap on the GPU share that array and
    must be serialised; the first call on a device looks up the array's
    address and should come before any stream capture."""
    _check("sp_rs_norm_dropout_bwd_noalloc",
           _lib.sp_rs_norm_dropout_bwd_noalloc(
               ctypes.byref(cfg), _ptrs(dn_partials), _p(dR_next),
               _p(residual_out), _p(gamma), _p(mask_bits), _p(mean), _p(rstd),
               _p(dresidual_in), _p(dY), _p(dgamma), _p(dbeta), _p(dbias),
               _stream(stream, residual_out)))


def sp_rowpar_linear_rs_fwd(cfg: sp_cfg, f: int, x, w, bias, residual,
                            residual_out, mask_bits=None, stream=None) -> None:
    """Row-parallel linear x [rows, f] @ w [h, f]^T whose t rank partials
    are reduced in the GEMM's accumulator, then bias, dropout and the
    residual add into residual_out (and mask_bits)."""
    _check("sp_rowpar_linear_rs_fwd",
           _lib.sp_rowpar_linear_rs_fwd(
               ctypes.byref(cfg), f, _p(x), _p(w), _p(bias), _p(residual),
               _p(residual_out), _p(mask_bits), _stream(stream, x)))


def sp_linear_rs_bias_dropout_add_norm_fwd(cfg: sp_cfg, f: int, x, w, bias,
                                           residual, gamma, beta,
                                           residual_out, gathered,
                                           mask_bits=None, mean=None,
                                           rstd=None, stream=None) -> None:
    """The forward boundary with its reduce-scatter in the row-parallel
    GEMM: sp_rowpar_linear_rs_fwd, then the norm and the all-gather."""
    gathered = list(gathered)
    _check("sp_linear_rs_bias_dropout_add_norm_fwd",
           _lib.sp_linear_rs_bias_dropout_add_norm_fwd(
               ctypes.byref(cfg), f, _p(x), _p(w), _p(bias), _p(residual),
               _p(gamma), _p(beta), _p(residual_out), _ptrs(gathered),
               len(gathered), _p(mask_bits), _p(mean), _p(rstd),
               _stream(stream, x)))


def sp_ag_colpar_linear_fwd(cfg: sp_cfg, f_out: int, shards, w, out,
                            stream=None) -> None:
    """Column-parallel linear on the all-gathered shards: out [N, f_out] =
    concat(shards) @ w [f_out, h]^T, reading the shards directly."""
    _check("sp_ag_colpar_linear_fwd",
           _lib.sp_ag_colpar_linear_fwd(
               ctypes.byref(cfg), f_out, _ptrs(shards), _p(w), _p(out),
               _stream(stream, out)))


def sp_ring_attention_fwd(cfg: sp_cfg, heads: int, scale: float, q, k, v, out,
                          lse=None, stream=None) -> None:
    """Ring attention over cfg.t context-parallel ranks: q, k, v, out
    [b, heads, s, 128] bf16, lse [b, heads, s] fp32 or None."""
    _check("sp_ring_attention_fwd",
           _lib.sp_ring_attention_fwd(ctypes.byref(cfg), heads, scale, _p(q),
                                      _p(k), _p(v), _p(out), _p(lse),
                                      _stream(stream, out)))


def sp_ring_attention_workspace_bytes(cfg: sp_cfg, heads: int,
                                      device=None) -> int:
    dev = torch.cuda.current_device() if device is None else int(device)
    n = ctypes.c_size_t(0)
    _check("sp_ring_attention_workspace_bytes",
           _lib.sp_ring_attention_workspace_bytes(ctypes.byref(cfg), heads, dev,
                                                  ctypes.byref(n)))
    return int(n.value)


def sp_ring_attention_fwd_ws(cfg: sp_cfg, heads: int, scale: float, q, k, v,
                             out, lse=None, workspace=None,
                             stream=None) -> None:
    """Ring attention with the last round of units split over the SMs
    (workspace: sp_ring_attention_workspace_bytes bytes, or None when 0)."""
    nbytes = 0 if workspace is None else \
        workspace.numel() * workspace.element_size()
    _check("sp_ring_attention_fwd_ws",
           _lib.sp_ring_attention_fwd_ws(ctypes.byref(cfg), heads, scale,
                                         _p(q), _p(k), _p(v), _p(out), _p(lse),
                                         _p(workspace), nbytes,
                                         _stream(stream, out)))


def sp_activation_bytes(s: int, b: int, h: int, a: int, t: int, mode: int,
                        bytes_per_elem: float) -> float:
    """mode 0: A_layer, 1: A_TP, 2: A_TP+SP, times bytes_per_elem."""
    out = ctypes.c_double(0.0)
    _check("sp_activation_bytes",
           _lib.sp_activation_bytes(s, b, h, a, t, mode, bytes_per_elem,
                                    ctypes.byref(out)))
    return out.value


def sp_device_error(device=None, clear: bool = True) -> int:
    dev = torch.cuda.current_device() if device is None else int(device)
    code = ctypes.c_int32(0)
    _check("sp_device_error",
           _lib.sp_device_error(dev, ctypes.byref(code), int(clear)))
    return int(code.value)


def sp_debug_wait_timeout(limit_ns: int, status: torch.Tensor,
                          stream=None) -> None:
    _check("sp_debug_wait_timeout",
           _lib.sp_debug_wait_timeout(limit_ns, _p(status),
                                      _stream(stream, status)))


def sp_status_string(status: int) -> str:
    return _status_string(status)


def sp_plan_count():
    """(forward plans, backward plans): valid hint values are 1..count."""
    f, b = ctypes.c_int32(0), ctypes.c_int32(0)
    _check("sp_plan_count", _lib.sp_plan_count(ctypes.byref(f),
                                                ctypes.byref(b)))
    return int(f.value), int(b.value)
