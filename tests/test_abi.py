"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and its host-only logic (closed forms, status strings,
argument validation before any device call) behaves as documented."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sp_region.h")
LIB = os.path.join(ROOT, "sp_region_b200", "libsp_region.so")


def _header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(sp_\w+)\s*\(", src,
                       flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "sp_region_build", os.path.join(ROOT, "sp_region_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    return ctypes.CDLL(LIB)


def test_header_declares_the_boundary_calls():
    names = _header_functions()
    for required in ("sp_rs_bias_dropout_add_norm_fwd", "sp_all_gather",
                     "sp_rs_norm_dropout_bwd", "sp_activation_bytes"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in _header_functions():
        assert hasattr(lib, name), name


def test_binding_covers_every_declared_symbol():
    import sp_region_b200 as sp
    assert sorted(sp.EXPORTS) == _header_functions()
    for name in _header_functions():
        assert callable(getattr(sp, name)), name


def test_status_strings():
    import sp_region_b200 as sp
    assert sp.sp_status_string(0) == "ok"
    assert "invalid" in sp.sp_status_string(1)
    assert sp.sp_status_string(99) == "unknown status"


def test_activation_bytes_matches_oracle(orc):
    import sp_region_b200 as sp
    for (s, b, h, a, t) in [(2048, 4, 12288, 96, 8), (32768, 1, 12288, 96, 16),
                            (4096, 1, 8192, 64, 8), (4, 1, 4, 1, 2),
                            (2048, 4, 6144, 48, 1)]:
        for mode in (0, 1, 2):
            for bpe in (1.0, 2.0):
                got = sp.sp_activation_bytes(s, b, h, a, t, mode, bpe)
                ref = orc.activation_bytes(s, b, h, a, t, mode, bpe)
                assert got == pytest.approx(ref, rel=1e-15)


def test_activation_bytes_rejects_bad_arguments():
    import sp_region_b200 as sp
    for args in [(0, 1, 1, 1, 1, 0, 2.0), (1, 1, 1, 1, 0, 0, 2.0),
                 (1, 1, 1, 1, 1, 3, 2.0), (1, 1, 1, 1, 1, 0, 0.0)]:
        with pytest.raises(sp.SPError) as e:
            sp.sp_activation_bytes(*args)
        assert e.value.status == sp.SP_ERR_INVALID_ARG


def _fake_call_fwd(lib, cfg, t, n_gathered=1, ptr=0x1000):
    """Call the forward with fake (never dereferenced) pointers; every case
    here must be rejected by host validation before any CUDA call."""
    import sp_region_b200 as sp
    parts = (ctypes.c_void_p * max(t, 1))(*([ptr] * max(t, 1)))
    outs = (ctypes.c_void_p * max(n_gathered, 1))(*([ptr] * max(n_gathered, 1)))
    return lib.sp_rs_bias_dropout_add_norm_fwd(
        ctypes.byref(cfg), parts, None, ctypes.c_void_p(ptr),
        ctypes.c_void_p(ptr), None, ctypes.c_void_p(ptr), outs, n_gathered,
        None, None, None, None)


@pytest.mark.parametrize("bad", [
    dict(s=6, t=4),               # s % t != 0
    dict(t=0), dict(t=65),        # t out of range
    dict(h=0), dict(s=0), dict(b=0),
    dict(p_drop=1.0), dict(p_drop=-0.1), dict(p_drop=float("nan")),
    dict(eps=0.0), dict(eps=float("inf")),
    dict(dtype=7), dict(norm=5),
    dict(s=2 ** 33, t=1),         # token row beyond the 32-bit counter
    dict(res_f32=2), dict(res_f32=-1),   # residual-stream flag is 0 or 1
])
def test_forward_validation_rejects_before_launch(lib, bad):
    import sp_region_b200 as sp
    kw = dict(s=8, b=2, h=64, t=4, dtype="bf16", norm="layernorm", eps=1e-5,
              p_drop=0.1)
    cfg = sp.make_cfg(**{k: v for k, v in kw.items()
                         if k not in ("dtype", "norm")},
                      dtype="bf16", norm="layernorm")
    for k, v in bad.items():
        setattr(cfg, k, v)
    t = max(1, min(int(cfg.t), 64))
    assert _fake_call_fwd(lib, cfg, t) == sp.SP_ERR_INVALID_ARG


def test_forward_rejects_null_and_misaligned(lib):
    import sp_region_b200 as sp
    cfg = sp.make_cfg(8, 2, 64, 4, dtype="bf16", p_drop=0.1)
    # n_gathered out of range
    assert _fake_call_fwd(lib, cfg, 4, n_gathered=0) == sp.SP_ERR_INVALID_ARG
    assert _fake_call_fwd(lib, cfg, 4, n_gathered=65) == sp.SP_ERR_INVALID_ARG
    # a pointer not aligned to the element size
    assert _fake_call_fwd(lib, cfg, 4, ptr=0x1001) == sp.SP_ERR_INVALID_ARG
    # NULL residual
    parts = (ctypes.c_void_p * 4)(*([0x1000] * 4))
    outs = (ctypes.c_void_p * 1)(0x1000)
    rc = lib.sp_rs_bias_dropout_add_norm_fwd(
        ctypes.byref(cfg), parts, None, None, ctypes.c_void_p(0x1000), None,
        ctypes.c_void_p(0x1000), outs, 1, None, None, None, None)
    assert rc == sp.SP_ERR_INVALID_ARG


def test_backward_validation(lib):
    import sp_region_b200 as sp
    cfg = sp.make_cfg(8, 2, 64, 4, dtype="bf16", p_drop=0.1)
    P = ctypes.c_void_p(0x1000)
    parts = (ctypes.c_void_p * 4)(*([0x1000] * 4))
    # p > 0 needs the mask
    rc = lib.sp_rs_norm_dropout_bwd(ctypes.byref(cfg), parts, None, P, P, None,
                                    P, P, P, P, P, None, None, P, 1 << 20, None)
    assert rc == sp.SP_ERR_INVALID_ARG
    # LayerNorm needs mean
    rc = lib.sp_rs_norm_dropout_bwd(ctypes.byref(cfg), parts, None, P, P, P,
                                    None, P, P, P, P, None, None, P, 1 << 20,
                                    None)
    assert rc == sp.SP_ERR_INVALID_ARG
    # workspace must be 16-byte aligned
    rc = lib.sp_rs_norm_dropout_bwd(ctypes.byref(cfg), parts, None, P, P, P,
                                    P, P, P, P, P, None, None,
                                    ctypes.c_void_p(0x1008), 1 << 20, None)
    assert rc == sp.SP_ERR_INVALID_ARG


def test_all_gather_validation(lib):
    import sp_region_b200 as sp
    cfg = sp.make_cfg(8, 2, 64, 4, dtype="bf16")
    sh = (ctypes.c_void_p * 4)(*([0x1000] * 4))
    outs = (ctypes.c_void_p * 1)(0x1000)
    assert lib.sp_all_gather(ctypes.byref(cfg), sh, outs, 0, None) == \
        sp.SP_ERR_INVALID_ARG
    cfg.s = 7
    assert lib.sp_all_gather(ctypes.byref(cfg), sh, outs, 1, None) == \
        sp.SP_ERR_INVALID_ARG


def test_ring_attention_validation(lib):
    """Both attention calls reject bad shapes, NULL or misaligned pointers, a
    bad scale and a misaligned workspace before any device query."""
    import sp_region_b200 as sp
    vp, f = ctypes.c_void_p, ctypes.c_float
    lib.sp_ring_attention_fwd.argtypes = [ctypes.c_void_p, ctypes.c_int32, f, vp, vp, vp, vp,
                                          vp, vp]
    lib.sp_ring_attention_fwd_ws.argtypes = [ctypes.c_void_p, ctypes.c_int32, f, vp, vp, vp,
                                             vp, vp, vp, ctypes.c_size_t, vp]
    cfg = sp.make_cfg(256, 1, 128, 2, dtype="bf16")
    ok, odd = vp(0x1000), vp(0x1008)
    ws_args = lambda *p: lib.sp_ring_attention_fwd_ws(ctypes.byref(cfg), 1, 0.1, *p)
    assert ws_args(None, ok, ok, ok, None, ok, 1 << 20, None) == sp.SP_ERR_INVALID_ARG
    assert ws_args(ok, ok, ok, odd, None, ok, 1 << 20, None) == sp.SP_ERR_INVALID_ARG
    assert ws_args(ok, ok, ok, ok, None, odd, 1 << 20, None) == sp.SP_ERR_INVALID_ARG
    assert lib.sp_ring_attention_fwd_ws(ctypes.byref(cfg), 1, -1.0, ok, ok, ok, ok, None, ok,
                                        1 << 20, None) == sp.SP_ERR_INVALID_ARG
    assert lib.sp_ring_attention_fwd(ctypes.byref(cfg), 0, 0.1, ok, ok, ok, ok, None,
                                     None) == sp.SP_ERR_INVALID_ARG
    bad = sp.make_cfg(384, 1, 128, 2, dtype="bf16")   # s / t = 192: not a 128-key tile
    assert lib.sp_ring_attention_fwd_ws(ctypes.byref(bad), 1, 0.1, ok, ok, ok, ok, None, ok,
                                        1 << 20, None) == sp.SP_ERR_UNSUPPORTED


def test_linears_validation(lib):
    """The tensor-core linears reject missing or misaligned operands, an inner
    dimension the ranks cannot split, shapes no kernel takes, and a missing
    dropout mask, before any device query."""
    import sp_region_b200 as sp
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    lib.sp_rowpar_linear_rs_fwd.argtypes = [vp, i64, vp, vp, vp, vp, vp, vp, vp]
    lib.sp_ag_colpar_linear_fwd.argtypes = [vp, i64, vp, vp, vp, vp]
    ok, odd = vp(0x1000), vp(0x1008)
    cfg = sp.make_cfg(256, 1, 256, 4, dtype="bf16", p_drop=0.1)
    row = lambda f, x, w, res, rout, mask: lib.sp_rowpar_linear_rs_fwd(
        ctypes.byref(cfg), f, x, w, None, res, rout, mask, None)
    assert row(512, None, ok, ok, ok, ok) == sp.SP_ERR_INVALID_ARG    # no x
    assert row(510, ok, ok, ok, ok, ok) == sp.SP_ERR_INVALID_ARG      # f % t != 0
    assert row(516, ok, ok, ok, ok, ok) == sp.SP_ERR_UNSUPPORTED      # f % 8 != 0
    assert row(512, ok, ok, ok, ok, None) == sp.SP_ERR_INVALID_ARG    # p > 0, no mask
    assert row(512, odd, ok, ok, ok, ok) == sp.SP_ERR_INVALID_ARG     # misaligned x
    f32 = sp.make_cfg(256, 1, 256, 4, dtype="f32")
    assert lib.sp_rowpar_linear_rs_fwd(ctypes.byref(f32), 512, ok, ok, None, ok, ok, None,
                                       None) == sp.SP_ERR_UNSUPPORTED  # bf16 only
    cfg_c = sp.make_cfg(256, 1, 256, 4, dtype="bf16")
    shards = (vp * 4)(*([0x1000] * 4))
    col = lambda f_out, sh, w, out: lib.sp_ag_colpar_linear_fwd(
        ctypes.byref(cfg_c), f_out, sh, w, out, None)
    assert col(512, None, ok, ok) == sp.SP_ERR_INVALID_ARG           # no shards
    assert col(0, shards, ok, ok) == sp.SP_ERR_INVALID_ARG           # no output features
    assert col(516, shards, ok, ok) == sp.SP_ERR_UNSUPPORTED         # f_out % 8 != 0
    ragged = sp.make_cfg(384, 1, 256, 4, dtype="bf16")               # 96 rows a shard
    assert lib.sp_ag_colpar_linear_fwd(ctypes.byref(ragged), 512, shards, ok, ok,
                                       None) == sp.SP_ERR_UNSUPPORTED


def test_fp32_residual_stream_needs_fp32_alignment(lib):
    """With res_f32 the residual-stream tensors are fp32: a pointer aligned
    for bf16 only is rejected before any launch, forward and backward."""
    import sp_region_b200 as sp
    cfg = sp.make_cfg(8, 2, 64, 4, dtype="bf16", p_drop=0.0, res_f32=True)
    A, M = ctypes.c_void_p(0x1000), ctypes.c_void_p(0x1002)
    parts = (ctypes.c_void_p * 4)(*([0x1000] * 4))
    outs = (ctypes.c_void_p * 1)(0x1000)
    for residual, rout in ((M, A), (A, M)):
        rc = lib.sp_rs_bias_dropout_add_norm_fwd(
            ctypes.byref(cfg), parts, None, residual, A, None, rout, outs, 1,
            None, None, None, None)
        assert rc == sp.SP_ERR_INVALID_ARG
    rc = lib.sp_norm_all_gather_fwd(ctypes.byref(cfg), M, A, None, outs, 1,
                                    None, None, None)
    assert rc == sp.SP_ERR_INVALID_ARG
    # backward: x (residual_out), dR_next and dresidual_in are fp32
    for drn, x, dres in ((M, A, A), (A, M, A), (A, A, M)):
        rc = lib.sp_rs_norm_dropout_bwd(ctypes.byref(cfg), parts, drn, x, A,
                                        None, A, A, dres, A, A, None, None, A,
                                        1 << 20, None)
        assert rc == sp.SP_ERR_INVALID_ARG
