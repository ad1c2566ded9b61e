"""The C ABI from plain C (no Python, no torch): tests/c/abi_from_c.c is
compiled with gcc against include/sp_region.h, linked with the library, run on
the CPU, and its answers checked against the oracle and the header."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "sp_region_b200")


def test_c_program_links_and_calls_the_abi(tmp_path, orc):
    if not os.path.exists(os.path.join(LIBDIR, "libsp_region.so")):
        pytest.fail("libsp_region.so is not built")
    exe = tmp_path / "abi_from_c"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror",
                    "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_from_c.c"),
                    "-L", LIBDIR, "-lsp_region", f"-Wl,-rpath,{LIBDIR}",
                    "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True,
                         text=True).stdout
    got = dict(line.split(" ", 1) for line in out.strip().splitlines())
    import sp_region_b200 as sp
    nf, nb = sp.sp_plan_count()
    assert got["plans"] == f"{nf} {nb}"
    want = orc.activation_bytes(2048, 1, 12288, 96, 8, 2, 2.0)
    assert abs(float(got["activation"]) - want) <= 0.05
    assert int(got["bad_mode"]) == sp.SP_ERR_INVALID_ARG
    assert got["status"] == sp.sp_status_string(sp.SP_ERR_INVALID_ARG)
    assert int(got["bad_cfg"]) == sp.SP_ERR_INVALID_ARG
    assert int(got["attn_ragged"]) == sp.SP_ERR_UNSUPPORTED
    assert int(got["attn_head64"]) == sp.SP_ERR_UNSUPPORTED
    assert int(got["attn_null"]) == sp.SP_ERR_INVALID_ARG
