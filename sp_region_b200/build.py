"""Build step of the SP boundary library: nvcc -> libsp_region.so (in-tree).

Run ``python sp_region_b200/build.py`` (``__graft_entry__.build()`` loads this
file by path).  It is run as a file, not as ``sp_region_b200.build``, because
importing the package loads the library that this script builds.

The library is compiled for sm_100a only and links the CUDA runtime
statically, so it loads next to any PyTorch build.  Its translation units are
compiled in parallel: the host entry points with the small kernels
(``sp_region.cu``), the tensor-core linears (``sp_gemm.cu``), and one unit
per (I/O dtype, norm) pair for each of the two fast streaming kernels, whose
plan tables make up most of the device code (``sp_inst_fwd.cu`` /
``sp_inst_bwd.cu`` with ``-DSP_T_BF16 -DSP_LN``).
"""
import concurrent.futures
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OBJDIR = os.path.join(HERE, "_build")
HEADERS = [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC))
           if f.endswith((".cuh", ".h"))] + \
    [os.path.join(ROOT, "include", "sp_region.h")]
LIB = os.path.join(HERE, "libsp_region.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
         "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I", os.path.join(ROOT, "include")]


def units():
    """(object path, source path, extra flags) of every translation unit."""
    out = [(os.path.join(OBJDIR, "sp_region.o"),
            os.path.join(CSRC, "sp_region.cu"), []),
           (os.path.join(OBJDIR, "sp_gemm.o"),
            os.path.join(CSRC, "sp_gemm.cu"), [])]
    for kind in ("fwd", "bwd"):
        for tb, tname in ((1, "bf16"), (0, "f32")):
            for ln, nname in ((1, "ln"), (0, "rms")):
                out.append((os.path.join(OBJDIR, f"sp_inst_{kind}_{tname}_{nname}.o"),
                            os.path.join(CSRC, f"sp_inst_{kind}.cu"),
                            [f"-DSP_T_BF16={tb}", f"-DSP_LN={ln}"]))
    return out


def sources():
    """Every file the library is built from (for staleness and hashing)."""
    return sorted({src for _, src, _ in units()} | set(HEADERS))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def up_to_date() -> bool:
    return not _stale(LIB, sources())


def _compile(unit, verbose_ptxas):
    obj, src, extra = unit
    cmd = [NVCC] + FLAGS + extra + (["-Xptxas", "-v"] if verbose_ptxas else []) + \
        ["-c", "-o", obj + ".tmp", src]
    subprocess.run(cmd, check=True)
    os.replace(obj + ".tmp", obj)
    return obj


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(OBJDIR, exist_ok=True)
    todo = [u for u in units()
            if force or verbose_ptxas or _stale(u[0], [u[1]] + HEADERS)]
    jobs = max(1, min(len(todo), os.cpu_count() or 1))
    with concurrent.futures.ThreadPoolExecutor(jobs) as ex:
        for f in [ex.submit(_compile, u, verbose_ptxas) for u in todo]:
            f.result()
    cmd = [NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
           "-o", LIB + ".tmp"] + [u[0] for u in units()]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv)
    print(LIB)
