"""Build step of the SP boundary library: nvcc -> libsp_region.so (in-tree).

Run ``python sp_region_b200/build.py`` (``__graft_entry__.build()`` loads this
file by path).  It is run as a file, not as ``sp_region_b200.build``, because
importing the package loads the library that this script builds.
The library is compiled for sm_100a only and links the CUDA runtime
statically, so it loads next to any PyTorch build.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "sp_region.cu")
DEPS = [os.path.join(HERE, "csrc", f) for f in
        ("sp_region.cu", "sp_device.cuh", "sp_fwd.cuh", "sp_bwd.cuh",
         "sp_gather.cuh", "sp_entry.cuh")] + [os.path.join(ROOT, "include", "sp_region.h")]
LIB = os.path.join(HERE, "libsp_region.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
         "-lineinfo", "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr",
         "-I", os.path.join(ROOT, "include")]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    cmd = [NVCC] + FLAGS + (["-Xptxas", "-v"] if verbose_ptxas else []) + \
        ["-o", LIB + ".tmp", SRC]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv)
    print(LIB)
