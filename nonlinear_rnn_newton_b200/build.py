"""Build libpararnn.so (the C-ABI CUDA library) in-tree for sm_100a.

    python -m nonlinear_rnn_newton_b200.build [--force] [--verbose]

nvcc cross-compiles without a GPU.  The library links the CUDA runtime
statically and reaches the driver API only through cudaGetDriverEntryPoint,
so it loads on a machine without a GPU (its entry points then report a CUDA
error).
"""
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libpararnn.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC",
         "-Xcompiler", "-fvisibility=hidden", "-shared", "-cudart", "static"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(CSRC, "*.h")) + [os.path.join(INCLUDE, "pararnn.h")])


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False, out: str = LIB, defines=()) -> str:
    """Compile the library to `out`; `defines` are extra -D tuning macros."""
    if not force and out == LIB and not defines and up_to_date():
        return LIB
    cmd = [NVCC, *ARCH, *FLAGS, *[f"-D{d}" for d in defines], "-I", INCLUDE, "-I", CSRC,
           os.path.join(CSRC, "pararnn_capi.cu"), "-o", out + ".tmp"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
