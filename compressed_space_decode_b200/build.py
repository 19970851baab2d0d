"""Build libisoquant.so (sm_100a) in-tree with nvcc.

The library is plain CUDA C++ behind the C ABI in include/isoquant.h; no
torch headers are involved, so it is compiled directly with nvcc.
"""
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC_DIR = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "libisoquant.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-I", os.path.join(ROOT, "include"),
]


def sources():
    return sorted(glob.glob(os.path.join(SRC_DIR, "*.cu")))


def _stale():
    if not os.path.exists(OUT):
        return True
    t = os.path.getmtime(OUT)
    deps = sources() + glob.glob(os.path.join(SRC_DIR, "*.cuh")) + [os.path.join(ROOT, "include", "isoquant.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force=False, verbose=False, extra=()):
    if not force and not _stale():
        return OUT
    cmd = [NVCC] + FLAGS + list(extra) + ["-o", OUT + ".tmp"] + sources()
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    # -v: register and shared-memory report; --nvtx: NVTX ranges around the C-ABI calls
    extra = (["-Xptxas", "-v"] if "-v" in sys.argv else []) + (["-DISOQUANT_NVTX"] if "--nvtx" in sys.argv else [])
    print(build(force=True, verbose=True, extra=extra))
