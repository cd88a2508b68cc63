"""Build libnattn.so in-tree for sm_100a.

    python -m alternative_normalizers_b200.build [--verbose]

Compiles ``csrc/nattn_api.cu`` (which includes every kernel) into
``alternative_normalizers_b200/lib/libnattn.so`` with nvcc.  The CUDA runtime
is linked statically; the driver's tensor-map encoder is looked up at run
time, so the library needs no libcuda at link time and cross-compiles on a
machine without a GPU.
"""

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc")
OUT_DIR = os.path.join(HERE, "lib")
LIB = os.path.join(OUT_DIR, "libnattn.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"),
                 "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; set NVCC or put CUDA on PATH")


def sources():
    return sorted(os.path.join(SRC, f) for f in os.listdir(SRC)
                  if f.endswith((".cu", ".cuh")))


def up_to_date():
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    deps = sources() + [os.path.join(HERE, "..", "include", "nattn.h"),
                        os.path.abspath(__file__)]
    return all(os.path.getmtime(p) <= t for p in deps if os.path.exists(p))


def build(force=False, verbose=False, extra=()):
    """Compile the library if any source is newer than it.  Returns the path."""
    if not force and up_to_date():
        return LIB
    os.makedirs(OUT_DIR, exist_ok=True)
    tmp = LIB + ".tmp"
    cmd = [nvcc_path(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "--expt-relaxed-constexpr", "-I", os.path.join(HERE, "..", "include"),
           *extra, os.path.join(SRC, "nattn_api.cu"), "-o", tmp]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    v = "--verbose" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas" in sys.argv else []
    print(build(force="--force" in sys.argv, verbose=v, extra=extra))
