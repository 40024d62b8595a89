"""Build libvda.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc.

    python -m frame_wise_delta_vda_b200.build [--force]

The library is one translation unit (csrc/vda.cu includes the kernel
headers), linked as a shared object with the CUDA runtime linked statically,
so it loads next to PyTorch's own runtime without symbol clashes.  ptxas
resource usage (registers, spills, shared memory) is written to
_build/ptxas.log.
"""

from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libvda.so")
BUILD_DIR = os.path.join(ROOT, "_build")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found (set NVCC or put the CUDA toolkit on PATH)")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def up_to_date():
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in sources() + [__file__])


def build(force=False, verbose=True, extra_flags=None):
    if not force and up_to_date():
        return LIB
    os.makedirs(BUILD_DIR, exist_ok=True)
    cmd = [_nvcc(), "-O3", "-std=c++17", *ARCH_FLAGS, "-lineinfo", "-Xptxas", "-v",
           "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--shared", "-cudart", "static", "-Xlinker", "-Bsymbolic",
           "-I", INCLUDE, "-I", CSRC,
           "-o", LIB + ".tmp", os.path.join(CSRC, "vda.cu")]
    if extra_flags:
        cmd[1:1] = list(extra_flags)
    if verbose:
        print("[vda build]", " ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    with open(os.path.join(BUILD_DIR, "ptxas.log"), "w") as f:
        f.write(r.stdout)
        f.write(r.stderr)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libvda.so (see _build/ptxas.log)")
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv)
    print(LIB)
