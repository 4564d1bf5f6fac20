"""Build libnsa.so (the C-ABI library) in-tree for sm_100a with nvcc."""
from __future__ import annotations

import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
SO = os.path.join(HERE, "libnsa.so")

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  [os.path.join(HERE, "..", "include", "nsa.h")])


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile csrc/nsa_capi.cu (one translation unit) into libnsa.so when stale."""
    newest = max(os.path.getmtime(s) for s in sources())
    if not force and os.path.exists(SO) and os.path.getmtime(SO) >= newest:
        return SO
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = SO + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, "-o", tmp, os.path.join(CSRC, "nsa_capi.cu")]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(tmp, SO)
    return SO


if __name__ == "__main__":
    print(build(force=True, verbose=True))
