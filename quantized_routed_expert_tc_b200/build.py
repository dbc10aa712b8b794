"""Build libqrx.so (the CUDA library) in-tree for sm_100a with nvcc, and its
bounds-checked twin libqrx_check.so (-DQRX_CHECK: kernels test data-derived
indices against their buffers and report a miss through qrx_last_error)."""
from __future__ import annotations

import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libqrx.so")
CHECK_LIB = os.path.join(HERE, "libqrx_check.so")
NVCC_FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
              "-Xcompiler", "-fPIC", "-shared"]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(CSRC, "*.h")) +
                  [os.path.join(HERE, "..", "include", "qrx.h")])


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False, check: bool = False) -> str:
    """Compile csrc/qrx_api.cu (which includes every kernel) into libqrx.so, or
    with check=True into the bounds-checked libqrx_check.so."""
    lib = CHECK_LIB if check else LIB
    if not force and not stale(lib):
        return lib
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, *(["-DQRX_CHECK"] if check else []), os.path.join(CSRC, "qrx_api.cu"),
           "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force=True))
    print(build(force=True, check=True))
