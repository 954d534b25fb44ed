"""Build ``libgdn_decode.so`` (the C-ABI library) for sm_100a with nvcc.

The library is built in-tree next to this file.  ``build()`` rebuilds only
when a source or header is newer than the library (or ``force=True``), and
returns the library path.  ``ptxas_report()`` returns nvcc's ``-Xptxas -v``
resource lines (registers, spills, shared memory) of the current sources.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libgdn_decode.so"
LIB_PATH = os.path.join(PKG, LIB_NAME)

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC,-fvisibility=hidden",
                     "-I", INCLUDE, "-I", CSRC, "--threads", "4"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libgdn_decode.so")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps() -> list[str]:
    return (sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
            + glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)])


def stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    built = os.path.getmtime(LIB_PATH)
    return any(os.path.getmtime(d) > built for d in _deps())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every CUDA source into the in-tree shared library."""
    if not force and not stale():
        return LIB_PATH
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, "-o", tmp, *sources()]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


def ptxas_report() -> str:
    """Registers / spills / shared memory of every kernel (nvcc -Xptxas -v)."""
    out = os.path.join(PKG, f".ptxas_probe{os.getpid()}.so")
    try:
        res = subprocess.run([nvcc(), *NVCC_FLAGS, "-Xptxas", "-v", "-o", out, *sources()],
                             check=True, capture_output=True, text=True)
    finally:
        if os.path.exists(out):
            os.remove(out)
    return "\n".join(l for l in res.stderr.splitlines() if "ptxas" in l)


if __name__ == "__main__":
    if "--ptxas" in sys.argv:
        print(ptxas_report())
    else:
        print(build(force="--force" in sys.argv, verbose=True))
