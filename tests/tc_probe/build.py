"""Build the test-only tensor-core probe library (TEST INFRASTRUCTURE)."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
CSRC = os.path.join(ROOT, "gated_deltanet_recurrent_sigmoid_b200", "csrc")
LIB = os.path.join(HERE, "libtc_probe.so")
SRC = os.path.join(HERE, "tc_gemm_probe.cu")


def build():
    deps = [SRC] + [os.path.join(CSRC, f) for f in ("tc_sm100.cuh", "mbarrier_sm100.cuh")]
    if os.path.exists(LIB) and all(os.path.getmtime(d) <= os.path.getmtime(LIB) for d in deps):
        return LIB
    nvcc = "/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else "nvcc"
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17", "-shared",
                    "-Xcompiler", "-fPIC,-fvisibility=hidden", "-I", CSRC, "-I", os.path.join(ROOT, "include"),
                    "-o", LIB, SRC], check=True)
    return LIB


if __name__ == "__main__":
    print(build())
