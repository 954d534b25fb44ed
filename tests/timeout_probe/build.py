"""Build the test-only copy of the library whose bounded waits run out
(TEST INFRASTRUCTURE).

The library's own sources, compiled with two switches that product builds
never set: GDN_TEST_WITHHOLD_STATE_ARRIVAL drops the expect-tx arrival that
pairs with each kernel's first bulk copy of a sequence's data (the copy
still lands, but the barrier phase it belongs to never completes), and
GDN_WAIT_LIMIT_NS shortens every bounded wait to 2 ms.  Every kernel that
waits for such a copy (the on-chip chunked kernel, the three split state
kernels, the pipelined kernel) then takes its timeout path: GDN_DEV_TIMEOUT in the status word, no
further work, its copies allowed to land (bounded), TMEM freed."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
CSRC = os.path.join(ROOT, "gated_deltanet_recurrent_sigmoid_b200", "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libgdn_timeout.so")
WAIT_LIMIT_NS = 2_000_000


def build():
    deps = ([os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh"))] +
            [os.path.join(INCLUDE, "gdn_decode.h"), os.path.abspath(__file__)])
    if os.path.exists(LIB) and all(os.path.getmtime(d) <= os.path.getmtime(LIB) for d in deps):
        return LIB
    nvcc = "/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else "nvcc"
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-shared",
                    "-Xcompiler", "-fPIC,-fvisibility=hidden", "-DGDN_TEST_WITHHOLD_STATE_ARRIVAL",
                    f"-DGDN_WAIT_LIMIT_NS={WAIT_LIMIT_NS}ull", "-I", CSRC, "-I", INCLUDE, "-o", tmp,
                    os.path.join(CSRC, "gdn_decode_api.cu")], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build())
