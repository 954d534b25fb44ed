"""Compile the C oracle into ``oracle/libgdn_oracle.so``.

TEST INFRASTRUCTURE ONLY.  Plain gcc, no vectorising or fast-math flags, and
``-ffp-contract=off`` so that every multiply and add rounds on its own as the
C source states it.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCES = ["gdn_oracle.c", "gdn_oracle_f32.c", "gdn_oracle_fin.c"]
HEADERS = ["gdn_oracle.h"]
LIB_PATH = os.path.join(HERE, "libgdn_oracle.so")

CFLAGS = ["-std=c11", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
          "-fno-fast-math", "-Wall", "-Wextra", "-Werror"]


def _stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    built = os.path.getmtime(LIB_PATH)
    deps = SOURCES + HEADERS + [os.path.basename(__file__)]
    return any(os.path.getmtime(os.path.join(HERE, d)) > built for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    """Build the oracle library if it is missing or older than its sources."""
    if not force and not _stale():
        return LIB_PATH
    cc = os.environ.get("CC", "gcc")
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    cmd = [cc, *CFLAGS, "-o", tmp, *[os.path.join(HERE, s) for s in SOURCES], "-lm"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
