"""Compile the FP64 CPU oracle (test infrastructure) into oracle/libpkv_oracle.so.

Plain gcc, -O2, no fast-math: the oracle's arithmetic is the IEEE double
arithmetic of the C source as written.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "pkv_oracle.c")
HDR = os.path.join(HERE, "pkv_oracle.h")
LIB = os.path.join(HERE, "libpkv_oracle.so")


def build(force: bool = False) -> str:
    """Build the oracle library if it is missing or older than its sources."""
    if not force and os.path.exists(LIB):
        newest = max(os.path.getmtime(SRC), os.path.getmtime(HDR))
        if os.path.getmtime(LIB) >= newest:
            return LIB
    cc = os.environ.get("CC", "gcc")
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = [cc, "-std=c11", "-O2", "-fno-fast-math", "-fPIC", "-shared", "-pthread",
           "-Wall", "-Wextra", SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
