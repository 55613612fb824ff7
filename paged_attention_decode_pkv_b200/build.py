"""Build libpkv.so (the C-ABI CUDA library) in-tree for sm_100a.

    python -m paged_attention_decode_pkv_b200.build [--force] [--verbose]

nvcc compiles every csrc/*.cu for sm_100a only (-gencode
arch=compute_100a,code=sm_100a) with line info, and links them into
paged_attention_decode_pkv_b200/libpkv.so against the shared CUDA runtime.
The driver API entry needed for TMA descriptors is fetched at run time, so
there is no link-time dependency on libcuda.
"""
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libpkv.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(INCLUDE, "pkv.h")]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    return os.path.getmtime(LIB) >= max(os.path.getmtime(p) for p in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = [nvcc, "-std=c++17", "-O3", "-lineinfo", *ARCH, "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
           "-shared", "-cudart", "shared", "-I", INCLUDE, "-I", CSRC,
           "--expt-relaxed-constexpr", *sources(), "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
