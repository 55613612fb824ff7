"""The C ABI used from C alone (tests/c_abi/fused_step.c): it must compile
and link against include/pkv.h and libpkv.so on any machine, and on a GPU
run one fused append + decode step that matches the FP64 oracle."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "paged_attention_decode_pkv_b200")
ORACLE = os.path.join(ROOT, "oracle")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _build(tmp_path):
    from oracle import build as oracle_build
    from paged_attention_decode_pkv_b200 import build as pkg_build
    pkg_build.build()
    oracle_build.build()
    exe = tmp_path / "fused_step"
    cmd = ["gcc", "-std=c11", "-O2", "-I", os.path.join(ROOT, "include"), "-I", ORACLE,
           "-I", os.path.join(CUDA, "include"), os.path.join(ROOT, "tests", "c_abi", "fused_step.c"),
           "-o", str(exe), "-L", PKG, "-lpkv", "-L", ORACLE, "-lpkv_oracle",
           "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-lm", "-lpthread",
           "-Wl,-rpath," + PKG, "-Wl,-rpath," + ORACLE, "-Wl,-rpath," + os.path.join(CUDA, "lib64")]
    subprocess.run(cmd, check=True)
    return exe


def test_c_program_compiles_and_links(tmp_path):
    assert _build(tmp_path).exists()


@pytest.mark.gpu
def test_c_program_runs_a_fused_step_against_the_oracle(tmp_path):
    exe = _build(tmp_path)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "max abs error" in r.stdout
