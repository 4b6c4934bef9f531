"""The C ABI from a plain C program (no Python or torch in the loop), on a B200."""

import os
import subprocess

import pytest

import oracle

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = "/usr/local/cuda"


def test_plain_c_program_drives_the_library(tmp_path):
    oracle.build()
    exe = tmp_path / "c_abi_check"
    lib_dir = os.path.join(ROOT, "sequence_all_re_b200")
    oracle_dir = os.path.dirname(oracle.__file__)
    subprocess.run(
        ["gcc", "-O1", "-std=c11", "-Wall", "-o", str(exe),
         os.path.join(ROOT, "tests", "c_abi_check.c"),
         "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
         "-L", lib_dir, "-lulysses_a2a", "-L", oracle_dir, "-lulysses_oracle",
         "-L", os.path.join(CUDA, "lib64"), "-lcudart",
         f"-Wl,-rpath,{lib_dir}:{oracle_dir}:{os.path.join(CUDA, 'lib64')}"],
        check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "all checks passed" in r.stdout
