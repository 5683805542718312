"""The boundary is a plain C ABI: a C99 program that includes only
include/gs.h builds against libgs_b200.so and runs its GPU-free checks
(tests/c_abi_check.c). No GPU is needed."""

import os
import shutil
import subprocess
import tempfile

import pytest

from gaussian_splatting_differentiable_ewa_b200 import api  # noqa: F401  (builds the library)
from gaussian_splatting_differentiable_ewa_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_client_builds_and_runs_against_the_library():
    lib = B.build()
    libdir = os.path.dirname(lib)
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "c_abi_check")
        cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
               os.path.join(ROOT, "tests", "c_abi_check.c"), "-o", exe, "-L", libdir,
               "-l:" + os.path.basename(lib), "-Wl,-rpath," + libdir]
        r = subprocess.run(cmd, capture_output=True, text=True)
        assert r.returncode == 0, r.stdout + r.stderr
        r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
        assert r.returncode == 0, r.stdout + r.stderr
        assert "c abi check ok" in r.stdout
