"""The C ABI from plain C: tests/abi_check.c is compiled with gcc -std=c99 -pedantic
-Werror against include/kron_linear.h and include/ks_linear.h, linked with libkronlinear.so and
run on the host.
Every call in it fails a host-side check, so no GPU is needed."""
import os
import shutil
import subprocess

import pytest

from kronecker_factored_structured_b200 import native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_checks_every_entry_point(tmp_path):
    lib = native.LIB_PATH
    assert os.path.exists(lib), "build the library first"
    exe = tmp_path / "abi_check"
    subprocess.check_call(
        ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
         "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "abi_check.c"),
         "-L", os.path.dirname(lib), "-lkronlinear",
         f"-Wl,-rpath,{os.path.dirname(lib)}", "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "all checks passed" in out.stdout
