"""The C ABI from plain C (no GPU): tests/c/abi_check.c is compiled as C11
against include/qstate.h with warnings as errors, linked against the
in-tree libqstate.so and run; every check it prints must hold."""
import os
import shutil
import subprocess

import pytest

from ssm_decode_step_b200 import qstate as Q

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_client(tmp_path):
    lib_dir = os.path.dirname(Q.LIB_PATH)
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    exe = str(tmp_path / "abi_check")
    cmd = ["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           "-I", cuda_inc, os.path.join(ROOT, "tests", "c", "abi_check.c"), "-L", lib_dir, "-lqstate",
           f"-Wl,-rpath,{lib_dir}", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    lines = r.stdout.splitlines()
    assert len(lines) >= 12 and all(l.startswith("ok") for l in lines), r.stdout
