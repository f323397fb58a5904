"""The C ABI from C: include/moe_b200.h compiles as strict C99 and a C program linked
against libmoe_b200.so runs the host-only entry points (tests/c/abi_host.c). No GPU."""
import os
import shutil
import subprocess

import pytest

import mixture_experts_expert_topk_b200  # noqa: F401  (builds nothing; the .so must exist)
from mixture_experts_expert_topk_b200 import _capi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_program_uses_the_abi(tmp_path):
    lib = _capi.LIB_PATH
    assert os.path.exists(lib), "build the library first"
    exe = tmp_path / "abi_host"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_host.c"), "-o", str(exe), lib,
           "-Wl,-rpath," + os.path.dirname(lib)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr
