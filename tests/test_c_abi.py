"""The C ABI from plain C: tests/c/abi_from_c.c is compiled as C11 with gcc
against include/lora_gemm.h, linked to the built library and run; it checks
the host-side entry points without a GPU."""

import os
import shutil
import subprocess

import pytest

import lora_gemm_b200 as lg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_plain_c_caller(tmp_path):
    exe = tmp_path / "abi_from_c"
    libdir = os.path.dirname(lg.LIB_PATH)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_from_c.c"), "-L", libdir, "-l:liblora_gemm.so",
                    f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip() == "ok"
