"""The C ABI from plain C: tests/abi_check.c is compiled as C99 against
include/zcmoe.h, linked against libzcmoe.so, and run.  It checks that the header
is valid C, that the library links and loads from a C program, and that the
entry points refuse bad arguments on the host.  CPU only: nothing reaches a device."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "mixture_experts_layer_shifted_b200")
CUDA_INC = "/usr/local/cuda/include"


def test_header_compiles_as_c99_and_the_library_links_from_c(tmp_path):
    if shutil.which("gcc") is None or not os.path.isdir(CUDA_INC):
        pytest.skip("gcc or the CUDA headers are not available")
    from mixture_experts_layer_shifted_b200 import build
    build.build()
    exe = str(tmp_path / "abi_check")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), "-I", CUDA_INC,
           os.path.join(ROOT, "tests", "abi_check.c"), "-o", exe, "-L", PKG, "-lzcmoe", f"-Wl,-rpath,{PKG}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "all host-side checks hold" in r.stdout
