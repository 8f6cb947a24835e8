"""CPU-only: include/fa.h compiles as C99 and a C program links to libfa.so and gets the
documented answers from every entry point's argument checks (tests/c_abi/abi_check.c)."""

from __future__ import annotations

import os
import shutil
import subprocess
import tempfile

import pytest

from exact_attention_111_b200 import build as fabuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_program_uses_the_boundary():
    lib = fabuild.build()
    libdir = os.path.dirname(lib)
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "abi_check")
        subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "c_abi", "abi_check.c"), "-o", exe, "-L", libdir, "-l:libfa.so",
                        f"-Wl,-rpath,{libdir}"], check=True)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
        assert r.returncode == 0, r.stdout + r.stderr
        assert "c abi ok" in r.stdout
