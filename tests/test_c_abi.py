"""The C ABI from plain C: tests/c_abi_check.c is compiled with gcc against
include/magi_bca.h (C99, warnings as errors), linked to libmagi_bca.so and run.
It needs no GPU: it calls only the host-side entry points and the argument
checks that return before any device work."""
import os
import shutil
import subprocess

import pytest

import block_causal_attention_gqa_b200 as bca

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not found")
def test_c_program_against_the_header_and_library(tmp_path):
    lib = bca.library_path
    exe = tmp_path / "c_abi_check"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_check.c"),
           lib, "-Wl,-rpath," + os.path.dirname(lib), "-o", str(exe)]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "C ABI check: ok" in run.stdout
