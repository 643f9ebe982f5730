"""The C ABI from a C compiler: tests/c/abi_client.c is compiled as strict C99 against
include/fp8bs.h, linked against the in-tree libfp8bs.so and run (host-side calls only, no
GPU)."""

import os
import shutil
import subprocess

import pytest

import fp8_block_scaled_a8w8_b200 as fb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_client_compiles_links_and_runs(tmp_path):
    lib = fb.lib()  # builds the library if needed
    libdir = os.path.dirname(fb.LIB_PATH)
    exe = str(tmp_path / "abi_client")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_client.c"), "-L", libdir, "-lfp8bs", f"-Wl,-rpath,{libdir}", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert lib is not None
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.count("ok:") == 11
