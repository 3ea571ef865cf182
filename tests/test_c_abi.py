"""The C ABI from a plain C program (CPU): tests/c/abi_client.c is compiled with
the system C compiler against include/kvsculpt.h and the in-tree library, then
run; it exercises the host-only entry points and the argument checks."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "kv_cache_compression_kvsculpt_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_client(tmp_path):
    lib = os.path.join(PKG, "libkvsculpt.so")
    assert os.path.exists(lib), "build the library first"
    exe = tmp_path / "abi_client"
    r = subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-O1",
                        "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "c", "abi_client.c"),
                        "-L", PKG, "-lkvsculpt", "-Wl,-rpath," + PKG, "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "c abi ok" in r.stdout
