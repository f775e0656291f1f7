"""The C ABI used from plain C: tests/c_abi/host_calls.c is compiled with gcc
as C11 against include/bsa.h, linked to libbsa.so and run (host-only entry
points; no GPU needed)."""
import os
import shutil
import subprocess

import pytest

import block_sparse_attention_38_b200 as bsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_host_entry_points_from_c(tmp_path):
    lib = bsa.LIB_PATH
    exe = tmp_path / "host_calls"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I" + os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi", "host_calls.c"), lib, "-o", str(exe),
                    "-Wl,-rpath," + os.path.dirname(lib)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip() == "ok"
