"""The C ABI used from plain C: tests/c/abi_host.c includes include/tq.h as
C (gcc, -std=c11 -Wall -Werror), links the in-tree libtq.so and checks the
calls that need no GPU (status strings, version, size queries of invalid
requests, host-side rejections).  No GPU is used."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB_DIR = os.path.join(ROOT, "vector_quantization_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_header_compiles_as_c_and_host_calls_answer(tmp_path):
    lib = os.path.join(LIB_DIR, "libtq.so")
    if not os.path.exists(lib):
        from vector_quantization_b200 import build
        build.build()
    exe = str(tmp_path / "abi_host")
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_host.c"), "-L", LIB_DIR, "-ltq",
                    "-Wl,-rpath," + LIB_DIR, "-o", exe], check=True, capture_output=True, text=True)
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stderr
    assert run.stdout.strip() == "ok"
