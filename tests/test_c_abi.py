"""The library is callable from plain C: tests/native/abi_c.c includes
include/pa.h, is compiled as strict C11 with warnings as errors, links
libpa.so and runs block-manager calls on a host-only pool (no GPU)."""
import os
import shutil
import subprocess

import pytest

import pagedattention_decode_03_b200 as pa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from pagedattention_decode_03_b200 import build
    build.build()


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c11_caller_links_and_runs():
    out = os.path.join(ROOT, "_build")
    os.makedirs(out, exist_ok=True)
    exe = os.path.join(out, "abi_c")
    libdir = os.path.dirname(pa.LIB_PATH)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "native", "abi_c.c"),
                    "-L", libdir, "-l:" + os.path.basename(pa.LIB_PATH),
                    "-Wl,-rpath," + libdir, "-o", exe],
                   check=True, capture_output=True, text=True, timeout=300)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr[-3000:]
    assert r.stdout.strip() == "ok"
