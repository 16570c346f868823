"""The boundary as a C program sees it: ``include/bsgemm.h`` compiles as C99
(and as C++) with warnings as errors, and ``tests/abi_c_client.c`` links
``libbsgemm.so`` and runs its host-only checks. No GPU is needed."""
import os
import shutil
import subprocess
import tempfile

import pytest

import fp8_block_scaled_bsgemm_b200 as bsg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
LIBDIR = os.path.dirname(bsg.LIB_PATH)

pytestmark = pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")


def _scratch():
    base = os.path.join(ROOT, "_build")
    os.makedirs(base, exist_ok=True)
    return tempfile.mkdtemp(prefix="abi_c_", dir=base)


def test_c_client_links_and_passes_its_host_checks():
    bsg.lib()   # the library is built
    d = _scratch()
    try:
        exe = os.path.join(d, "abi_c_client")
        subprocess.run(["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror", "-I", INCLUDE,
                        os.path.join(ROOT, "tests", "abi_c_client.c"), "-o", exe, "-L", LIBDIR,
                        "-lbsgemm", "-Wl,-rpath," + LIBDIR], check=True)
        r = subprocess.run([exe], capture_output=True, text=True)
        assert r.returncode == 0, r.stdout + r.stderr
        assert "all checks passed" in r.stdout
    finally:
        shutil.rmtree(d, ignore_errors=True)


def test_header_compiles_as_cxx():
    if shutil.which("g++") is None:
        pytest.skip("needs g++")
    d = _scratch()
    try:
        src = os.path.join(d, "h.cpp")
        with open(src, "w") as f:
            f.write('#include "bsgemm.h"\nint main() { return bsgemm_version() > 0 ? 0 : 1; }\n')
        subprocess.run(["g++", "-std=c++11", "-Wall", "-Wextra", "-Werror", "-I", INCLUDE, "-c", src,
                        "-o", os.path.join(d, "h.o")], check=True)
    finally:
        shutil.rmtree(d, ignore_errors=True)
