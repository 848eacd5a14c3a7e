"""The header is plain C99 and a C program links and calls the library:
compile tests/c/abi_check.c with gcc against include/fckl.h and libfckl.so and
run it (host-only entry points and argument checks; no GPU needed)."""
import os
import shutil
import subprocess
import tempfile

import pytest

import chunked_kl_loss_tcgen05_b200 as fk
from chunked_kl_loss_tcgen05_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_c_program_links_and_runs():
    build()
    lib = fk.lib_path()
    libdir = os.path.dirname(lib)
    with tempfile.TemporaryDirectory() as tmp:
        # link against the library under its soname-less file name
        os.symlink(lib, os.path.join(tmp, "libfckl.so"))
        exe = os.path.join(tmp, "abi_check")
        cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
               "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_check.c"),
               "-L", tmp, "-lfckl", "-Wl,-rpath," + tmp, "-lm", "-o", exe]
        r = subprocess.run(cmd, capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
        r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
        assert r.returncode == 0, r.stdout + r.stderr
        assert "0 failure(s)" in r.stdout
