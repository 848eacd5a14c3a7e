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


def _cuda_root():
    for cand in (os.environ.get("CUDA_HOME"), "/usr/local/cuda"):
        if cand and os.path.exists(os.path.join(cand, "include", "cuda_runtime_api.h")):
            return cand
    return None


@pytest.mark.gpu
@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_c_program_runs_the_gpu_path():
    """tests/c/gpu_closed_form.c: a C99 program allocates device buffers with the
    CUDA runtime, calls fckl_fwd_bwd and fckl_check, and checks the K = 1
    cross-entropy case against its own double-precision reference and the
    teacher = student case against zero."""
    cuda = _cuda_root()
    assert cuda is not None, "CUDA runtime headers not found"
    build()
    lib = fk.lib_path()
    with tempfile.TemporaryDirectory() as tmp:
        os.symlink(lib, os.path.join(tmp, "libfckl.so"))
        exe = os.path.join(tmp, "gpu_closed_form")
        cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
               "-I", os.path.join(ROOT, "include"), "-isystem", os.path.join(cuda, "include"),
               os.path.join(ROOT, "tests", "c", "gpu_closed_form.c"),
               "-L", tmp, "-lfckl", "-L", os.path.join(cuda, "lib64"), "-lcudart",
               "-Wl,-rpath," + tmp, "-Wl,-rpath," + os.path.join(cuda, "lib64"), "-lm", "-o", exe]
        r = subprocess.run(cmd, capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
        r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
        print(r.stdout)
        assert r.returncode == 0, r.stdout + r.stderr
        assert "0 failure(s)" in r.stdout
