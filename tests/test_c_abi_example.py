"""The C ABI on its own: a plain C host (tests/c_abi_example.c) that allocates with the CUDA
runtime and calls libslm.so, with no Python or torch on its path.  It compiles here; on a
GPU it runs and checks the closed forms of W = 0 (CE = log V, dH = 0, dW's formula)."""

import os
import shutil
import subprocess

import pytest

from lm_head_loss_streaming_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _compile(tmp_path):
    if not os.path.exists(_lib.LIB_PATH):
        from lm_head_loss_streaming_b200.build import build
        build()
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    exe = str(tmp_path / "c_abi_example")
    libdir = os.path.dirname(_lib.LIB_PATH)
    cmd = [cc, "-O2", "-std=c99", os.path.join(ROOT, "tests", "c_abi_example.c"),
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           "-L", libdir, "-lslm", f"-Wl,-rpath,{libdir}",
           "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}",
           "-lm", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    return exe


def test_c_host_compiles_and_links(tmp_path):
    assert os.path.exists(_compile(tmp_path))


@pytest.mark.gpu
def test_c_host_runs(tmp_path):
    exe = _compile(tmp_path)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip().endswith("ok")
