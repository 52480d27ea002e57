"""Build ``libslm.so`` in-tree with nvcc for sm_100a (B200).

    python -m lm_head_loss_streaming_b200.build [--verbose] [--force]
    python -m lm_head_loss_streaming_b200.build --out _build/g1/libslm.so -D SLM_GROUP_B=1

The second form builds a variant library elsewhere with extra preprocessor definitions:
the GEMM schedule's knobs in ``csrc/slm_schedule.h`` (``SLM_GROUP_PAIRS``, ``SLM_MAX_RUNS``,
``SLM_GROUP_B``, ``SLM_SYNC_*``) are overridable that way.  ``SLM_LIBRARY=<path>`` makes
the Python binding load such a library instead of the in-tree one.

The library is plain CUDA C++ behind a C ABI: no PyTorch headers, no JIT cache.  The CUDA
runtime is linked statically; the driver's tensor-map encoder is fetched at run time, so
no driver library is needed at link time and the build runs on a machine without a GPU.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libslm.so")
BUILD_DIR = os.path.join(ROOT, "_build")

SOURCES = ["slm_api.cu", "slm_kernels.cu", "slm_noalloc.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "--use_fast_math", "-Xcompiler", "-fPIC",
         "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC]


def nvcc():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _newer(target, deps):
    if not os.path.exists(target):
        return False
    t = os.path.getmtime(target)
    return all(os.path.getmtime(d) <= t for d in deps)


def build(verbose=False, force=False, ptxas_verbose=False, out=None, defines=()):
    """Build the library (in-tree by default; at `out`, with `defines` as extra -D
    definitions, for a variant).  Returns its path."""
    lib = os.path.abspath(out) if out else LIB
    defines = list(defines)
    for dfn in defines:
        if not dfn.replace("=", "").replace("_", "").replace("-", "").isalnum():
            raise ValueError(f"bad definition {dfn!r}: expected NAME or NAME=VALUE")
    obj_dir = BUILD_DIR if not out else os.path.join(os.path.dirname(lib), "_obj")
    os.makedirs(obj_dir, exist_ok=True)
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    headers.append(os.path.join(INCLUDE, "slm.h"))
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    if not force and not out and _newer(lib, srcs + headers + [os.path.abspath(__file__)]):
        return lib
    exe = nvcc()
    extra = ["-Xptxas", "-v"] if ptxas_verbose else []
    extra += ["-D" + dfn for dfn in defines]

    def compile_one(src):
        obj = os.path.join(obj_dir, os.path.basename(src) + ".o")
        cmd = [exe, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        if verbose or ptxas_verbose:
            sys.stdout.write(r.stdout + r.stderr)
        return obj

    with ThreadPoolExecutor(len(srcs)) as ex:
        objs = list(ex.map(compile_one, srcs))
    tmp = lib + ".tmp"
    cmd = [exe, *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    import argparse

    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    ap.add_argument("--out", default=None, help="build a variant library at this path")
    ap.add_argument("-D", dest="defines", action="append", default=[],
                    help="extra preprocessor definition (NAME or NAME=VALUE) for --out")
    a = ap.parse_args()
    if a.defines and not a.out:
        ap.error("-D needs --out: the in-tree library keeps the default schedule")
    print(build(verbose=a.verbose, force=a.force, ptxas_verbose=a.ptxas_verbose, out=a.out,
                defines=a.defines))
