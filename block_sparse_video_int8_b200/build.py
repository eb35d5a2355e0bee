"""Build the in-tree CUDA library ``libbsva.so`` for sm_100a with nvcc.

Each ``csrc/*.cu`` compiles to an object under ``_build/`` (in parallel), then
nvcc links the shared library next to this file. The CUDA runtime is linked
statically and the driver's tensor-map encoder is resolved at run time, so the
library loads on a machine without a GPU (its entry points then report that no
device is present).
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libbsva.so")
# The same sources with BSVA_DEVICE_CHECKS: kernels validate the indices they take from their inputs
# (kept counts and lists, table rows) and record a failure in the status word instead of using them.
LIB_CHECKED = os.path.join(HERE, "libbsva_checked.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _compile(src: str, extra, objdir: str = BUILD) -> str:
    obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
    cmd = [_nvcc(), *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    if r.stderr.strip() and "-Xptxas" in " ".join(extra):
        sys.stderr.write(r.stderr)
    return obj


def build(force: bool = False, extra=(), checked: bool = False) -> str:
    """Compile every kernel source and link ``libbsva.so`` (or, with ``checked``, the
    ``BSVA_DEVICE_CHECKS`` build ``libbsva_checked.so``); returns its path."""
    lib = LIB_CHECKED if checked else LIB
    objdir = os.path.join(BUILD, "checked") if checked else BUILD
    extra = list(extra) + (["-DBSVA_DEVICE_CHECKS"] if checked else [])
    srcs = sources()
    deps = srcs + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    deps.append(os.path.join(ROOT, "include", "bsva.h"))
    if (not force and (checked or not extra) and os.path.exists(lib)
            and os.path.getmtime(lib) >= max(os.path.getmtime(p) for p in deps)):
        return lib
    os.makedirs(objdir, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra, objdir), srcs))
    tmp = lib + ".tmp"
    cmd = [_nvcc(), *ARCH, "-shared", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    args = sys.argv[1:]
    checked = "--checked" in args
    extra = [a for a in args if a != "--checked"]
    print(build(force=True, extra=extra, checked=checked))
