"""Build step of the CUDA library: compiles csrc/*.cu for sm_100a into
libnvfp4rac.so next to this file (in-tree, so it travels with the sources)."""
from __future__ import annotations

import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SOURCES = ["api.cu", "quant.cu", "select.cu", "gemm.cu", "noalloc.cu"]
LIB = os.path.join(PKG, "libnvfp4rac.so")
# the index-checked build (NVFP4_CHECKS): same sources, every kernel store and
# gathered load tests its index
LIB_CHECKED = os.path.join(PKG, "libnvfp4rac_checked.so")
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-gencode", "arch=compute_100a,code=sm_100a",
         "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-warn-spills"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(PKG, "csrc", f) for f in os.listdir(os.path.join(PKG, "csrc"))]
    deps.append(os.path.join(ROOT, "include", "nvfp4rac.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    lib = LIB_CHECKED if checked else LIB
    if not force and not needs_build(lib):
        return lib
    cmd = [nvcc(), *FLAGS, *(["-DNVFP4_CHECKS"] if checked else []), "-I", os.path.join(ROOT, "include"),
           *[os.path.join(PKG, "csrc", s) for s in SOURCES], "-o", lib + ".tmp"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose and (res.stdout or res.stderr):
        print(res.stdout + res.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose=True))
    print(build(force=True, verbose=True, checked=True))
