"""Build libpa370.so in-tree: CUDA kernels for sm_100a plus the host C++ code.

    python -m paged_kv_cache_370_b200.build [--force]

nvcc compiles every ``csrc/*.cu`` for ``sm_100a`` (and nothing else); g++
compiles ``csrc/*.cpp``; the objects are linked into one shared library next
to this file, with the CUDA runtime linked statically so the library depends
only on the driver at run time.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(ROOT, "_build", "pa370")
LIB_NAME = "libpa370.so"
LIB_PATH = os.path.join(PKG, LIB_NAME)

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
              "--expt-relaxed-constexpr"]
CXX_FLAGS = ["-O2", "-std=c++17", "-fPIC", "-Wall", "-Wextra"]


def _nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libpa370.so")
    return cand


def _sources():
    cu = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    cpp = sorted(glob.glob(os.path.join(CSRC, "*.cpp")))
    hdr = sorted(glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h")))
    return cu, cpp, hdr


def needs_build() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    cu, cpp, hdr = _sources()
    newest = max(os.path.getmtime(p) for p in cu + cpp + hdr + [__file__])
    return os.path.getmtime(LIB_PATH) < newest


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not needs_build():
        return LIB_PATH
    os.makedirs(BUILD_DIR, exist_ok=True)
    nvcc = _nvcc()
    cu, cpp, _ = _sources()
    objs = []
    for src in cu:
        obj = os.path.join(BUILD_DIR, os.path.basename(src) + ".o")
        extra = os.environ.get("PA370_NVCC_FLAGS", "").split()  # e.g. -DPA_STREAM_STAGES_D128=4
        cmd = [nvcc, *ARCH_FLAGS, *NVCC_FLAGS, *extra, f"-I{INCLUDE}", f"-I{CSRC}", "-c", src, "-o",
               obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        subprocess.run(cmd, check=True)
        objs.append(obj)
    for src in cpp:
        obj = os.path.join(BUILD_DIR, os.path.basename(src) + ".o")
        subprocess.run(["g++", *CXX_FLAGS, f"-I{INCLUDE}", "-c", src, "-o", obj], check=True)
        objs.append(obj)
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    subprocess.run([nvcc, *ARCH_FLAGS, "-shared", "-cudart", "static", "-o", tmp, *objs],
                   check=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print ptxas register/spill report")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
