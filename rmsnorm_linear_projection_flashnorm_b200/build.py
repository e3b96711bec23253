"""Build the C-ABI shared library (libflashnorm.so) in-tree with nvcc for sm_100a.

    python -m rmsnorm_linear_projection_flashnorm_b200.build [--verbose-ptxas]

Each CUDA source is compiled for sm_100a only (tcgen05 and TMA need the
architecture-specific target) and linked against the static CUDA runtime, so
the library loads without a GPU and the Python binding can check its exports.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys
from typing import List

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libflashnorm.so"
LIB_PATH = os.path.join(PKG_DIR, LIB_NAME)
SOURCES = ["api.cu", "fold.cu", "decode.cu", "decode_cl.cu", "decode_fp8.cu", "decode_mx.cu", "tc.cu", "tc2.cu", "tc8.cu", "noalloc.cu",
           "post_scale.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libflashnorm.so")


def _stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose_ptxas: bool = False, jobs: int = 4) -> str:
    if not force and not verbose_ptxas and not _stale():
        return LIB_PATH
    obj_dir = os.path.join(ROOT, "_build")
    os.makedirs(obj_dir, exist_ok=True)
    common = [nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC,-O3",
              "-I", INCLUDE, "-I", CSRC]
    if verbose_ptxas:
        common += ["-Xptxas", "-v"]
    procs: List[subprocess.Popen] = []
    objs = []
    for src in SOURCES:
        obj = os.path.join(obj_dir, src.replace(".cu", ".o"))
        objs.append(obj)
        cmd = common + ["-c", os.path.join(CSRC, src), "-o", obj]
        procs.append(subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True))
        if len(procs) >= jobs:
            _finish(procs.pop(0))
    for p in procs:
        _finish(p)
    tmp = LIB_PATH + ".tmp"
    subprocess.run([nvcc(), *ARCH, "-shared", "-o", tmp, *objs], check=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


def _finish(p: subprocess.Popen) -> None:
    out, _ = p.communicate()
    if out:
        sys.stdout.write(out)
    if p.returncode != 0:
        raise RuntimeError(f"nvcc failed ({' '.join(p.args[-3:])})")


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--force", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas))
