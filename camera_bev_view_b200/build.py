"""Build ``libbevsample.so`` in-tree with nvcc for sm_100a, and its
bounds-checked twin ``libbevsample_checked.so`` (-DBEV_BOUNDS_CHECK: the dense
kernels test every geometry-derived address before using it and report a
failed test as BEV_ERR_INTERNAL; for tests and debugging, not for speed).

    python -m camera_bev_view_b200.build [--verbose-ptxas] [--no-checked]
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libbevsample.so")
LIB_CHECKED = os.path.join(PKG, "libbevsample_checked.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-shared", "-Xcompiler", "-fPIC,-fvisibility=hidden",
              "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libbevsample.so")
    return cand


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def deps():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [os.path.join(INCLUDE, "bevsample.h")]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in deps())


def _build_one(lib: str, defines, ptxas_verbose: bool) -> None:
    tmpdir = tempfile.mkdtemp(prefix="bevsample-build-")
    try:
        compile_flags = [f for f in NVCC_FLAGS if f != "-shared"] + list(defines)
        extra = ["-Xptxas", "-v"] if ptxas_verbose else []

        def one(src):
            obj = os.path.join(tmpdir, os.path.basename(src) + ".o")
            r = subprocess.run([nvcc(), *extra, *ARCH, *compile_flags, "-c", src, "-o", obj],
                               capture_output=True, text=True)
            return src, obj, r

        with ThreadPoolExecutor(max_workers=max(1, min(len(sources()), os.cpu_count() or 1))) as ex:
            results = list(ex.map(one, sources()))
        for src, _, r in results:
            sys.stdout.write(r.stdout)
            sys.stderr.write(r.stderr)
            if r.returncode != 0:
                raise subprocess.CalledProcessError(r.returncode, f"nvcc -c {src}")
        tmp = lib + f".tmp{os.getpid()}"
        subprocess.run([nvcc(), *ARCH, "-shared", "-o", tmp, *[o for _, o, _ in results]], check=True)
        os.replace(tmp, lib)
    finally:
        shutil.rmtree(tmpdir, ignore_errors=True)


def build(force: bool = False, ptxas_verbose: bool = False, checked: bool = True) -> str:
    """Compile every .cu to an object in parallel (whole-program device code
    per file, no relocatable device code), then link the shared library; with
    `checked`, the bounds-checked library as well."""
    if force or not up_to_date(LIB):
        _build_one(LIB, [], ptxas_verbose)
    if checked and (force or not up_to_date(LIB_CHECKED)):
        _build_one(LIB_CHECKED, ["-DBEV_BOUNDS_CHECK"], False)
    return LIB


if __name__ == "__main__":
    build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv, checked="--no-checked" not in sys.argv)
    print(LIB)
