"""Builds libsal.so (the C-ABI CUDA library) in-tree with nvcc for sm_100a, and its
bounds-checked variant libsal_checked.so (the same sources compiled with SAL_CHECKED).

    python -m speech_audio_encoder_b200.build [--force] [--ptxas-info]

Objects go to ``_build/`` (``_build/checked/``) at the repository root; the libraries
land next to this file.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libsal.so")
LIB_CHECKED = os.path.join(PKG, "libsal_checked.so")
SOURCES = ["sal_api.cu", "frontend.cu", "rowops.cu", "gemm.cu", "attention.cu", "noalloc.cu", "ctc.cu",
           "weights_io.cu"]
HEADERS = ["sal_internal.h", "sal_ptx.cuh", "sal_check.cuh"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
                     "-Xcompiler", "-fPIC,-O2", "-I" + INCLUDE]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: libsal.so cannot be built")


def _newest_input() -> float:
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "sal.h")]
    return max(os.path.getmtime(f) for f in files)


def build(force: bool = False, ptxas_info: bool = False, quiet: bool = False, checked: bool = True) -> str:
    """Builds libsal.so (and, with `checked`, libsal_checked.so) if a source is newer."""
    lib = _build_one(LIB, BUILD, [], force, ptxas_info, quiet)
    if checked:
        _build_one(LIB_CHECKED, os.path.join(BUILD, "checked"), ["-DSAL_CHECKED"], force, False, quiet)
    return lib


def _build_one(lib: str, build_dir: str, defines: list, force: bool, ptxas_info: bool, quiet: bool) -> str:
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= _newest_input():
        return lib
    os.makedirs(build_dir, exist_ok=True)
    cc = nvcc()
    extra = ["-Xptxas", "-v"] if ptxas_info else []

    def compile_one(src: str) -> str:
        obj = os.path.join(build_dir, src.replace(".cu", ".o"))
        cmd = [cc, *NVCC_FLAGS, *defines, *extra, "-c", os.path.join(CSRC, src), "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        if ptxas_info and not quiet:
            sys.stderr.write(r.stderr)
        return obj

    with ThreadPoolExecutor(max_workers=min(len(SOURCES), os.cpu_count() or 4)) as ex:
        objs = list(ex.map(compile_one, SOURCES))
    tmp = lib + ".tmp"
    cmd = [cc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs, "-ldl", "-lpthread", "-lrt"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    if not quiet:
        print(f"built {lib}")
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    a = ap.parse_args()
    build(force=a.force or a.ptxas_info, ptxas_info=a.ptxas_info)
