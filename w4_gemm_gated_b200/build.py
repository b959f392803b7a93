"""Build the CUDA library ``libspear.so`` in-tree for sm_100a.

Usage: ``python -m w4_gemm_gated_b200.build [--force] [--verbose] [--checked]``.
Objects go to ``_build/`` at the repository root; the shared library is
written next to this file so that it travels with the source tree.
``--checked`` builds the device-check variant ``libspear_checked.so`` (the
same sources with -DSPEAR_DEVICE_CHECKS; objects in ``_build/checked``).
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libspear.so")
LIB_CHECKED = os.path.join(PKG, "libspear_checked.so")
SOURCES = ["api.cu", "pack.cu", "decode.cu", "decode2.cu", "decode3.cu", "ec.cu", "tc_gemm.cu", "noalloc.cu"]
HEADERS = ["common.cuh", "kernels.h", "tma.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC",
    "-Xptxas", "-v",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps_mtime() -> float:
    paths = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", "spear.h")]
    return max(os.path.getmtime(p) for p in paths)


def _compile(src: str, verbose: bool, checked: bool = False) -> tuple[str, str]:
    odir = os.path.join(BUILD, "checked") if checked else BUILD
    obj = os.path.join(odir, os.path.splitext(src)[0] + ".o")
    extra = ["-DSPEAR_DEVICE_CHECKS"] if checked else []
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", os.path.join(ROOT, "include"), "-c", os.path.join(CSRC, src), "-o",
           obj]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{res.stdout}\n{res.stderr}")
    log = res.stderr if verbose else ""
    return obj, log


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    lib = LIB_CHECKED if checked else LIB
    os.makedirs(os.path.join(BUILD, "checked") if checked else BUILD, exist_ok=True)
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    if not force and os.path.exists(lib):
        newest = max([os.path.getmtime(s) for s in srcs] + [_deps_mtime(), os.path.getmtime(__file__)])
        if os.path.getmtime(lib) >= newest:
            return lib
    with cf.ThreadPoolExecutor(max_workers=min(len(SOURCES), os.cpu_count() or 4)) as ex:
        results = list(ex.map(lambda s: _compile(s, verbose, checked), SOURCES))
    objs = [o for o, _ in results]
    if verbose:
        for _, log in results:
            sys.stderr.write(log)
    tmp = lib + ".tmp"
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-Xcompiler", "-fPIC", *objs,
           "-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"link failed:\n{res.stdout}\n{res.stderr}")
    os.replace(tmp, lib)
    return lib


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--checked", action="store_true", help="build the device-check variant")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose, checked=args.checked))


if __name__ == "__main__":
    main()
