"""Builds the in-tree CUDA library `libss1.so` for sm_100a with nvcc.

    python -m structured_compressed_linear_b200.build [--force] [-v] [--checked]

Every .cu under csrc/ is compiled separately (in parallel) for sm_100a and linked into one
shared library next to this file. The CUDA runtime is linked statically; the driver API
(tensor-map encoding) is reached through cudaGetDriverEntryPoint, so the library has no
link-time dependency on libcuda and can be loaded on a machine without a GPU.

`--checked` builds the debug library `libss1_checked.so` from the same sources with
SS1_CHECKED=1: every global access a kernel addresses by its own index arithmetic is tested
against its buffer's extent first (see ss1_bounds_check in include/ss1.h). The tests share one
device word, so that build uses relocatable device code.
"""

from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libss1.so")
LIB_CHECKED = os.path.join(PKG, "libss1_checked.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden",
          "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h")) + [__file__]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    lib = LIB_CHECKED if checked else LIB
    if not force and up_to_date(lib):
        return lib
    build_dir = os.path.join(BUILD_DIR, "checked") if checked else BUILD_DIR
    extra = ["-DSS1_CHECKED=1", "-rdc=true"] if checked else []
    os.makedirs(build_dir, exist_ok=True)
    cc = nvcc()

    def compile_one(src):
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        cmd = [cc, *ARCH, *COMMON, *extra, "-c", src, "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        if verbose and r.stderr:
            sys.stderr.write(r.stderr)
        return obj

    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, sources()))
    tmp = lib + ".tmp"
    cmd = [cc, *ARCH, *extra[1:], "-shared", "-Xcompiler", "-fPIC", "-cudart", "static", "-o", tmp, *objs, "-ldl",
           "-lpthread", "-lrt"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true", help="print ptxas register/smem usage")
    ap.add_argument("--checked", action="store_true", help="build the bounds-checked debug library")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, checked=a.checked))


if __name__ == "__main__":
    main()
