"""Builds the C-ABI shared library libqlora_b200.so in-tree with nvcc.

Every translation unit under csrc/ is compiled for sm_100a only
(-gencode arch=compute_100a,code=sm_100a) and linked with the static CUDA
runtime; the library loads without PyTorch.

With --debug the same sources are compiled with QLORA_DEBUG into
libqlora_b200_debug.so: the bounds-checked build, whose kernels record a
failed index check instead of faulting (qlora_debug_bounds in qlora.h).

Usage: python bit_nf4_quantized_16_b200/build.py [--force] [-v] [--debug]
(run by path: importing the package itself needs the built library)
"""

import argparse
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libqlora_b200.so")
LIB_DEBUG = os.path.join(HERE, "libqlora_b200_debug.so")
OBJ_DIR = os.path.join(ROOT, "_build")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [
        os.path.join(ROOT, "include", "qlora.h"), __file__]


def up_to_date(debug: bool = False) -> bool:
    lib = LIB_DEBUG if debug else LIB
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and up_to_date(debug):
        return lib
    obj_dir = os.path.join(OBJ_DIR, "debug") if debug else OBJ_DIR
    os.makedirs(obj_dir, exist_ok=True)
    objs = []
    for src in _sources():
        obj = os.path.join(obj_dir, os.path.basename(src) + ".o")
        cmd = [NVCC] + ARCH + FLAGS + (["-DQLORA_DEBUG"] if debug else []) + ["-c", src, "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)
        objs.append(obj)
    cmd = [NVCC] + ARCH + ["-shared", "-o", lib] + objs + ["-cudart", "static"]
    subprocess.check_call(cmd)
    return lib


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--debug", action="store_true", help="the bounds-checked build (QLORA_DEBUG)")
    a = ap.parse_args(argv)
    print(build(force=a.force, verbose=a.verbose, debug=a.debug))


if __name__ == "__main__":
    sys.exit(main())
