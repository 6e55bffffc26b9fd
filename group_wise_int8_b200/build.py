"""Build the CUDA library in-tree: group_wise_int8_b200/libwino_b200.so (sm_100a),
and its debug build libwino_b200_debug.so.

    python -m group_wise_int8_b200.build [--force] [--verbose]

Each translation unit is compiled by nvcc for sm_100a only (no PTX for other
targets), without fast-math (the quantised pipeline relies on IEEE fp32
division, fma and round-to-nearest-even), then linked into one shared
library with the static CUDA runtime.  The debug build is the same source
compiled with -DWINO_DEBUG: every kernel checks the element index of each
global access against its buffer, skips an access that fails and records it in
the device error word (no trap).
"""
import concurrent.futures
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libwino_b200.so")
LIB_DEBUG = os.path.join(HERE, "libwino_b200_debug.so")
SOURCES = ["plan.cpp", "api.cu", "weight_transform.cu", "input_transform.cu", "hadamard_tc.cu",
           "hadamard_simt.cu", "output_transform.cu", "input_quant.cu", "noalloc.cu", "fused_small.cu"]
HEADERS = ["plan.h", "common.cuh", "sm100.cuh", "kernels.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "wino.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def _compile(src: str, verbose: bool, debug: bool = False) -> str:
    outdir = os.path.join(BUILD, "debug") if debug else BUILD
    obj = os.path.join(outdir, os.path.basename(src) + ".o")
    cmd = [nvcc(), "-c", "-std=c++17", "-O3", "-lineinfo", *ARCH, "-Xcompiler", "-fPIC,-O2",
           "-I", os.path.join(ROOT, "include"), "-o", obj, os.path.join(CSRC, src)]
    if debug:
        cmd.insert(2, "-DWINO_DEBUG")
    if verbose and src.endswith(".cu"):
        cmd[1:1] = ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed for %s:\n%s\n%s" % (src, r.stdout, r.stderr))
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    return obj


def _build_one(lib: str, debug: bool, verbose: bool, ex) -> None:
    os.makedirs(os.path.join(BUILD, "debug") if debug else BUILD, exist_ok=True)
    objs = list(ex.map(lambda s: _compile(s, verbose, debug), SOURCES))
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [nvcc(), "-shared", *ARCH, "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("link failed:\n%s\n%s" % (r.stdout, r.stderr))
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> str:
    """Builds whichever of the release and (with debug) the debug library is out of date; returns
    the release path."""
    libs = ((LIB, False), (LIB_DEBUG, True)) if debug else ((LIB, False),)
    todo = [(lib, dbg) for lib, dbg in libs if force or not up_to_date(lib)]
    if todo:
        with concurrent.futures.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            for lib, dbg in todo:
                _build_one(lib, dbg, verbose, ex)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
