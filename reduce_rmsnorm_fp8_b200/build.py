"""Build ``librrf.so`` (the C-ABI CUDA library) in-tree for sm_100a.

    python -m reduce_rmsnorm_fp8_b200.build [--force] [--verbose] [--debug]

Every translation unit under ``csrc/`` is compiled by nvcc for
``-gencode arch=compute_100a,code=sm_100a`` (the fused kernel once per input
bound, in parallel) and linked into ``reduce_rmsnorm_fp8_b200/librrf.so``
with the CUDA runtime linked statically.  No GPU is needed to build.

``--debug`` builds the bounds-checking variant, ``librrf_debug.so`` (the same
sources with RRF_DEBUG defined: every kernel checks the indices of its global
and shared accesses, skips an access that would fall outside its buffer and
reports it as RRF_DEVICE_ERROR_BOUNDS in the device error word).  The binding
loads it instead of ``librrf.so`` when RRF_DEBUG_LIBRARY=1 is set.
"""
from __future__ import annotations

import argparse
import concurrent.futures
import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "librrf.so")
DEBUG_BUILD_DIR = os.path.join(PKG, "_build_debug")
DEBUG_LIB = os.path.join(PKG, "librrf_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                     "-Xcompiler", "-Wall", "-I", INCLUDE, "-I", CSRC]

# (source, extra flags, object name)
UNITS = [("rrf_api.cu", [], "rrf_api.o"), ("rrf_sum.cu", [], "rrf_sum.o"),
         ("rrf_post.cu", [], "rrf_post.o"), ("rrf_allreduce.cu", [], "rrf_allreduce.o"),
         ("rrf_gemm.cu", [], "rrf_gemm.o"), ("rrf_noalloc.cu", [], "rrf_noalloc.o")] + [
    ("rrf_fused.cu", [f"-DRRF_RB={rb}"], f"rrf_fused_rb{rb}.o") for rb in (2, 4, 8, 16)]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build librrf.so")
    return path


def _inputs():
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC))] + \
        [os.path.join(INCLUDE, f) for f in sorted(os.listdir(INCLUDE))]


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _inputs() + [__file__])


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile and link librrf.so (debug: librrf_debug.so, the bounds-checking
    build) unless it is newer than every source."""
    lib_path, build_dir = (DEBUG_LIB, DEBUG_BUILD_DIR) if debug else (LIB, BUILD_DIR)
    if not force and not stale(lib_path):
        return lib_path
    os.makedirs(build_dir, exist_ok=True)
    cc = nvcc()
    flags = NVCC_FLAGS + (["-DRRF_DEBUG"] if debug else [])

    def compile_unit(unit):
        src, extra, obj = unit
        cmd = [cc, *flags, *extra, "-c", os.path.join(CSRC, src),
               "-o", os.path.join(build_dir, obj)]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        return r.stderr

    with concurrent.futures.ThreadPoolExecutor(max_workers=len(UNITS)) as ex:
        logs = list(ex.map(compile_unit, UNITS))
    if verbose:
        for log in logs:
            print(log)
    tmp = lib_path + f".tmp{os.getpid()}"
    cmd = [cc, *ARCH, "-shared", "-o", tmp] + \
        [os.path.join(build_dir, u[2]) for u in UNITS]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib_path)
    return lib_path


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true", help="print ptxas register use")
    ap.add_argument("--debug", action="store_true",
                    help="the bounds-checking build (librrf_debug.so)")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose, debug=args.debug))


if __name__ == "__main__":
    main()
