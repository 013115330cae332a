"""Build the CUDA library libaqlm_b200.so in-tree with nvcc (sm_100a only).

The library exposes the C ABI declared in include/aqlm.h; it links the CUDA
runtime statically and fetches the driver's tensor-map encoder at run time,
so it needs no libcuda at link time.  The debug variant
libaqlm_b200_debug_bounds.so is the same sources built with
-DAQLM_DEBUG_BOUNDS (device index checks that record, and skip, an
out-of-range access).  Usage: python -m additive_codebook_b200.build [--debug-bounds]
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libaqlm_b200.so")
DEBUG_LIB = os.path.join(PKG, "libaqlm_b200_debug_bounds.so")
SOURCES = ["abi.cu", "dequant.cu", "encode.cu", "gemv.cu", "gemm_tcgen05.cu", "gemv_noalloc.cu", "gemv_lut.cu",
           "gemv_rows.cu", "gemv_tc.cu", "probe.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "-cudart", "static"]


def _stale(lib):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "aqlm.h"), __file__]
    return any(os.path.getmtime(p) > t for p in deps)


def _compile(src, obj, extra, verbose):
    cmd = [NVCC, *FLAGS, *extra, "-c", "-I", INCLUDE, "-I", CSRC, "-o", obj, os.path.join(CSRC, src)]
    if verbose:
        print(" ".join(cmd), flush=True)
    return subprocess.run(cmd, capture_output=True, text=True)


def build(force=False, verbose=False, ptxas_info=False, debug_bounds=False, out_lib=None, objdir=None):
    """Compile every source in parallel, then link the shared library (the
    debug-bounds variant with debug_bounds=True; out_lib / objdir override
    where it goes)."""
    lib = out_lib or (DEBUG_LIB if debug_bounds else LIB)
    if not force and not _stale(lib):
        return lib
    objdir = objdir or os.path.join(PKG, "_build_debug_bounds" if debug_bounds else "_build")
    os.makedirs(objdir, exist_ok=True)
    extra = ["-Xptxas", "-v"] if ptxas_info else []
    if debug_bounds:
        extra += ["-DAQLM_DEBUG_BOUNDS"]
    objs = [os.path.join(objdir, s.replace(".cu", ".o")) for s in SOURCES]
    with ThreadPoolExecutor(max_workers=min(len(SOURCES), os.cpu_count() or 4)) as ex:
        results = list(ex.map(lambda so: _compile(so[0], so[1], extra, verbose), zip(SOURCES, objs)))
    failed = False
    for src, r in zip(SOURCES, results):
        if verbose or r.returncode != 0:
            sys.stdout.write(r.stdout)
            sys.stderr.write(r.stderr)
        failed |= r.returncode != 0
    if failed:
        raise RuntimeError("nvcc failed")
    tmp = lib + f".tmp{os.getpid()}"
    link = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static", "-o", tmp, *objs]
    if verbose:
        print(" ".join(link), flush=True)
    subprocess.run(link, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose=True, ptxas_info="-v" in sys.argv, debug_bounds="--debug-bounds" in sys.argv))
