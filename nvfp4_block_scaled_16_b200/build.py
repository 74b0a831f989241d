"""Build ``libnvfp4.so`` (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m nvfp4_block_scaled_16_b200.build [--force] [--verbose] [--debug]

``--debug`` builds ``libnvfp4_debug.so`` instead: the same kernels with every plain global
load and store index checked against its operand's extent (NVFP4_DEBUG_INDEX; a failed
check skips the access and records NVFP4_ERR_INDEX in the device status word).  The
binding loads it when NVFP4_LIBRARY=debug.

The library is plain CUDA C++ with an ``extern "C"`` surface (``include/nvfp4.h``);
it links the CUDA runtime statically and fetches ``cuTensorMapEncodeTiled`` from the
driver at run time, so it needs neither PyTorch nor -lcuda.
"""
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libnvfp4.so")
LIB_DEBUG = os.path.join(PKG, "libnvfp4_debug.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden",
         "-Xptxas", "-warn-spills", "--expt-relaxed-constexpr"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib=LIB):
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra=(), debug=None) -> str:
    """Builds the release library, or the debug one when `debug` (default: NVFP4_LIBRARY=debug)."""
    if debug is None:
        debug = os.environ.get("NVFP4_LIBRARY") == "debug"
    lib = LIB_DEBUG if debug else LIB
    if not force and not _stale(lib):
        return lib
    if debug:
        extra = (*extra, "-DNVFP4_DEBUG_INDEX")
    objdir = os.path.join(ROOT, "_build_debug" if debug else "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    procs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [NVCC, *ARCH, *FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
            print(" ".join(cmd))
        procs.append((subprocess.Popen(cmd), src))
        objs.append(obj)
    failed = [src for p, src in procs if p.wait() != 0]
    if failed:
        raise RuntimeError(f"nvcc failed for {failed}")
    tmp = lib + ".tmp"
    subprocess.run([NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"], check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, debug="--debug" in sys.argv))
