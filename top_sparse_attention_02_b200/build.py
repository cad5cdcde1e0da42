"""Build libtsa.so (the CUDA kernels and the C ABI) in-tree with nvcc for sm_100a.

Also builds libtsa_debug.so, a test-only variant of the same sources whose
bounded device waits give up after a few polls and which exports one knob,
tsa_debug_skip_tile, that leaves a chosen tile's load out so that the waits on
it run out (the failure-detection test).  The product library has neither."""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libtsa.so")
BUILD_DIR = os.path.join(PKG, "_build")
DEBUG_LIB = os.path.join(PKG, "libtsa_debug.so")
DEBUG_BUILD_DIR = os.path.join(PKG, "_build_debug")
DEBUG_FLAGS = ["-DTSA_WAIT_SPINS=1024", "-DTSA_DEBUG_KNOBS"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xptxas", "-v",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(target: str, deps: list) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile every csrc/*.cu to an object (in parallel), then link libtsa.so
    (debug: the same sources with DEBUG_FLAGS into libtsa_debug.so)."""
    nvcc = _nvcc()
    build_dir, lib, extra = (DEBUG_BUILD_DIR, DEBUG_LIB, DEBUG_FLAGS) if debug else (BUILD_DIR, LIB, [])
    os.makedirs(build_dir, exist_ok=True)
    headers = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))
    objs, procs = [], []
    for src in sources():
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        objs.append(obj)
        if force or _stale(obj, [src] + headers):
            log = open(obj + ".log", "w")
            procs.append((src, subprocess.Popen([nvcc, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj],
                                                stdout=log, stderr=subprocess.STDOUT), obj + ".log"))
    failed = []
    for src, p, log in procs:
        if p.wait() != 0:
            failed.append((src, log))
    if failed:
        msg = "\n".join(f"--- {s}\n" + open(l).read() for s, l in failed)
        raise RuntimeError("nvcc failed:\n" + msg)
    if verbose:
        for _, _, log in procs:
            sys.stdout.write(open(log).read())
    if force or procs or _stale(lib, objs):
        tmp = lib + f".tmp{os.getpid()}"
        subprocess.check_call([nvcc, *ARCH, "-shared", "-o", tmp, *objs])
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
