"""Build libmoe.so (the CUDA library behind include/moe.h) in-tree, for sm_100a.

nvcc cross-compiles without a GPU, so this runs on any machine with CUDA 12.9.
The CUDA runtime is linked statically; the driver entry point for tensor-map
encoding is looked up at run time, so the library has no libcuda link-time
dependency.
"""
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libmoe.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-I", os.path.join(ROOT, "include"),
]
OBJ_DIR = os.path.join(HERE, "_build")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(ROOT, "include", "moe.h"),
                                                    os.path.abspath(__file__)]


def _obj(src):
    return os.path.join(OBJ_DIR, os.path.basename(src)[:-3] + ".o")


def _stale(target, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every .cu to an object (in parallel), then link libmoe.so."""
    os.makedirs(OBJ_DIR, exist_ok=True)
    hdrs = _headers()
    todo = [src for src in sources() if force or _stale(_obj(src), [src] + hdrs)]
    procs = []
    for src in todo:
        cmd = [NVCC, *NVCC_FLAGS, *(["-Xptxas", "-v"] if verbose else []), "-c", "-o",
               _obj(src) + ".tmp", src]
        procs.append((src, subprocess.Popen(cmd)))
    failed = [src for src, p in procs if p.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, f"nvcc {' '.join(failed)}")
    for src, _ in procs:
        os.replace(_obj(src) + ".tmp", _obj(src))
    objs = [_obj(src) for src in sources()]
    if force or todo or _stale(LIB, objs):
        tmp = LIB + ".tmp"
        subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                               "-Xcompiler", "-fvisibility=hidden", "-o", tmp, *objs])
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose="-v" in sys.argv))
