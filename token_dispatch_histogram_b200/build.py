"""Build libep.so, the sm_100a CUDA library behind include/ep.h.

nvcc -gencode arch=compute_100a,code=sm_100a, static CUDA runtime, in-tree output
(token_dispatch_histogram_b200/libep.so) so the built library travels with the
source tree."""
import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SO = os.path.join(HERE, "libep.so")
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(HERE, "_build")

NVCC_FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
              "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
              "-I" + INCLUDE, "-I" + CSRC]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(INCLUDE, "ep.h"), __file__]


def stale():
    if not os.path.exists(SO):
        return True
    t = os.path.getmtime(SO)
    return any(os.path.getmtime(p) > t for p in _deps())


def build(force=False, verbose=False, extra_flags=()):
    if not force and not stale():
        return SO
    os.makedirs(BUILD_DIR, exist_ok=True)
    objs = []
    procs = []
    for src in sources():
        obj = os.path.join(BUILD_DIR, os.path.basename(src) + ".o")
        cmd = ["nvcc", "-c", src, "-o", obj] + NVCC_FLAGS + list(extra_flags)
        if verbose:
            print(" ".join(cmd))
        procs.append((subprocess.Popen(cmd), src))
        objs.append(obj)
    for p, src in procs:
        if p.wait() != 0:
            raise RuntimeError(f"nvcc failed on {src}")
    tmp = SO + ".tmp"
    subprocess.check_call(["nvcc", "-shared", "-o", tmp] + objs + ["-gencode", "arch=compute_100a,code=sm_100a",
                                                                      "-cudart", "static", "-Xcompiler", "-fPIC"])
    os.replace(tmp, SO)
    return SO


if __name__ == "__main__":
    build(force=True, verbose=True)
