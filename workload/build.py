"""Build the seeded input generators: libgen.so (host, gcc) and
libgen_dev.so (its CUDA twin, nvcc for sm_100a).  Both are inputs-only."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
HOST_SO = os.path.join(HERE, "libgen.so")
DEV_SO = os.path.join(HERE, "libgen_dev.so")


def _stale(target, sources):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def build_host(force=False):
    src = os.path.join(HERE, "gen.c")
    if force or _stale(HOST_SO, [src, __file__]):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
                               "-Wall", "-o", HOST_SO, src, "-lm"])
    return HOST_SO


def build_device(force=False):
    src = os.path.join(HERE, "gen_dev.cu")
    if force or _stale(DEV_SO, [src, __file__]):
        subprocess.check_call(["nvcc", "-O3", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
                               "-Xcompiler", "-fPIC", "-shared", "-o", DEV_SO, src])
    return DEV_SO


def build(force=False):
    build_host(force)
    build_device(force)


if __name__ == "__main__":
    build(force=True)
