"""Build the CPU oracle (liboracle.so) with gcc.  Test infrastructure only."""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SO = os.path.join(HERE, "liboracle.so")


def build(force=False, defines=(), out=None):
    """Compile oracle.c.  `defines`/`out` exist for the mutation tests, which
    build deliberately broken copies of the oracle to prove the pins catch them."""
    src = os.path.join(HERE, "oracle.c")
    target = out or SO
    stale = (not os.path.exists(target) or os.path.getmtime(target) < max(os.path.getmtime(src),
                                                                           os.path.getmtime(__file__)))
    if force or stale or defines:
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math", "-Wall",
               "-o", target, src]
        cmd += ["-D" + d for d in defines]
        subprocess.check_call(cmd)
    return target


if __name__ == "__main__":
    build(force=True)
