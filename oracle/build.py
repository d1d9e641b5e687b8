"""Compile the CPU oracle (plain C) into ``oracle/liboracle.so``.

Test infrastructure: the library path never builds or loads this.
Flags: IEEE binary32 semantics in source order (no contraction into fused
multiply-add, no fast-math), single-threaded code.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "bq_oracle.c")
HDR = os.path.join(HERE, "bq_oracle.h")
LIB = os.path.join(HERE, "liboracle.so")

CFLAGS = ["-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math",
          "-fexcess-precision=standard", "-fPIC", "-shared", "-Wall", "-Wextra"]


def compile_oracle(src=SRC, out=LIB, extra=()):
    """Compile ``src`` into the shared library ``out``; returns ``out``."""
    cmd = ["gcc", *CFLAGS, *extra, "-I", HERE, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def build(force=False):
    """Build liboracle.so when it is missing or older than its sources."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= max(os.path.getmtime(SRC), os.path.getmtime(HDR))):
        return LIB
    return compile_oracle()


if __name__ == "__main__":
    print(build(force=True))
