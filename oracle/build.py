"""Compile the oracle into oracle/liboracle.so with the host C compiler.

The oracle is test infrastructure: only the tests, the package smoke check and
the benchmark's CPU-baseline leg load it. Flags: no fused-multiply-add
contraction (-ffp-contract=off) and no fast-math, so the C source's operation
order is the one executed.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "vattn_oracle.c")
OUT = os.path.join(HERE, "liboracle.so")
CFLAGS = ["-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
          "-Wall", "-Wextra", "-Wno-unused-parameter"]


def build(src=SRC, out=OUT, extra=()):
    """Build `src` into the shared library `out`; returns `out`."""
    cmd = ["gcc", *CFLAGS, *extra, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def needs_build(src=SRC, out=OUT):
    return not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src)


if __name__ == "__main__":
    print(build(*sys.argv[1:2] or [SRC]))
