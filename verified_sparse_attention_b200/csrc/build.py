"""Build libvattn.so (the C-ABI library) for sm_100a with nvcc, in-tree.

    python -m verified_sparse_attention_b200.csrc.build [--ptxas-verbose]
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
PKG = os.path.dirname(HERE)
ROOT = os.path.dirname(PKG)
SRCS = [os.path.join(HERE, "vattn_api.cu"), os.path.join(HERE, "vattn_static.cu")]
DEPS = [*SRCS, os.path.join(HERE, "vattn_kernels.cuh"), os.path.join(HERE, "vattn_device.cuh"),
        os.path.join(ROOT, "include", "vattn.h")]
OUT = os.path.join(PKG, "libvattn.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"), "-I", HERE]


def needs_build():
    if not os.path.exists(OUT):
        return True
    t = os.path.getmtime(OUT)
    return any(os.path.getmtime(d) > t for d in DEPS)


def build(verbose_ptxas=False, out=OUT):
    cmd = [NVCC, *FLAGS, *SRCS, "-o", out]
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(verbose_ptxas="--ptxas-verbose" in sys.argv))
