"""Build libabattn.so in-tree with nvcc for sm_100a.

Usage: python -m block_sparse_attention_ibcs_b200.build [--verbose-ptxas]
"""

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "abattn.cu")
OUT = os.path.join(HERE, "libabattn.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def nvcc_cmd(verbose_ptxas: bool = False):
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-shared", "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include"),
           "-I", os.path.join(HERE, "csrc"), SRC, "-o", OUT, "-cudart", "static"]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    return cmd


def sources():
    d = os.path.join(HERE, "csrc")
    return [os.path.join(d, f) for f in os.listdir(d)] + [os.path.join(ROOT, "include", "abattn.h")]


def up_to_date() -> bool:
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if force or verbose_ptxas or not up_to_date():
        r = subprocess.run(nvcc_cmd(verbose_ptxas), capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("nvcc failed building libabattn.so")
        if verbose_ptxas:
            sys.stderr.write(r.stderr)
    return OUT


if __name__ == "__main__":
    build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv)
    print(OUT)
