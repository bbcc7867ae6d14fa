"""Build libautoround.so in-tree with nvcc for sm_100a.

    python -m post_weight_quantization_autoround_b200.build [--verbose-ptxas]

Compiles every ``csrc/*.cu`` with relocatable device code (one status word is
shared by all translation units) and links a shared library next to this file.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libautoround.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libautoround.so")
    return cand


def sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))


def build(verbose_ptxas: bool = False, extra=None, out: str = LIB) -> str:
    srcs = sources()
    cmd = [
        nvcc_path(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-rdc=true", "-shared",
        "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
        "-I", os.path.join(ROOT, "include"),
        "-o", out, *srcs,
    ]
    if verbose_ptxas:
        cmd[1:1] = ["-Xptxas", "-v"]
    if extra:
        cmd[1:1] = list(extra)
    subprocess.run(cmd, check=True)
    return out


def up_to_date(out: str = LIB) -> bool:
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    deps = sources() + glob.glob(os.path.join(HERE, "csrc", "*.h")) + glob.glob(os.path.join(HERE, "csrc", "*.cuh"))
    deps += glob.glob(os.path.join(ROOT, "include", "*.h"))
    return all(os.path.getmtime(d) <= t for d in deps)


if __name__ == "__main__":
    build(verbose_ptxas="--verbose-ptxas" in sys.argv)
    print(LIB)
