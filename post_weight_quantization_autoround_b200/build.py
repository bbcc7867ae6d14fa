"""Build libautoround.so in-tree with nvcc for sm_100a.

    python -m post_weight_quantization_autoround_b200.build [--verbose-ptxas]

Compiles every ``csrc/*.cu`` with relocatable device code (one status word is
shared by all translation units) into ``_build/obj`` and links a shared library
next to this file.
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


def _compile(args):
    cmd, = args
    subprocess.run(cmd, check=True)


def build(verbose_ptxas: bool = False, extra=None, out: str = LIB, jobs: int | None = None) -> str:
    """Compiles each source to a relocatable object (in parallel, only those
    older than a source or header), then device-links them into ``out``."""
    srcs = sources()
    obj_dir = os.path.join(ROOT, "_build", "obj")
    os.makedirs(obj_dir, exist_ok=True)
    common = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-rdc=true", "-Xcompiler", "-fPIC",
              "-Xcompiler", "-fvisibility=hidden", "-I", os.path.join(ROOT, "include")]
    if verbose_ptxas:
        common = ["-Xptxas", "-v", *common]
    if extra:
        common = [*extra, *common]
    headers = glob.glob(os.path.join(HERE, "csrc", "*.h")) + glob.glob(os.path.join(HERE, "csrc", "*.cuh"))
    headers += glob.glob(os.path.join(ROOT, "include", "*.h"))
    newest_header = max((os.path.getmtime(h) for h in headers), default=0.0)
    stamp = os.path.join(obj_dir, "flags.txt")
    flags = " ".join(common)
    same_flags = os.path.exists(stamp) and open(stamp).read() == flags
    objs, todo = [], []
    for src in srcs:
        obj = os.path.join(obj_dir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        fresh = (same_flags and os.path.exists(obj)
                 and os.path.getmtime(obj) >= max(os.path.getmtime(src), newest_header))
        if not fresh or verbose_ptxas:
            todo.append(([nvcc_path(), *common, "-dc", "-o", obj, src],))
    if todo:
        from concurrent.futures import ThreadPoolExecutor

        with ThreadPoolExecutor(max_workers=jobs or os.cpu_count() or 4) as ex:
            list(ex.map(_compile, todo))
        with open(stamp, "w") as f:
            f.write(flags)
    subprocess.run([nvcc_path(), *ARCH, "-shared", "-rdc=true", "-Xcompiler", "-fPIC", "-o", out, *objs], check=True)
    return out


if __name__ == "__main__":
    build(verbose_ptxas="--verbose-ptxas" in sys.argv)
    print(LIB)
