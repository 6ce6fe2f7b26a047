"""Build libmoe_layout.so (the CUDA library behind include/moe_layout.h) for
B200 (sm_100a) with nvcc, in-tree next to this file.

    python -m combine_moe_layout_06_b200.build [--force] [--verbose-ptxas]
"""
from __future__ import annotations

import concurrent.futures
import glob
import hashlib
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmoe_layout.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2", "-shared", "-cudart", "static",
    "--expt-relaxed-constexpr",
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs() -> list[str]:
    return (sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
            + glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)])


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def build(force: bool = False, verbose_ptxas: bool = False, out: str | None = None,
          defines: tuple = ()) -> str:
    """Compile the library (to `out` instead of the in-tree path when given,
    with extra -D `defines` for the compile-time tunables).  Each source is
    compiled to an object in parallel, then the objects are linked."""
    target = out or LIB
    if out is None and not defines and not force and up_to_date():
        return LIB
    tag = hashlib.sha1(" ".join(defines).encode()).hexdigest()[:8]
    objdir = os.path.join(PKG, "_build", tag)
    os.makedirs(objdir, exist_ok=True)
    base = [NVCC, *FLAGS, *[f"-D{d}" for d in defines], "-I", INCLUDE, "-I", CSRC]
    if verbose_ptxas:
        base.insert(1, "-Xptxas=-v")
    objs = []

    def compile_one(src):
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [c for c in base if c != "-shared"] + ["-c", "-o", obj, src]
        subprocess.run(cmd, check=True)
        return obj

    with concurrent.futures.ThreadPoolExecutor(max_workers=max(1, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(compile_one, sources()))
    tmp = target + f".tmp{os.getpid()}"
    subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart",
                    "static", "-o", tmp, *objs], check=True)
    os.replace(tmp, target)
    return target


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--verbose-ptxas" in sys.argv))
