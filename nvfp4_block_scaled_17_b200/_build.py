"""Build step for the CUDA library: nvcc -> an in-tree shared object.

Compiles every ``csrc/*.cu`` for sm_100a only (``-gencode
arch=compute_100a,code=sm_100a``), one object per file in parallel under ``_build/``,
and links them with the CUDA runtime linked statically, so the library does not
depend on the runtime version PyTorch ships.  No GPU is needed to build.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libnvfp4_b200.so"
LIB_PATH = os.path.join(PKG, LIB_NAME)

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared", "-cudart", "static",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the NVFP4 CUDA library cannot be built")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def inputs() -> list[str]:
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
                              + glob.glob(os.path.join(INCLUDE, "*.h"))) + [__file__]


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(f) <= t for f in inputs())


OBJ_DIR = os.path.join(ROOT, "_build")


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None) -> str:
    """Each translation unit is compiled to an object in parallel (they share no device
    symbols), then nvcc links the shared object."""
    if not force and up_to_date():
        return LIB_PATH
    from concurrent.futures import ThreadPoolExecutor
    os.makedirs(OBJ_DIR, exist_ok=True)
    tag = f"{os.getpid()}"
    compile_flags = [f for f in NVCC_FLAGS if f != "-shared"]
    jobs = []
    for src in sources():
        obj = os.path.join(OBJ_DIR, os.path.basename(src) + f".{tag}.o")
        cmd = [nvcc(), *compile_flags, "-I", INCLUDE, "-I", CSRC, *(extra or []), "-c", "-o", obj, src]
        jobs.append((cmd, obj))
    if verbose:
        for cmd, _ in jobs:
            print(" ".join(cmd), file=sys.stderr)
    with ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 1)) as ex:
        results = list(ex.map(lambda j: subprocess.run(j[0], capture_output=True, text=True), jobs))
    failed = [r for r in results if r.returncode != 0]
    for r in results:
        if r.stderr:
            print(r.stderr, file=sys.stderr, end="")
    if failed:
        for _, obj in jobs:
            if os.path.exists(obj):
                os.remove(obj)
        raise RuntimeError("nvcc failed for " + ", ".join(r.args[-1] for r in failed))
    tmp = LIB_PATH + f".{tag}.tmp"
    link = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static",
            "-Xcompiler", "-fPIC", "-o", tmp, *[obj for _, obj in jobs]]
    if verbose:
        print(" ".join(link), file=sys.stderr)
    try:
        subprocess.run(link, check=True)
    finally:
        for _, obj in jobs:
            if os.path.exists(obj):
                os.remove(obj)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
