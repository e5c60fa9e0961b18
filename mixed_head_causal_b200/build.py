"""Builds libsaf.so (the sm_100a CUDA library behind include/saf.h) in-tree.

    python -m mixed_head_causal_b200.build [--force] [--checked]

nvcc compiles every csrc/*.cu for sm_100a only (``-gencode
arch=compute_100a,code=sm_100a``), links the CUDA runtime statically and
writes mixed_head_causal_b200/libsaf.so next to this file (with --checked:
libsaf_checked.so, the kernels' index checks compiled in, for tests).
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libsaf.so")
# the checked build: index checks compiled in (-DSAF_CHECKED), for tests
LIB_CHECKED = os.path.join(HERE, "libsaf_checked.so")
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    """Builds libsaf.so, or with `checked` libsaf_checked.so: the same sources
    with the kernels' index checks compiled in (SAF_CHECKED_OK records a failed
    check in the workspace error word and the access it guards is skipped)."""
    lib = LIB_CHECKED if checked else LIB
    if not force and not _stale(lib):
        return lib
    objdir = os.path.join(ROOT, "_build", "checked" if checked else "regular")
    os.makedirs(objdir, exist_ok=True)
    flags = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
             "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE,
             "--expt-relaxed-constexpr"]
    if checked:
        flags += ["-DSAF_CHECKED"]
    if verbose:
        flags += ["-Xptxas", "-v"]
    objs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [nvcc(), *flags, "-c", src, "-o", obj]
        subprocess.check_call(cmd)
        objs.append(obj)
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.check_call([nvcc(), "-shared", "-cudart", "static", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-o", tmp, *objs])
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, checked="--checked" in sys.argv))
