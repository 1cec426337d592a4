"""Build step for libhashgrid.so: compiles the CUDA sources of ``csrc/`` for sm_100a with
nvcc into this package's folder (in-tree, so the built library travels with the sources).

    python multiresolution_hash_grid_b200/build.py [--force] [--verbose] [--checked]

(Run it by path: importing the package itself needs the built library.)

``--verbose`` passes ``-Xptxas -v`` (registers, spills, shared memory per kernel).
``--checked`` builds libhashgrid_checked.so instead, with -DHASHGRID_CHECKED: every global
memory access of the kernels is range-checked against the buffers of its call and a
violation is returned as HASHGRID_ERR_DEVICE_CHECK (the binding loads it when the
environment sets HASHGRID_CHECKED=1).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libhashgrid.so")
LIB_CHECKED = os.path.join(HERE, "libhashgrid_checked.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build libhashgrid.so")


def sources() -> list[str]:
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def deps() -> list[str]:
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    return files + [os.path.abspath(__file__)]


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in deps())


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    lib = LIB_CHECKED if checked else LIB
    if not force and not needs_build(lib):
        return lib
    tmp = lib + ".tmp.%d" % os.getpid()
    cmd = [nvcc(), *ARCH, "-lineinfo", "-O3", "-std=c++17", "--expt-relaxed-constexpr",
           "-Xcompiler", "-fPIC,-O2,-Wall", "-shared", "-I", INCLUDE, "-I", CSRC,
           "-o", tmp, *sources()]
    if checked:
        cmd += ["-DHASHGRID_CHECKED"]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, checked="--checked" in sys.argv))
