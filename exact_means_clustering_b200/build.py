"""Builds libfkm.so in-tree with nvcc for sm_100a.

    python -m exact_means_clustering_b200.build [--force] [--verbose] [--checked]

--checked builds libfkm_checked.so instead: the same sources with
FKM_CHECKED defined, so the kernels verify the indices they gather and
scatter with and record an out-of-range one in the status word (instead of
touching memory); the binding loads it when FKM_LIB_VARIANT=checked.

Sources: csrc/*.cu; public header: include/fkm.h.  The CUDA runtime is linked
statically and the driver's tensor-map encoder is looked up at run time, so
the library loads on a machine without a GPU driver (its entry points then
return FKM_ERR_CUDA).
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libfkm.so")
LIB_CHECKED = os.path.join(HERE, "libfkm_checked.so")
BUILD_DIR = os.path.join(ROOT, "_build")
BUILD_DIR_CHECKED = os.path.join(ROOT, "_build_checked")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
    "-I" + INCLUDE, "-I" + CSRC,
]


def _nvcc() -> str:
    for c in ("/usr/local/cuda/bin/nvcc", "nvcc"):
        if os.path.sep not in c or os.path.exists(c):
            return c
    return "nvcc"


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib=LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + [os.path.join(INCLUDE, "fkm.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    lib = LIB_CHECKED if checked else LIB
    bdir = BUILD_DIR_CHECKED if checked else BUILD_DIR
    if not force and not _stale(lib):
        return lib
    os.makedirs(bdir, exist_ok=True)
    objs = []
    procs = []
    for src in sources():
        obj = os.path.join(bdir, os.path.basename(src) + ".o")
        cmd = [_nvcc(), *NVCC_FLAGS, *(["-DFKM_CHECKED"] if checked else []), "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT,
                                            text=True)))
        objs.append(obj)
    failed = []
    for src, p in procs:
        out, _ = p.communicate()
        if verbose or p.returncode != 0:
            sys.stdout.write(out)
        if p.returncode != 0:
            failed.append(src)
    if failed:
        raise RuntimeError("nvcc failed for: " + ", ".join(failed))
    tmp = lib + f".tmp{os.getpid()}"
    link = [_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp, *objs,
            "-Xcompiler", "-fvisibility=hidden"]
    subprocess.run(link, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                checked="--checked" in sys.argv))
