"""Build libkivi.so (sm_100a) in-tree with nvcc.

The library is plain CUDA C++ with an extern "C" boundary (include/kivi.h);
it links the CUDA runtime statically and depends on nothing else.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libkivi.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
]
LINK_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-cudart", "static"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return os.path.getmtime(LIB) < max(os.path.getmtime(p) for p in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every source to an object in parallel, then link the library."""
    if not force and not _stale():
        return LIB
    import concurrent.futures
    import tempfile

    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = LIB + f".tmp{os.getpid()}"
    with tempfile.TemporaryDirectory(prefix="kivi_build_") as obj_dir:
        objs, cmds = [], []
        for src in sources():
            obj = os.path.join(obj_dir, os.path.basename(src) + ".o")
            objs.append(obj)
            cmds.append([nvcc, *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-c", "-o", obj, src])
        workers = max(1, min(len(cmds), os.cpu_count() or 1))
        with concurrent.futures.ThreadPoolExecutor(workers) as ex:
            for cmd, res in zip(cmds, ex.map(_run(verbose), cmds)):
                if res.returncode != 0:
                    raise subprocess.CalledProcessError(res.returncode, cmd)
        link = [nvcc, *LINK_FLAGS, "-o", tmp, *objs]
        _run(verbose)(link).check_returncode()
    os.replace(tmp, LIB)
    return LIB


def _run(verbose: bool):
    def run(cmd):
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        return subprocess.run(cmd)
    return run


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
