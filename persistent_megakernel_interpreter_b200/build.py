"""Build libmk.so in-tree with nvcc for sm_100a (no JIT, no torch extension).

``python -m persistent_megakernel_interpreter_b200.build`` or ``build_library()``.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmk.so")
SOURCES = ["api.cu", "megakernel.cu", "megakernel_trace.cu", "baseline.cu", "noalloc.cu", "select.cu", "pack.cpp",
           "schedule.cpp"]
HEADERS = ["mk_internal.h", "mk_device.cuh", "pack.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "mk.h"),
                                                                 os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps)


def build_library(force: bool = False, verbose: bool = False, extra: list[str] | None = None) -> str:
    """Compile every source to an object in parallel, then link libmk.so."""
    if not force and not _stale():
        return LIB
    tag = f".tmp{os.getpid()}"
    common = [_nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
              "--expt-relaxed-constexpr", f"-I{INCLUDE}", f"-I{CSRC}"] + list(extra or [])
    if verbose:
        common.insert(1, "-Xptxas=-v")
    objs = [os.path.join(CSRC, f + tag + ".o") for f in SOURCES]

    def compile_one(i: int) -> None:
        cmd = common + ["-c", "-o", objs[i], os.path.join(CSRC, SOURCES[i])]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.check_call(cmd)

    try:
        with ThreadPoolExecutor(max_workers=min(len(SOURCES), os.cpu_count() or 1)) as ex:
            list(ex.map(compile_one, range(len(SOURCES))))
        subprocess.check_call([_nvcc(), *ARCH, "-shared", "-o", LIB + tag] + objs)
        os.replace(LIB + tag, LIB)
    finally:
        for o in objs:
            if os.path.exists(o):
                os.remove(o)
    return LIB


if __name__ == "__main__":
    build_library(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
