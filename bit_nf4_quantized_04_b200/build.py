"""Build libqnf4.so in-tree for sm_100a (B200) with nvcc.

Run ``python bit_nf4_quantized_04_b200/build.py`` (or call ``build()``; this file is
loaded by path, since importing the package loads the library). The library
links the CUDA runtime statically and finds the driver's tensor-map encoder at run
time, so it loads on a machine without a GPU (entry points then report a CUDA error).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libqnf4.so")
# The checked build: the same library with index checks in the kernels (-DQNF4_CHECKED);
# an index outside its buffer is skipped and reported by qnf4_check as QNF4_ERR_BOUNDS.
LIB_CHECKED = os.path.join(HERE, "libqnf4_checked.so")
SOURCES = ["api.cu", "codebook.cpp"]
HEADERS = ["common.cuh", "quant.cuh", "chanq.cuh", "gemm.cuh", "decode.cuh", "loftq.cuh", "tables.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libqnf4.so")


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "qnf4.h"))
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(d) > t for d in deps if os.path.exists(d))


def _cmd(lib: str, extra: list[str]) -> list[str]:
    return [_nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
            "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
            "-I", os.path.join(ROOT, "include"), *extra,
            *[os.path.join(CSRC, f) for f in SOURCES], "-ldl", "-o", lib + ".tmp"]


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None,
          checked: bool = True) -> str:
    """Compile libqnf4.so (and, with checked=True, libqnf4_checked.so) if any source is
    newer; the two compilations run in parallel. Returns the main library's path."""
    jobs = []
    if force or _stale(LIB):
        jobs.append((LIB, _cmd(LIB, list(extra or []))))
    if checked and (force or _stale(LIB_CHECKED)):
        jobs.append((LIB_CHECKED, _cmd(LIB_CHECKED, ["-DQNF4_CHECKED", *(extra or [])])))
    procs = []
    for lib, cmd in jobs:
        if verbose:
            print(" ".join(cmd), flush=True)
        procs.append((lib, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.PIPE,
                                            text=True)))
    failed = []
    for lib, pr in procs:
        out, err = pr.communicate()
        if pr.returncode != 0:
            sys.stderr.write(out + err)
            failed.append(os.path.basename(lib))
        else:
            if verbose and (out or err):
                sys.stderr.write(out + err)
            os.replace(lib + ".tmp", lib)
    if failed:
        raise RuntimeError("nvcc failed building " + ", ".join(failed))
    return LIB


if __name__ == "__main__":
    force = "--force" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None
    print(build(force=force, verbose=True, extra=extra, checked="--no-checked" not in sys.argv))
