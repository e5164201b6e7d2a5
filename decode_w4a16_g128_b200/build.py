"""Build the in-tree shared library libw4a16.so for sm_100a with nvcc.

The library is one translation unit (csrc/w4a16.cu includes every kernel);
the C ABI it exports is declared in include/w4a16.h at the repository root.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBRARY = os.path.join(HERE, "libw4a16.so")
MAIN = os.path.join(CSRC, "w4a16.cu")


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(INCLUDE, "w4a16.h")])


def command(out: str, extra=()) -> list[str]:
    return [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
            "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE,
            *extra, MAIN, "-o", out]


def build(force: bool = False, verbose: bool = False) -> str:
    stale = (not os.path.exists(LIBRARY) or
             os.path.getmtime(LIBRARY) < max(os.path.getmtime(s) for s in sources()))
    if force or stale:
        tmp = LIBRARY + f".tmp{os.getpid()}"
        cmd = command(tmp, ("-Xptxas", "-v") if verbose else ())
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
        if verbose:
            sys.stderr.write(r.stdout + r.stderr)
        os.replace(tmp, LIBRARY)
    return LIBRARY


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
