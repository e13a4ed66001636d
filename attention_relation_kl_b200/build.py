"""Build librelkl.so in-tree for sm_100a (B200) with nvcc.

    python -m attention_relation_kl_b200.build        # or build() from Python

The library is placed next to this file so that it travels with the source
tree.  nvcc cross-compiles without a GPU.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "librelkl.so")
SOURCES = ["relkl_api.cu", "relkl_tc.cu", "relkl_simt.cu", "relkl_chain.cu", "relkl_gemm.cu"]
HEADERS = ["relkl_device.cuh", "relkl_params.h"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "relkl.h"))
    deps.append(__file__)
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, checks: bool = False) -> str:
    """Compile librelkl.so if any source is newer; returns its path.

    ``checks`` (or RELKL_CHECKS=1 in the environment) builds the debug variant
    that replays every tensor-core launch's schedule on the host first
    (relkl_check_schedule) and refuses a launch whose schedule is unsound."""
    checks = checks or os.environ.get("RELKL_CHECKS") == "1"
    if not force and not checks and not _stale():
        return LIB
    tmp = LIB + ".tmp"
    cmd = [nvcc_path(), *NVCC_FLAGS, *(["-DRELKL_CHECKS"] if checks else []),
           "-I", os.path.join(ROOT, "include"),
           *[os.path.join(CSRC, f) for f in SOURCES], "-ldl", "-o", tmp]
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, checks="--checks" in sys.argv))
