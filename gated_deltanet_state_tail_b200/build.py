"""Build the Tail-Replay CUDA library in-tree (sm_100a).

    python -m gated_deltanet_state_tail_b200.build

produces gated_deltanet_state_tail_b200/libgdn_tail_replay.so from csrc/*.cu,
and the debug build libgdn_tail_replay_debug.so (-DGDN_DEBUG_BOUNDS: every
kernel checks the global indices it computes against the plan's extents and
reports GDN_ERR_BOUNDS instead of accessing out of range).
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libgdn_tail_replay.so")
DEBUG_LIB = os.path.join(PKG, "libgdn_tail_replay_debug.so")
BUILD_DIR = os.path.join(PKG, "_build")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def _nvcc():
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(ROOT, "include", "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def _build_one(lib, defines, objdir, verbose):
    os.makedirs(objdir, exist_ok=True)
    objs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [_nvcc(), *NVCC_FLAGS, *defines, "-I", os.path.join(ROOT, "include"), "-I", CSRC,
               "-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd))
        subprocess.check_call(cmd)
        objs.append(obj)
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp, *objs,
           "-lcudart", "-lcuda"]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> str:
    """Build the release library (and, with `debug`, the bounds-checked one); returns
    the release library's path."""
    if force or _stale(LIB):
        _build_one(LIB, [], BUILD_DIR, verbose)
    if debug and (force or _stale(DEBUG_LIB)):
        _build_one(DEBUG_LIB, ["-DGDN_DEBUG_BOUNDS"], os.path.join(BUILD_DIR, "debug"), verbose)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, debug="--no-debug" not in sys.argv)
