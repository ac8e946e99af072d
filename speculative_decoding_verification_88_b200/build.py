"""Build libspecverify.so (sm_100a) in-tree with nvcc.

    python -m speculative_decoding_verification_88_b200.build [--force]

The library lands in ``speculative_decoding_verification_88_b200/_lib/`` so
that it travels with the source tree; it links the CUDA runtime statically.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_DIR = os.path.join(PKG, "_lib")
LIB_PATH = os.path.join(LIB_DIR, "libspecverify.so")
# The same sources built with every global index checked against its buffer
# (SV_DEBUG_BOUNDS): a violation raises SV_FLAG_BOUNDS instead of an access.
# For tests, in place of a memory checker; never the default library.
BOUNDS_LIB_PATH = os.path.join(LIB_DIR, "libspecverify_bounds.so")

SOURCES = ["sv_api.cu", "sv_kernels.cu", "sv_noalloc.cu", "sv_tree_stoch.cu"]
HEADERS = [os.path.join(CSRC, h) for h in ("sv_internal.h", "sv_device.cuh")] + [
    os.path.join(INCLUDE, "spec_verify.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; set NVCC or add the CUDA toolkit to PATH")


def _stale(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    deps = [os.path.join(CSRC, s) for s in SOURCES] + HEADERS + [os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra_flags: list[str] | None = None,
          bounds: bool = False) -> str:
    """Compile the library if a source is newer than it (or `force`);
    `bounds` builds the bounds-checked variant instead."""
    path = BOUNDS_LIB_PATH if bounds else LIB_PATH
    if not force and not _stale(path):
        return path
    os.makedirs(LIB_DIR, exist_ok=True)
    tmp = path + f".tmp{os.getpid()}"
    flags = [*(extra_flags or []), *(["-DSV_DEBUG_BOUNDS"] if bounds else [])]
    cmd = [nvcc_path(), *NVCC_FLAGS, *flags, f"-I{INCLUDE}", f"-I{CSRC}",
           "-o", tmp, *[os.path.join(CSRC, s) for s in SOURCES]]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, path)
    return path


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers / spills")
    a = ap.parse_args()
    print(build(force=a.force or a.ptxas_info, verbose=True,
                extra_flags=["-Xptxas", "-v"] if a.ptxas_info else None))
