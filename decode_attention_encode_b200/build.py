"""Builds liblla.so, the sm_100a CUDA library, in-tree with nvcc.

    python -m decode_attention_encode_b200.build [--force] [--verbose] [--check]

--check builds the bounds-check variant, liblla_check.so (LLA_BOUNDS_CHECK:
every computed global access of the kernels is tested against the extent of
its buffer; a miss sets a device status bit and is not made). The binding
loads it instead of liblla.so when LLA_LIBRARY_VARIANT=check.
"""

from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "liblla.so")
LIB_CHECK = os.path.join(PKG, "liblla_check.so")


def lib_path(variant: str = "release") -> str:
    """The library file of a build variant ("release" or "check")."""
    if variant not in ("release", "check"):
        raise ValueError(f"unknown library variant {variant!r}")
    return LIB_CHECK if variant == "check" else LIB

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(path: str = LIB) -> bool:
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(
        os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, variant: str = "release") -> str:
    """Compile every .cu under csrc/ into one shared library (sm_100a)."""
    out = lib_path(variant)
    if not force and not _stale(out):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc_path(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "--shared",
           "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "-I", INCLUDE, "-o", tmp, *sources()]
    if variant == "check":
        cmd.insert(1, "-DLLA_BOUNDS_CHECK")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    proc = subprocess.run(cmd, capture_output=True, text=True)
    if proc.returncode != 0:
        sys.stderr.write(proc.stdout + proc.stderr)
        raise RuntimeError("nvcc failed building liblla.so")
    if verbose:
        sys.stderr.write(proc.stdout + proc.stderr)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                variant="check" if "--check" in sys.argv else "release"))
