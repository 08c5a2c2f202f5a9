"""Build the sm_100a CUDA library in-tree (libcsa_b200.so next to this file)."""

from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(HERE, "libcsa_b200.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))


def sources_sha(files: list[str] | None = None) -> str:
    """Hash of kernel sources (ties a profile to the code it measured): the given files
    under csrc/, or every source plus the ABI header."""
    import hashlib

    h = hashlib.sha256()
    paths = ([os.path.join(HERE, "csrc", f) for f in files] if files else
             sorted(glob.glob(os.path.join(HERE, "csrc", "*"))) +
             [os.path.join(HERE, "..", "include", "csa.h")])
    for f in paths:
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def build(force: bool = False, verbose: bool = False) -> str:
    srcs = sources()
    deps = srcs + glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + [
        os.path.join(HERE, "..", "include", "csa.h")]
    if not force and os.path.exists(LIB) and all(
            os.path.getmtime(LIB) >= os.path.getmtime(d) for d in deps):
        return LIB
    tmp = LIB + f".{os.getpid()}.tmp"
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xptxas", "-v" if verbose else "-O3", "-o", tmp, *srcs]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
