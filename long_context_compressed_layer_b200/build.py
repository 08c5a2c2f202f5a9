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


def compile_objects(srcs: list[str], outdir: str, verbose: bool = False) -> tuple[list[str], str]:
    """Compile each source to an object in outdir with the library's flags, all at once on
    the host's cores (a faster check of every translation unit than build()); returns
    the objects and the compilers' combined output (ptxas's resource report with verbose).
    Raises CalledProcessError, carrying that output, if any source fails."""
    from concurrent.futures import ThreadPoolExecutor

    def one(src):
        obj = os.path.join(outdir, os.path.basename(src) + ".o")
        cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
               "-Xptxas", "-v" if verbose else "-O3", "-c", "-o", obj, src]
        r = subprocess.run(cmd, capture_output=True, text=True)
        return obj, r.returncode, cmd, r.stdout + r.stderr

    with ThreadPoolExecutor(max(1, min(len(srcs), os.cpu_count() or 1))) as ex:
        res = list(ex.map(one, srcs))
    log = "".join(r[3] for r in res)
    for _, rc, cmd, out in res:
        if rc:
            raise subprocess.CalledProcessError(rc, cmd, output=log, stderr=out)
    return [r[0] for r in res], log


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
