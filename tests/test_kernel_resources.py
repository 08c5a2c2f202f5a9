"""Compile-time resources of the sm_100a kernels, read from ptxas's own report (no GPU):
no kernel or device function spills registers to local memory."""

import os
import re
import shutil
import subprocess

import pytest

from long_context_compressed_layer_b200 import build as b


def test_no_register_spills(tmp_path):
    try:
        nvcc = b.nvcc()
    except RuntimeError:
        pytest.skip("no nvcc")
    if not shutil.which("g++"):
        pytest.skip("no host compiler")
    out = subprocess.run([nvcc, *b.ARCH, "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
                          "-Xptxas", "-v", "-o", str(tmp_path / "lib.so"), *b.sources()],
                         capture_output=True, text=True)
    assert out.returncode == 0, out.stderr[-2000:]
    log = out.stdout + out.stderr
    entries = re.findall(r"Compiling entry function '(\w+)'", log)
    assert len(entries) >= 10, "ptxas printed no resource report"
    spills = re.findall(r"(\d+) bytes spill stores, (\d+) bytes spill loads", log)
    assert spills and all(s == ("0", "0") for s in spills), [
        line for line in log.splitlines() if "spill" in line and " 0 bytes spill stores" not in line]
    assert os.path.getsize(tmp_path / "lib.so") > 0
