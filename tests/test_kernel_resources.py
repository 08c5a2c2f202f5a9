"""Compile-time resources of the sm_100a kernels, read from ptxas's own report (no GPU):
no kernel or device function spills registers to local memory."""

import os
import re
import shutil

import pytest

from long_context_compressed_layer_b200 import build as b


def test_no_register_spills(tmp_path):
    try:
        b.nvcc()
    except RuntimeError:
        pytest.skip("no nvcc")
    if not shutil.which("g++"):
        pytest.skip("no host compiler")
    objs, log = b.compile_objects(b.sources(), str(tmp_path), verbose=True)
    entries = re.findall(r"Compiling entry function '(\w+)'", log)
    assert len(entries) >= 10, "ptxas printed no resource report"
    spills = re.findall(r"(\d+) bytes spill stores, (\d+) bytes spill loads", log)
    assert spills and all(s == ("0", "0") for s in spills), [
        line for line in log.splitlines() if "spill" in line and " 0 bytes spill stores" not in line]
    assert len(objs) == len(b.sources()) and all(os.path.getsize(o) > 0 for o in objs)
