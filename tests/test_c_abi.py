"""The boundary as a C ABI: a C99 program that includes only include/csa.h compiles with
warnings as errors, links against the library and sees the documented host-side status
codes (no GPU needed)."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "long_context_compressed_layer_b200")


def test_c99_client_compiles_links_and_runs(tmp_path):
    if not shutil.which("gcc"):
        pytest.skip("no C compiler")
    lib = os.path.join(PKG, "libcsa_b200.so")
    if not os.path.exists(lib):
        pytest.skip("library not built")
    exe = str(tmp_path / "abi_check")
    subprocess.check_call([
        "gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
        "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_check.c"),
        "-L", PKG, "-lcsa_b200", "-Wl,-rpath," + PKG, "-o", exe])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
