"""The C ABI from plain C: tests/c_abi_check.c, compiled as C99 with warnings as
errors against include/rssm.h and linked to the in-tree librssm.so, runs the
calls that need no GPU."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "hybrid_ssm_decode_replayssm_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_header_compiles_as_c99_and_library_links():
    if not os.path.exists(os.path.join(PKG, "librssm.so")):
        pytest.fail("librssm.so is not built")
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "c_abi_check")
        subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "c_abi_check.c"), "-L", PKG, "-lrssm",
                        "-Wl,-rpath," + PKG, "-o", exe], check=True)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
        assert r.returncode == 0, f"check {r.returncode} failed: {r.stdout} {r.stderr}"
        assert "c abi ok" in r.stdout
