"""The boundary from C (CPU): tests/c/abi_smoke.c, a C99 program that includes include/moe.h
and links the in-tree library, compiles with -Wall -Wextra -pedantic -Werror and runs the calls
that need no device (sizes, argument errors, the T == 0 no-op, status strings)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "fine_grained_mixture_route_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_c_program_compiles_links_and_runs(tmp_path):
    lib = os.path.join(PKG, "libmoe_b200.so")
    if not os.path.exists(lib):
        pytest.fail("libmoe_b200.so is missing: build it with `python -m fine_grained_mixture_route_b200.build`")
    exe = str(tmp_path / "abi_smoke")
    cc = ["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
          os.path.join(ROOT, "tests", "c", "abi_smoke.c"), "-L", PKG, "-lmoe_b200", f"-Wl,-rpath,{PKG}", "-o", exe]
    r = subprocess.run(cc, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert "sm_100a" in r.stdout
