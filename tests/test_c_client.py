"""The boundary from C (CPU only): tests/c_abi_client.c includes only
include/coll.h, is compiled as C99 with warnings as errors, linked against
libmvrcoll.so, and run.  It checks the host-side answers (sizes, forms,
error strings, argument rejection before any launch) without Python in
between, so the header is plain C and the library is usable from C."""
import os
import shutil
import subprocess

import pytest

import movement_virtual_rank_b200 as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_client_compiles_links_and_runs(tmp_path):
    M.lib()  # raises if the library has not been built
    libdir = os.path.dirname(M.LIB_PATH)
    exe = tmp_path / "c_abi_client"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_abi_client.c"), "-L", libdir, "-lmvrcoll", f"-Wl,-rpath,{libdir}",
           "-o", str(exe)]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok"
