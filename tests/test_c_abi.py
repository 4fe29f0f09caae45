"""The boundary is a C ABI: a plain C11 program (tests/c/abi_check.c) includes include/nvfp4.h,
links libnvfp4.so and calls it, with no Python or C++ in between. Needs gcc; no GPU."""
import os
import shutil
import subprocess

import pytest

import bit_kv_cache_24_b200 as nv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_client_builds_links_and_runs(tmp_path):
    nv.lib()                                              # the library must exist (raises otherwise)
    libdir = os.path.dirname(nv.LIB_PATH)
    exe = tmp_path / "abi_check"
    subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
                           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_check.c"),
                           "-L", libdir, "-lnvfp4", f"-Wl,-rpath,{libdir}", "-o", str(exe)])
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "c abi ok"
