"""The bounds-checked debug build (libnvfp4_checked.so, compiled with NVFP4_DEBUG_CHECKS): every
kernel access whose address comes from index arithmetic is compared with its buffer's extent,
which the host derives from the caller's tensor shapes, and an access outside it is skipped with
NVFP4_ERR_OUT_OF_BOUNDS in the status word instead of faulting.  It stands in for a memory
checker, which is not available on every GPU host.

1. The check is live in the checked build and absent in the release build (a guarded write into
   a buffer whose declared extent is smaller than its allocation, so neither build can write
   outside memory).
2. The GPU parity suite, rerun in a child process against the checked build, passes with every
   status word at 0 (tests/conftest.py checks the binding's own words after each test)."""
import ctypes
import os
import subprocess
import sys

import pytest
import torch

import bit_kv_cache_24_b200 as nv
from bit_kv_cache_24_b200 import build

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SELFTEST = r"""
import ctypes, sys, torch
import bit_kv_cache_24_b200 as nv
L = nv.lib()
buf = torch.zeros(1024, dtype=torch.uint8, device="cuda")
st = torch.zeros(1, dtype=torch.int32, device="cuda")
def call(extent, index):
    st.zero_(); buf.zero_()
    rc = L.nvfp4_selftest_bounds(ctypes.c_void_p(buf.data_ptr()), extent, index, ctypes.c_void_p(st.data_ptr()),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return rc, int(st.item()), int(buf[index].item())
print(int(L.nvfp4_checked_build()), *call(512, 100), *call(512, 600))
"""


def _run(code, lib_path, timeout=300):
    env = dict(os.environ, NVFP4_LIB=lib_path)
    return subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=timeout)


def test_bounds_check_is_live_only_in_the_checked_build():
    checked = build.build(checked=True)
    r = _run(SELFTEST, checked)
    assert r.returncode == 0, r.stderr[-2000:]
    flag, rc_in, st_in, b_in, rc_out, st_out, b_out = map(int, r.stdout.split())
    assert flag == 1
    assert (rc_in, st_in, b_in) == (nv.NVFP4_OK, 0, 0xAB)                    # inside: written
    assert (rc_out, st_out, b_out) == (nv.NVFP4_OK, nv.NVFP4_ERR_OUT_OF_BOUNDS, 0)   # outside: skipped
    r = _run(SELFTEST, build.build())
    assert r.returncode == 0, r.stderr[-2000:]
    flag, rc_in, st_in, b_in, rc_out, st_out, b_out = map(int, r.stdout.split())
    assert flag == 0 and (st_in, b_in) == (0, 0xAB) and (st_out, b_out) == (0, 0xAB)   # no check


def test_gpu_parity_suite_under_the_checked_build():
    checked = build.build(checked=True)
    files = ["tests/test_gpu_quantize.py", "tests/test_gpu_kv.py", "tests/test_gpu_gemm.py",
             "tests/test_gpu_gemm_quant.py", "tests/test_gpu_colamax.py", "tests/test_gpu_attention.py",
             "tests/test_gpu_sink_cache.py", "tests/test_gpu_launch_chain.py", "tests/test_gpu_codecs.py",
             "tests/test_gpu_sp_exchange.py", "tests/test_zz_no_alloc.py"]
    env = dict(os.environ, NVFP4_LIB=checked)
    # the full-size workloads are covered by the release run; the checked rerun keeps the ragged
    # and multi-tile shapes, which exercise every index path of every kernel
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "gpu", "-k", "not full_size and not full_window and not full_cache",
                        "-p", "no:cacheprovider", *files], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=2400)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
