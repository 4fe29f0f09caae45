"""C-ABI checks that need no GPU: the library loads, exports every function include/nvfp4.h
declares, its size arithmetic agrees with the oracle's independent layout code, and argument
errors are rejected before any device work."""
import ctypes

import pytest

import bit_kv_cache_24_b200 as nv


def test_library_exports_every_header_function():
    L = nv.lib()
    names = nv.header_functions()
    assert len(names) >= 15
    for n in ["nvfp4_quantize", "nvfp4_gemm", "kv_quant_append", "kv_dequant", "nvfp4_amax"]:
        assert n in names
    for n in names:
        assert hasattr(L, n), n
    assert L.nvfp4_version() >= 100


@pytest.mark.parametrize("rows,cols", [(1, 16), (128, 256), (4680, 3072), (3072, 4680), (37440, 3072), (3, 17)])
def test_layout_sizes_match_oracle(orc, rows, cols):
    L = nv.lib()
    assert L.nvfp4_codes_pitch(cols) == orc.codes_pitch(cols)
    assert L.nvfp4_sf_bytes(rows, cols, nv.SF_LINEAR) == rows * orc.sf_pitch(cols)
    assert L.nvfp4_sf_bytes(rows, cols, nv.SF_MMA) == orc.sf_mma_bytes(rows, cols)
    assert L.nvfp4_sf_bytes(rows, cols, 7) == -1


def test_kv_cache_sizes():
    L = nv.lib()
    # 30 layers x 12 slots x 4680 tokens x 3072: codes 0.5 B, scales 1/16 B per element
    n = 30 * 12 * 4680 * 3072
    assert L.nvfp4_kv_cache_bytes(30, 24, 128, 12, 4680, 0) == n // 2
    assert L.nvfp4_kv_cache_bytes(30, 24, 128, 12, 4680, 1) == n // 16
    assert L.nvfp4_kv_cache_bytes(30, 24, 128, 12, 4680, 2) == 30 * 12 * 4
    assert L.nvfp4_kv_cache_bytes(0, 24, 128, 12, 4680, 0) == -1


def test_argument_errors_are_synchronous():
    L = nv.lib()
    t = nv._Tensor(None, None, None, 4, 32, nv.SF_MMA)
    assert L.nvfp4_quantize(None, 4, 32, 32, 0, None, ctypes.byref(t), None, 0, None, None) == nv.NVFP4_ERR_INVALID_ARG
    assert L.nvfp4_gemm(None, None, None, None, None, 0, 0, None, None) == nv.NVFP4_ERR_INVALID_ARG
    assert L.kv_dequant(None, 0, None, 0, None, None, None, None) == nv.NVFP4_ERR_INVALID_ARG
    for s in range(6):
        assert L.nvfp4_status_string(s)
