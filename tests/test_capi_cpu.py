"""C-ABI checks that need no GPU: the library loads, exports every function include/nvfp4.h
declares, its size arithmetic agrees with the oracle's independent layout code, and argument
errors are rejected before any device work."""
import ctypes

import numpy as np
import pytest
import torch

import bit_kv_cache_24_b200 as nv
from bit_kv_cache_24_b200 import synth


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


def _fake_cache(heads=2, head_dim=128, slots=3, lens=(5, 0, 7)):
    """A cache descriptor whose arrays are never dereferenced by the argument checks (host
    buffers stand in for the device arrays; the slot lengths are a real host array)."""
    buf = (ctypes.c_uint8 * 4096)()
    base = (ctypes.addressof(buf) + 15) // 16 * 16
    ln = (ctypes.c_int32 * slots)(*lens)
    c = nv._KVCache(1, heads, head_dim, slots, 8, base, base, base, base, base, base,
                    ctypes.cast(ln, ctypes.POINTER(ctypes.c_int32)))
    return c, buf, ln, base


def test_kv_attention_argument_errors():
    L = nv.lib()
    c, buf, ln, base = _fake_cache()
    row = 2 * 128
    slots = (ctypes.c_int32 * 3)(0, 1, 2)

    def call(cache=c, layer=0, sl=slots, n=3, q=base, tq=4, ldq=row, scale=1.0, o=base, ldo=row):
        return L.kv_attention(None if cache is None else ctypes.byref(cache), layer, sl, n, q, tq, ldq, scale, o,
                              ldo, None, None)

    inv, uns = nv.NVFP4_ERR_INVALID_ARG, nv.NVFP4_ERR_UNSUPPORTED
    assert call(cache=None) == inv
    assert call(layer=-1) == inv and call(layer=1) == inv
    assert call(n=0) == inv and call(n=129) == inv
    assert call(sl=(ctypes.c_int32 * 3)(0, 3, 2)) == inv          # slot id out of range
    assert call(tq=-1) == inv
    assert call(scale=float("inf")) == inv and call(scale=float("nan")) == inv
    assert call(ldq=row - 8) == inv and call(ldo=row - 8) == inv
    assert call(q=None) == inv and call(o=None) == inv
    assert call(ldq=row + 4) == uns                                # row stride not a multiple of 8
    assert call(q=base + 2) == uns and call(o=base + 8) == uns     # not 16-byte aligned
    assert call(sl=(ctypes.c_int32 * 1)(1), n=1) == inv            # empty window
    ln[0] = 9                                                      # longer than a slot holds
    assert call() == inv
    ln[0] = 5
    # no queries: nothing to launch, even with no q/o buffers
    assert call(tq=0, q=None, o=None) == nv.NVFP4_OK
    c64, buf64, ln64, base64 = _fake_cache(head_dim=64)
    assert L.kv_attention(ctypes.byref(c64), 0, slots, 3, base64, 4, 128, 1.0, base64, 128, None, None) == uns


@pytest.mark.parametrize("rows,cols", [(1, 16), (3, 17), (128, 256), (130, 96), (300, 512), (4680, 3072)])
def test_scale_layout_conversion_matches_oracle(orc, rows, cols):
    L = nv.lib()
    nb = (cols + 15) // 16
    lin = np.random.default_rng(rows * 7 + cols).integers(0, 256, size=rows * nb, dtype=np.uint8)
    mma = np.full(L.nvfp4_sf_bytes(rows, cols, nv.SF_MMA), 0xAB, dtype=np.uint8)   # padding must be zeroed
    assert L.nvfp4_sf_to_mma(lin.ctypes.data, rows, cols, mma.ctypes.data) == nv.NVFP4_OK
    assert np.array_equal(mma, orc.sf_linear_to_mma(lin, rows, cols))        # the oracle's own layout code
    back = np.zeros(rows * nb, dtype=np.uint8)
    assert L.nvfp4_sf_to_linear(mma.ctypes.data, rows, cols, back.ctypes.data) == nv.NVFP4_OK
    assert np.array_equal(back, lin)


def test_scale_layout_conversion_argument_errors():
    L = nv.lib()
    buf = (ctypes.c_uint8 * 512)()
    assert L.nvfp4_sf_to_linear(None, 4, 32, buf) == nv.NVFP4_ERR_INVALID_ARG
    assert L.nvfp4_sf_to_mma(buf, 0, 32, buf) == nv.NVFP4_ERR_INVALID_ARG
    assert L.nvfp4_sf_to_mma(buf, 4, -1, buf) == nv.NVFP4_ERR_INVALID_ARG


def test_sf_to_linear_of_a_host_qtensor(orc):
    x = synth.ragged(3, 200, 96, "wide")
    _, ref = orc.quantize(x)
    q = nv.QTensor(200, 96, nv.SF_MMA, "cpu")
    q.sf.copy_(torch.from_numpy(orc.sf_linear_to_mma(ref.sf.reshape(-1), 200, 96)))
    assert np.array_equal(nv.sf_to_linear(q).numpy(), ref.sf.reshape(200, -1))


def test_kv_append_that_fails_leaves_slot_length_unchanged():
    """The cache's per-slot token counts are host bookkeeping written when an append is enqueued
    (the ordering rule of nvfp4_kv_cache.len): an append that returns an error, whether from its
    argument checks or (on this GPU-less host) from the device check, must not touch them."""
    L = nv.lib()
    c, buf, ln, base = _fake_cache(heads=2, head_dim=128, slots=3, lens=(5, 0, 7))
    ws = (ctypes.c_uint8 * (L.nvfp4_kv_append_workspace(8, 2, 128) + 16))()
    wsp = (ctypes.addressof(ws) + 15) // 16 * 16
    row = 2 * 128

    def append(slot, ntok, ld=row, k=base):
        return L.kv_quant_append(ctypes.byref(c), 0, slot, k, base, ntok, ld, wsp,
                                 L.nvfp4_kv_append_workspace(8, 2, 128), None, None)

    assert append(1, 9) == nv.NVFP4_ERR_INVALID_ARG               # more tokens than a slot holds
    assert append(3, 4) == nv.NVFP4_ERR_INVALID_ARG               # slot out of range
    assert append(1, 4, ld=row + 4) == nv.NVFP4_ERR_UNSUPPORTED   # row stride not a multiple of 8
    assert append(1, 4, k=base + 2) == nv.NVFP4_ERR_UNSUPPORTED   # K not 16-byte aligned
    if not torch.cuda.is_available():
        assert append(1, 4) in (nv.NVFP4_ERR_CUDA, nv.NVFP4_ERR_UNSUPPORTED)   # no device here
    assert list(ln) == [5, 0, 7]
