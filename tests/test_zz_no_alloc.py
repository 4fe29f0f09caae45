"""nvfp4_quantize_noalloc: the quantizer for callers that cannot allocate (engine plugin hooks,
embedded host programs that hand over only their input and output buffers).  It must give the
same bytes as nvfp4_quantize, which takes a caller-provided workspace, and as the CPU oracle, on
consecutive calls that share its static scratch array.  Called here directly through the C ABI.

This file is collected last on purpose; it passes both alone in a fresh process and after the
rest of the suite."""
import ctypes

import pytest
import torch

import bit_kv_cache_24_b200 as nv
from bit_kv_cache_24_b200 import synth
from tests.parity_util import assert_quantized_equal

pytestmark = pytest.mark.gpu


def _noalloc(x, direction, sf_layout, status):
    M, K = x.shape
    out = nv.QTensor(M, K, sf_layout) if direction == nv.ROWWISE else nv.QTensor(K, M, sf_layout)
    st = out.struct()
    rc = nv.lib().nvfp4_quantize_noalloc(ctypes.c_void_p(x.data_ptr()), M, K, x.stride(0), direction,
                                         ctypes.byref(st), ctypes.c_void_p(status.data_ptr()),
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == nv.NVFP4_OK, nv.lib().nvfp4_last_error()
    return out


def _same(a, b):
    assert torch.equal(a.codes, b.codes)
    assert torch.equal(a.sf, b.sf)
    assert torch.equal(a.g, b.g)


def test_noalloc_matches_workspace_quantizer_on_consecutive_calls(orc):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    x1 = synth.ragged(21, 4680, 3072, "lognormal").cuda()          # large: fills many scratch slots
    x2 = synth.ragged(22, 130, 96, "outliers").cuda()              # small: fewer slots
    first = _noalloc(x1, nv.ROWWISE, nv.SF_MMA, status)
    second = _noalloc(x2, nv.COLWISE, nv.SF_LINEAR, status)        # reuses the slots of the first
    torch.cuda.synchronize()
    assert status.item() == 0
    _same(first, nv.nvfp4_quantize(x1, nv.ROWWISE, sf_layout=nv.SF_MMA))
    _same(second, nv.nvfp4_quantize(x2, nv.COLWISE, sf_layout=nv.SF_LINEAR))
    # and once more on the first input after the scratch held the second call's partials
    third = _noalloc(x1, nv.ROWWISE, nv.SF_MMA, status)
    torch.cuda.synchronize()
    _same(third, first)
    # the bytes themselves against the CPU oracle
    assert_quantized_equal(orc, first, orc.quantize(x1.cpu())[1], "no-alloc row-wise")
    assert_quantized_equal(orc, second, orc.quantize(x2.cpu(), colwise=True)[1], "no-alloc column-wise")


def test_noalloc_rejects_bad_arguments_without_launching():
    x = torch.zeros(16, 32, dtype=torch.bfloat16, device="cuda")
    out = nv.QTensor(16, 32)
    st = out.struct()
    assert nv.lib().nvfp4_quantize_noalloc(None, 16, 32, 32, nv.ROWWISE, ctypes.byref(st), None, None) == \
        nv.NVFP4_ERR_INVALID_ARG
    assert nv.lib().nvfp4_quantize_noalloc(ctypes.c_void_p(x.data_ptr()), 16, 32, 32, nv.COLWISE,
                                           ctypes.byref(st), None, None) == nv.NVFP4_ERR_INVALID_ARG
    # both layouts in one call are not offered here (one output tensor)
    assert nv.lib().nvfp4_quantize_noalloc(ctypes.c_void_p(x.data_ptr()), 16, 32, 32, nv.ROWCOL,
                                           ctypes.byref(st), None, None) == nv.NVFP4_ERR_INVALID_ARG
