"""GPU tests of the GEMM's column-group amax (nvfp4_gemm_colamax) and of the KV append that takes
it (kv_quant_append_amax): the BF16 output must equal nvfp4_gemm's bit for bit, each group's amax
must equal max |Y| over that group of the returned BF16 output exactly, and a KV append given the
K and V slices' amax must write the same cache bytes as the append that computes it."""
import numpy as np
import pytest
import torch

import bit_kv_cache_24_b200 as nv
from bit_kv_cache_24_b200 import synth

pytestmark = pytest.mark.gpu


def _check(gA, gW, group, bias=None, resid=None):
    y_ref = nv.nvfp4_gemm(gA, gW, bias=bias, resid=resid)
    y, amax = nv.nvfp4_gemm_colamax(gA, gW, group, bias=bias, resid=resid)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
    want = y.float().abs().reshape(y.shape[0], -1, group).amax(dim=(0, 2))
    assert torch.equal(amax, want), (amax, want)
    return y, amax


@pytest.mark.parametrize("M,N,K,group", [(77, 768, 64, 256), (128, 256, 256, 256), (300, 512, 320, 256),
                                         (513, 1024, 272, 512)])
def test_group_amax_ragged(M, N, K, group):
    a = synth.ragged(M + 5, M, K, "outliers").cuda()
    w = synth.ragged(N + 7, N, K, "normal").cuda()
    bias = synth.ragged(9, 1, N, "normal")[0].contiguous().cuda()
    _check(nv.nvfp4_quantize(a), nv.nvfp4_quantize(w), group, bias=bias)


def test_qkv_projection_and_kv_append_from_epilogue_amax():
    """The fused QKV projection of one chunk: the K and V slices' amax from the GEMM epilogue feed
    the KV append, which must then write exactly what the self-contained append writes."""
    d = synth.qkv()
    gA, gW = nv.nvfp4_quantize(d["A"].cuda()), nv.nvfp4_quantize(d["W"].cuda())
    y, amax = _check(gA, gW, 3072, bias=d["bias"].cuda())
    c1 = nv.KVCache(1, 24, 128, 2, 4680)
    c2 = nv.KVCache(1, 24, 128, 2, 4680)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.kv_quant_append(c1, 0, 1, y[:, 3072:6144], y[:, 6144:], status=st)
    nv.kv_quant_append(c2, 0, 1, y[:, 3072:6144], y[:, 6144:], status=st, amax_kv=amax[1:])
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    half = c1.codes_k.numel() // 2
    hs = c1.sf_k.numel() // 2
    for a, b, n in ((c1.codes_k, c2.codes_k, half), (c1.codes_v, c2.codes_v, half), (c1.sf_k, c2.sf_k, hs),
                    (c1.sf_v, c2.sf_v, hs)):
        assert torch.equal(a[n:], b[n:])                   # slot 1
    assert torch.equal(c1.g_k[1:], c2.g_k[1:]) and torch.equal(c1.g_v[1:], c2.g_v[1:])


def test_nonfinite_amax_kv_reports():
    c = nv.KVCache(1, 2, 64, 1, 32)
    k = synth.ragged(3, 32, 128, "normal").cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    amax = torch.tensor([float("nan"), 1.0], device="cuda")
    nv.kv_quant_append(c, 0, 0, k, k, status=st, amax_kv=amax)
    torch.cuda.synchronize()
    assert int(st.item()) == nv.NVFP4_ERR_NONFINITE


def test_unsupported_group():
    gA = nv.nvfp4_quantize(synth.ragged(1, 130, 64, "normal").cuda())
    gW = nv.nvfp4_quantize(synth.ragged(2, 384, 64, "normal").cuda())
    with pytest.raises(nv.NVFP4Error):
        nv.nvfp4_gemm_colamax(gA, gW, 128)                 # group not a multiple of 256
    with pytest.raises(nv.NVFP4Error):
        nv.nvfp4_gemm_colamax(gA, gW, 256)                 # N not a multiple of the group
