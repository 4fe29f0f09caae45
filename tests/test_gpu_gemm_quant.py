"""GPU parity of nvfp4_gemm_quant_out: the GEMM epilogue that also emits the row-wise NVFP4
quantization of its BF16 output, with the per-tensor scale of a given amax.

The BF16 output must equal nvfp4_gemm's bit for bit (same kernel, same epilogue arithmetic; the
GEMM itself is checked against the oracle's fp64 GEMM in test_gpu_gemm.py), and the emitted
codes, scales (padding included) and g must equal the oracle's row-wise quantization of that
BF16 output with amax_in, bit for bit -- including an amax below the output's (saturation)."""
import numpy as np
import pytest
import torch

import bit_kv_cache_24_b200 as nv
from bit_kv_cache_24_b200 import synth
from tests.parity_util import assert_quantized_equal

pytestmark = pytest.mark.gpu


def _operands(M, N, K, seed=0):
    a = synth.ragged(seed + M + K, M, K, "outliers").cuda()
    w = synth.ragged(seed + N + 3 * K, N, K, "normal").cuda()
    return nv.nvfp4_quantize(a), nv.nvfp4_quantize(w)


def _amax(y):
    return float(y.float().abs().max().item())


def _run(orc, gA, gW, amax, layout=nv.SF_MMA, bias=None, resid=None):
    amax_t = torch.tensor([amax], dtype=torch.float32, device="cuda")
    y_ref = nv.nvfp4_gemm(gA, gW, bias=bias, resid=resid)
    y, q = nv.nvfp4_gemm_quant_out(gA, gW, amax_t, bias=bias, resid=resid, sf_layout=layout)
    torch.cuda.synchronize()
    assert torch.equal(y.cpu(), y_ref.cpu())
    st, oq = orc.quantize(y.cpu(), amax_in=np.float32(amax))
    assert st == 0
    assert_quantized_equal(orc, q, oq)
    return y, q


@pytest.mark.parametrize("layout", [nv.SF_MMA, nv.SF_LINEAR])
def test_tiny_one_cta_kernel(orc, layout):
    d = synth.tiny()
    gA, gW = nv.nvfp4_quantize(d["A"].cuda()), nv.nvfp4_quantize(d["W"].cuda())
    y = nv.nvfp4_gemm(gA, gW)
    _run(orc, gA, gW, _amax(y), layout)


@pytest.mark.parametrize("M,N,K", [(77, 64, 32), (130, 256, 64), (300, 320, 320), (513, 192, 272)])
@pytest.mark.parametrize("layout", [nv.SF_MMA, nv.SF_LINEAR])
def test_ragged_shapes(orc, M, N, K, layout):
    gA, gW = _operands(M, N, K)
    bias = synth.ragged(7, 1, N, "normal")[0].contiguous().cuda()
    y = nv.nvfp4_gemm(gA, gW, bias=bias)
    _run(orc, gA, gW, _amax(y), layout, bias=bias)


def test_saturating_amax(orc):
    """amax_in below the output's own amax (a scale carried over from another step): blocks
    above it saturate to the largest scale and code, exactly as the quantizer does."""
    gA, gW = _operands(300, 256, 256, seed=11)
    y = nv.nvfp4_gemm(gA, gW)
    _, q = _run(orc, gA, gW, 0.25 * _amax(y))
    sf = q.sf.cpu().numpy()
    assert (sf == 0x7E).any()


def test_residual_and_no_bf16_output(orc):
    M, N, K = 260, 256, 192
    gA, gW = _operands(M, N, K, seed=3)
    resid = synth.ragged(5, M, N, "normal").cuda()
    y = nv.nvfp4_gemm(gA, gW, resid=resid)
    amax = _amax(y)
    _, q1 = _run(orc, gA, gW, amax, resid=resid)
    amax_t = torch.tensor([amax], dtype=torch.float32, device="cuda")
    y2, q2 = nv.nvfp4_gemm_quant_out(gA, gW, amax_t, resid=resid, write_y=False)
    torch.cuda.synchronize()
    assert y2 is None
    assert torch.equal(q1.codes, q2.codes) and torch.equal(q1.sf, q2.sf) and torch.equal(q1.g, q2.g)


def test_qkv_projection_full_size(orc):
    """The QKV projection of one chunk (4680 x 9216 x 3072, + bias): the emitted NVFP4 of Y (the
    K/V slices' and the next layer's operand) against the oracle over all 43 M elements."""
    d = synth.qkv()
    gA, gW = nv.nvfp4_quantize(d["A"].cuda()), nv.nvfp4_quantize(d["W"].cuda())
    bias = d["bias"].cuda()
    y = nv.nvfp4_gemm(gA, gW, bias=bias)
    _run(orc, gA, gW, _amax(y), bias=bias)


def test_nonfinite_amax_reports_and_writes_nothing():
    gA, gW = _operands(130, 128, 64, seed=2)
    q = nv.QTensor(130, 128)
    q.codes.fill_(0xAB)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    amax_t = torch.tensor([float("inf")], dtype=torch.float32, device="cuda")
    nv.nvfp4_gemm_quant_out(gA, gW, amax_t, q_out=q, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == nv.NVFP4_ERR_NONFINITE
    assert bool((q.codes == 0xAB).all())


def test_unsupported_width():
    gA, gW = _operands(130, 96, 64, seed=4)                # N % 64 != 0
    amax_t = torch.ones(1, dtype=torch.float32, device="cuda")
    with pytest.raises(nv.NVFP4Error):
        nv.nvfp4_gemm_quant_out(gA, gW, amax_t)
