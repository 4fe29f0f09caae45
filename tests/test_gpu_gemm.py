"""GPU parity of nvfp4_gemm (tcgen05 block-scaled MMA) against the oracle's fp64 GEMM of the
dequantized operands (LongLive-2.0's W4A4 NVFP4 linear layers and NVFP4 training GEMMs: arXiv
abstract, fugumt.com).

Every output element is checked, at full size too (the oracle's fp64 matmul of the dequantized
operands, gemm_full), so the persistent multi-tile loop of the CTA-pair kernel (accumulator
phases, the tensor-memory handoff, tile order) is covered on every tile it computes.

Tolerance (stated with the method's target): max |Y - Y64| <= 1e-3 * sqrt(K) * max|Adeq| *
max|Bdeq| on every element, and on the FP32-output variant of the same kernel a relative
Frobenius error <= 1e-5 (only FP32 accumulation order differs).  BF16 output must equal the
round-to-nearest-even of the kernel's own FP32 output bit for bit (one kernel, two epilogues),
and lie within one BF16 step of the single rounding of the exact fp64 result wherever half a
BF16 step exceeds the FP32 error level the Frobenius bound allows (|Y64| >= 2^9 * 1e-5 *
rms(Y64)); below that level only the max-abs bound applies.  Operands come from the CUDA
quantizer, whose bytes are first checked against the oracle's."""
import numpy as np
import pytest
import torch

import bit_kv_cache_24_b200 as nv
from bit_kv_cache_24_b200 import synth
from tests.parity_util import assert_quantized_equal, gemm_tolerance, rel_fro

pytestmark = pytest.mark.gpu


def _quant_both(orc, x, colwise=False):
    g = nv.nvfp4_quantize(x.cuda(), nv.COLWISE if colwise else nv.ROWWISE)
    _, o = orc.quantize(x, colwise=colwise)
    assert_quantized_equal(orc, g, o)
    return g, o


def _bf16_ordinal(u16):
    """BF16 bit patterns -> integers that are consecutive for adjacent BF16 values."""
    u = u16.astype(np.int32)
    return np.where(u & 0x8000, -(u & 0x7FFF), u)


def _check(orc, gA, oA, gB, oB, rows=None, bias=None, resid=None):
    K = oA.cols
    y16 = nv.nvfp4_gemm(gA, gB, bias=None if bias is None else bias.cuda(),
                        resid=None if resid is None else resid.cuda())
    y32 = nv.nvfp4_gemm(gA, gB, bias=None if bias is None else bias.cuda(),
                        resid=None if resid is None else resid.cuda(), out_dtype=nv.OUT_F32)
    torch.cuda.synchronize()
    y32c = y32.cpu()
    y16c = y16.cpu()
    del y16, y32
    assert torch.equal(y16c, y32c.to(torch.bfloat16))
    if rows is None:
        ref = orc.gemm_full(oA, oB, bias=bias, resid=resid)
        got = y32c.double().numpy()
        got16 = y16c.view(torch.int16).numpy().view(np.uint16)
        adeq = orc.dequant_f64(oA)
    else:
        ref = orc.gemm_rows(oA, oB, rows=rows, bias=bias, resid=resid)
        sel = torch.as_tensor(rows)
        got = y32c[sel].double().numpy()
        got16 = y16c[sel].view(torch.int16).numpy().view(np.uint16)
        adeq = orc.dequant_f64(oA)[rows]
    del y32c, y16c
    amax = np.abs(adeq).max()
    del adeq
    bmax = np.abs(orc.dequant_f64(oB)).max()
    tol = gemm_tolerance(amax, bmax, K)
    err = np.abs(got - ref).max()
    fro = rel_fro(got, ref)
    assert err <= tol, (err, tol)
    assert fro <= 1e-5, fro
    # BF16 output against the single BF16 rounding of the exact result
    del got
    level = 2.0 ** 9 * 1e-5 * np.sqrt(np.mean(ref * ref))
    big = np.abs(ref) >= level
    steps = np.abs(_bf16_ordinal(got16) - _bf16_ordinal(orc.bf16_from_f64(ref)))
    worst = int(steps[big].max()) if big.any() else 0
    assert worst <= 1, ("BF16 output more than one step from bf16(Y64)", worst, int((steps[big] > 1).sum()))
    y16f = (got16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.abs(y16f - ref)[~big].max(initial=0.0) <= tol
    return fro


def test_tiny_w4a4_linear(orc):
    d = synth.tiny()
    gA, oA = _quant_both(orc, d["A"])
    gW, oW = _quant_both(orc, d["W"])
    _check(orc, gA, oA, gW, oW)


@pytest.mark.parametrize("M,N,K", [(1, 8, 16), (77, 64, 32), (130, 256, 64), (128, 264, 96), (300, 520, 320),
                                   (129, 512, 1008), (256, 768, 2048), (513, 256, 272),
                                   # more tiles than CTA pairs: clusters run several tiles each
                                   (4100, 1288, 96), (2333, 4104, 160)])
def test_ragged_shapes(orc, M, N, K):
    a = synth.ragged(M + K, M, K, "outliers")
    w = synth.ragged(N + 3 * K, N, K, "normal")
    gA, oA = _quant_both(orc, a)
    gW, oW = _quant_both(orc, w)
    _check(orc, gA, oA, gW, oW)


def test_bias_and_inplace_residual(orc):
    M, N, K = 200, 264, 512
    gA, oA = _quant_both(orc, synth.ragged(1, M, K, "lognormal"))
    gW, oW = _quant_both(orc, synth.ragged(2, N, K, "normal"))
    bias = synth.ragged(3, 1, N, "normal")[0].contiguous()
    resid = synth.ragged(4, M, N, "normal")
    _check(orc, gA, oA, gW, oW, bias=bias)
    _check(orc, gA, oA, gW, oW, resid=resid)
    # in place: y aliases the residual
    y = resid.cuda().clone()
    nv.nvfp4_gemm(gA, gW, resid=y, out=y)
    y2 = nv.nvfp4_gemm(gA, gW, resid=resid.cuda())
    torch.cuda.synchronize()
    assert torch.equal(y, y2)


def test_full_size_qkv_projection(orc):
    d = synth.qkv()
    gA, oA = _quant_both(orc, d["A"])
    gW, oW = _quant_both(orc, d["W"])
    _check(orc, gA, oA, gW, oW, bias=d["bias"])


def test_full_size_ffn(orc):
    d = synth.ffn()
    gA, oA = _quant_both(orc, d["A_up"])
    gW, oW = _quant_both(orc, d["W_up"])
    _check(orc, gA, oA, gW, oW)
    del gW, oW
    gA2, oA2 = _quant_both(orc, d["A_down"])
    gW2, oW2 = _quant_both(orc, d["W_down"])
    _check(orc, gA2, oA2, gW2, oW2, resid=d["R"])


def test_full_size_training_gemms(orc):
    """fprop X.W^T, dgrad dY.W (B = W^T via column-wise quantization of W) and wgrad dY^T.X
    (both operands column-wise, K = 37440 tokens)."""
    d = synth.train()
    gX, oX = _quant_both(orc, d["X"])
    gW, oW = _quant_both(orc, d["W"])
    _check(orc, gX, oX, gW, oW)
    del gX, oX
    gdY, odY = _quant_both(orc, d["dY"])
    gWt, oWt = _quant_both(orc, d["W"], colwise=True)
    _check(orc, gdY, odY, gWt, oWt)
    del gdY, odY, gWt, oWt
    gdYt, odYt = _quant_both(orc, d["dY"], colwise=True)
    gXt, oXt = _quant_both(orc, d["X"], colwise=True)
    _check(orc, gdYt, odYt, gXt, oXt)
