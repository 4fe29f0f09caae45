"""GPU parity of nvfp4_gemm (tcgen05 block-scaled MMA) against the oracle's fp64 GEMM of the
dequantized operands.

Tolerance (stated with the method's target): max |Y - Y64| <= 1e-3 * sqrt(K) * max|Adeq| *
max|Bdeq| on every checked element, and on the FP32-output variant of the same kernel a relative
Frobenius error <= 1e-5 (only FP32 accumulation order differs).  BF16 output must equal the
round-to-nearest-even of the kernel's own FP32 output bit for bit (one kernel, two epilogues).
Operands come from the CUDA quantizer, whose bytes are first checked against the oracle's."""
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


def _check(orc, gA, oA, gB, oB, rows=None, bias=None, resid=None):
    K = oA.cols
    y16 = nv.nvfp4_gemm(gA, gB, bias=None if bias is None else bias.cuda(),
                        resid=None if resid is None else resid.cuda())
    y32 = nv.nvfp4_gemm(gA, gB, bias=None if bias is None else bias.cuda(),
                        resid=None if resid is None else resid.cuda(), out_dtype=nv.OUT_F32)
    torch.cuda.synchronize()
    y32c = y32.cpu()
    assert torch.equal(y16.cpu(), y32c.to(torch.bfloat16))
    ref = orc.gemm_rows(oA, oB, rows=rows, bias=bias, resid=resid)
    got = (y32c if rows is None else y32c[torch.as_tensor(rows)]).double().numpy()
    amax = np.abs(orc.dequant_f64(oA)[rows if rows is not None else slice(None)]).max()
    bmax = np.abs(orc.dequant_f64(oB)).max()
    tol = gemm_tolerance(amax, bmax, K)
    err = np.abs(got - ref).max()
    fro = rel_fro(got, ref)
    assert err <= tol, (err, tol)
    assert fro <= 1e-5, fro
    return fro


def test_tiny_w4a4_linear(orc):
    d = synth.tiny()
    gA, oA = _quant_both(orc, d["A"])
    gW, oW = _quant_both(orc, d["W"])
    _check(orc, gA, oA, gW, oW)


@pytest.mark.parametrize("M,N,K", [(1, 8, 16), (77, 64, 32), (130, 256, 64), (128, 264, 96), (300, 520, 320),
                                   (129, 512, 1008), (256, 768, 2048), (513, 256, 272)])
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


def _rows(M, n=40, seed=0):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, M - 1], rng.choice(M, n, replace=False), np.arange(M - (M % 128 or 128), M)[-8:]]))


def test_full_size_qkv_projection(orc):
    d = synth.qkv()
    gA, oA = _quant_both(orc, d["A"])
    gW, oW = _quant_both(orc, d["W"])
    _check(orc, gA, oA, gW, oW, rows=_rows(4680), bias=d["bias"])


def test_full_size_ffn(orc):
    d = synth.ffn()
    gA, oA = _quant_both(orc, d["A_up"])
    gW, oW = _quant_both(orc, d["W_up"])
    _check(orc, gA, oA, gW, oW, rows=_rows(4680, 24, 1))
    del gW, oW
    gA2, oA2 = _quant_both(orc, d["A_down"])
    gW2, oW2 = _quant_both(orc, d["W_down"])
    _check(orc, gA2, oA2, gW2, oW2, rows=_rows(4680, 24, 2), resid=d["R"])


def test_full_size_training_gemms(orc):
    """fprop X.W^T, dgrad dY.W (B = W^T via column-wise quantization of W) and wgrad dY^T.X
    (both operands column-wise, K = 37440 tokens)."""
    d = synth.train()
    gX, oX = _quant_both(orc, d["X"])
    gW, oW = _quant_both(orc, d["W"])
    _check(orc, gX, oX, gW, oW, rows=_rows(37440, 24, 3))
    del gX, oX
    gdY, odY = _quant_both(orc, d["dY"])
    gWt, oWt = _quant_both(orc, d["W"], colwise=True)
    _check(orc, gdY, odY, gWt, oWt, rows=_rows(37440, 24, 4))
    del gdY, odY, gWt, oWt
    gdYt, odYt = _quant_both(orc, d["dY"], colwise=True)
    gXt, oXt = _quant_both(orc, d["X"], colwise=True)
    _check(orc, gdYt, odYt, gXt, oXt, rows=_rows(3072, 24, 5))
