"""Ordering of chained launches.  Every kernel is launched with programmatic stream serialization;
two kernels deliberately start before their predecessor ends (the column pass of a both-layouts
quantization runs alongside the row pass).  These tests consume outputs immediately, with no
host synchronisation, across long mixed chains, and require bit-identical results to the same
work run with a device synchronisation after every call."""
import pytest
import torch

import bit_kv_cache_24_b200 as nv
from bit_kv_cache_24_b200 import synth

pytestmark = pytest.mark.gpu


def test_rowcol_outputs_consumed_at_once():
    M, K, N = 512, 256, 128
    x = synth.ragged(61, M, K, "outliers").cuda()
    d = synth.ragged(62, M, N, "normal").cuda()
    w = synth.ragged(63, N, K, "normal").cuda()
    Wq, Dc = nv.nvfp4_quantize(w), nv.nvfp4_quantize(d, nv.COLWISE)
    Xr_ref, Xc_ref = nv.nvfp4_quantize(x), nv.nvfp4_quantize(x, nv.COLWISE)
    torch.cuda.synchronize()
    y_ref = nv.nvfp4_gemm(Xr_ref, Wq)                      # fprop with the row-wise operand
    g_ref = nv.nvfp4_gemm(Xc_ref, Dc)                      # wgrad X^T dY with the column-wise ones
    torch.cuda.synchronize()
    for _ in range(10):
        Xr, Xc = nv.nvfp4_quantize(x, nv.ROWCOL)
        y = nv.nvfp4_gemm(Xr, Wq)
        g = nv.nvfp4_gemm(Xc, Dc)
        torch.cuda.synchronize()
        assert torch.equal(y, y_ref) and torch.equal(g, g_ref)


def _chain(sync, iters=20):
    out = []
    cache = nv.KVCache(1, 4, 64, 4, 256, "cuda")
    W = nv.nvfp4_quantize(synth.ragged(70, 768, 256, "normal").cuda())
    amax = torch.tensor([40.0], device="cuda")
    s = (lambda: torch.cuda.synchronize()) if sync else (lambda: None)
    for i in range(iters):
        a = synth.ragged(100 + i, 256, 256, ["normal", "outliers", "lognormal", "wide"][i % 4]).cuda()
        Ar, Ac = nv.nvfp4_quantize(a, nv.ROWCOL); s()
        y = nv.nvfp4_gemm(Ar, W); s()
        nv.kv_quant_append(cache, 0, i % 4, y[:, 256:512], y[:, 512:]); s()
        K, V = nv.kv_dequant(cache, 0, [(i + j) % 4 for j in range(4)] if i >= 3 else [0]); s()
        y2, q = nv.nvfp4_gemm_quant_out(Ar, W, amax); s()
        out += [Ar.codes, Ar.sf, Ac.codes, Ac.sf, y, K, V, y2, q.codes, q.sf]
    torch.cuda.synchronize()
    return [t.clone() for t in out]


def test_mixed_chain_without_synchronisation():
    ref = _chain(sync=True)
    for _ in range(3):
        got = _chain(sync=False)
        assert all(torch.equal(a, b) for a, b in zip(got, ref))
