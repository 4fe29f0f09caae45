"""GPU parity of kv_attention (the restore fused into attention) against the oracle's fp64
attention over the restored window.

Tolerance, from the kernel's arithmetic (per head h, output column c):
    |O - O_ref| <= 2^-8 * (|O_ref| + max_j |v[j, h, c]|)
- The probabilities are rounded to BF16 for the P.V product while their sum stays FP32. This
  perturbs each weight by at most 2^-9 relative, hence O by at most 2^-9 * max_j |v[j, h, c]|.
- The output is rounded to BF16, adding at most 2^-9 * |O|.
- The FP32 accumulation of scores and products and the hardware exp2 approximation (relative
  error ~2^-22; results below 2^-126 flush to 0) stay orders of magnitude below these two terms
  at these sizes.
The K and V the kernel multiplies are the restore's values bit for bit (same rounding steps), so
a one-token window returns that token's V exactly.
"""
import math

import numpy as np
import pytest
import torch

import bit_kv_cache_24_b200 as nv
from bit_kv_cache_24_b200 import synth

pytestmark = pytest.mark.gpu
D = 128


def _tol_check(got, ref, vdeq):
    """got, ref [tq, H, D]; vdeq the window's V [Tk, H, D] (float)."""
    vmax = np.abs(vdeq).max(axis=0)                              # [H, D]
    tol = 2.0 ** -8 * (np.abs(ref) + vmax[None])
    err = np.abs(got - ref)
    worst = float((err / tol).max())
    assert np.isfinite(got).all()
    assert worst <= 1.0, f"max error / tolerance = {worst:.3f}"
    return worst


def _fill(orc, heads, lens, seed=0):
    cache = nv.KVCache(1, heads, D, len(lens), max(max(lens), 1), "cuda")
    model = orc.KVCacheModel(1, heads, D, len(lens), max(max(lens), 1))
    for s, n in enumerate(lens):
        if n == 0:
            continue
        k, v = synth.kv_chunk(seed, s, tokens=n)
        k, v = k[:, :heads].contiguous(), v[:, :heads].contiguous()
        nv.kv_quant_append(cache, 0, s, k.cuda(), v.cuda())
        model.append(0, s, k, v)
    return cache, model


@pytest.mark.parametrize("heads,lens,order,tq", [
    (2, (45, 80), (1, 0), 70),               # slot boundary inside a tile, ragged last tile, 2 CTAs
    (1, (64, 64, 64), (0, 1, 2), 64),        # tile-aligned window, one full CTA
    (2, (200, 0, 17), (2, 1, 0), 129),       # an empty slot, 3 CTAs with a one-row tail
    (3, (5,), (0,), 3),                      # window shorter than a tile
    (2, (130, 260), (0, 1), 300),            # two CTAs of two 128-row Q tiles, the last partly live
])
def test_matches_oracle(orc, heads, lens, order, tq):
    cache, model = _fill(orc, heads, lens)
    q = synth.normal(7 + tq, 0, (tq, heads, D))
    scale = 1.0 / math.sqrt(D)
    o = nv.kv_attention(cache, 0, list(order), q.cuda(), scale)
    torch.cuda.synchronize()
    live = [s for s in order if lens[s] > 0]
    ref = model.attention(0, live, q, scale)
    _, vbits = model.dequant(0, live)
    _tol_check(o.float().cpu().numpy(), ref, orc.bf16_bits_to_f32(vbits))


def test_one_token_window_returns_its_value_exactly(orc):
    # one token: its weight is exp2(0) = 1 and the sum is 1, so O = v bit for bit
    heads = 4
    cache, model = _fill(orc, heads, (1,))
    q = synth.normal(3, 0, (9, heads, D))
    o = nv.kv_attention(cache, 0, [0], q.cuda(), 0.3)
    _, v = nv.kv_dequant(cache, 0, [0])
    torch.cuda.synchronize()
    assert torch.equal(o.cpu(), v.cpu().expand(9, heads, D))


def test_q_from_fused_qkv_layout(orc):
    # q = the first third of a [tq, 3 * heads * D] QKV output: row stride 3 * heads * D
    heads, tq = 4, 100
    cache, model = _fill(orc, heads, (90, 33), seed=1)
    y = synth.normal(5, 0, (tq, 3 * heads * D))
    qv = y.cuda()[:, : heads * D]
    out = torch.full((tq, heads * D + 64), float("nan"), dtype=torch.bfloat16, device="cuda")[:, : heads * D]
    o = nv.kv_attention(cache, 0, [0, 1], qv, 0.07, out=out)
    torch.cuda.synchronize()
    q = y[:, : heads * D].contiguous().view(tq, heads, D)
    ref = model.attention(0, [0, 1], q, 0.07)
    _, vbits = model.dequant(0, [0, 1])
    _tol_check(o.float().cpu().numpy().reshape(tq, heads, D), ref, orc.bf16_bits_to_f32(vbits))


def test_full_window_sampled_rows(orc):
    # the 12-slot window of the QKV step: 24 heads, 12 x 4680 tokens, 4680 queries; the oracle
    # checks sampled rows (first and last rows of CTAs and the tail), one head at a time
    heads, slots, tok = 24, 12, 4680
    cache = nv.KVCache(1, heads, D, slots, tok, "cuda")
    model = orc.KVCacheModel(1, heads, D, slots, tok)
    for s in range(slots):
        k, v = synth.kv_chunk(0, s)
        nv.kv_quant_append(cache, 0, s, k.cuda(), v.cuda())
        model.append(0, s, k, v)
    q = synth.normal(21, 0, (tok, heads, D))
    scale = 1.0 / math.sqrt(D)
    o = nv.kv_attention(cache, 0, list(range(slots)), q.cuda(), scale).float().cpu().numpy()
    rows = [0, 63, 64, 2047, 4095, 4608, tok - 1]
    kbits, vbits = model.dequant(0, list(range(slots)))
    for h in (0, 7, 23):
        ref = orc.attention(q[rows][:, h:h + 1], kbits[:, h:h + 1], vbits[:, h:h + 1], scale)
        _tol_check(o[rows][:, h:h + 1], ref, orc.bf16_bits_to_f32(vbits[:, h:h + 1]))


def test_argument_errors(orc):
    cache, _ = _fill(orc, 2, (10, 0))
    q = torch.zeros(4, 2, D, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nv.NVFP4Error) as e:
        nv.kv_attention(cache, 0, [1], q, 1.0)               # empty window
    assert e.value.status == nv.NVFP4_ERR_INVALID_ARG
    with pytest.raises(nv.NVFP4Error) as e:
        nv.kv_attention(cache, 0, [0], q, float("inf"))
    assert e.value.status == nv.NVFP4_ERR_INVALID_ARG
    small = nv.KVCache(1, 2, 64, 1, 8, "cuda")
    k = torch.zeros(8, 2, 64, dtype=torch.bfloat16, device="cuda")
    nv.kv_quant_append(small, 0, 0, k, k)
    with pytest.raises(nv.NVFP4Error) as e:
        nv.kv_attention(small, 0, [0], torch.zeros(4, 2, 64, dtype=torch.bfloat16, device="cuda"), 1.0)
    assert e.value.status == nv.NVFP4_ERR_UNSUPPORTED
    # no queries: nothing to do
    out = nv.kv_attention(cache, 0, [0], q[:0], 1.0)
    assert out.shape == (0, 2, D)


def test_negative_scale(orc):
    # the row maximum of scale * s is the scale times the row minimum of s when scale < 0
    heads = 2
    cache, model = _fill(orc, heads, (100, 40), seed=3)
    q = synth.normal(11, 0, (50, heads, D))
    o = nv.kv_attention(cache, 0, [0, 1], q.cuda(), -0.06)
    torch.cuda.synchronize()
    ref = model.attention(0, [0, 1], q, -0.06)
    _, vbits = model.dequant(0, [0, 1])
    _tol_check(o.float().cpu().numpy(), ref, orc.bf16_bits_to_f32(vbits))
