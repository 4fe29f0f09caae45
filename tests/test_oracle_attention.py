"""Pins for the oracle's fp64 attention over a restored KV window.

LongLive-2.0 keeps the KV cache in NVFP4 and restores it for attention (d9249.github.io review,
section "핵심 아이디어 / 구조 / 동작 방식"); attention itself is the textbook softmax attention.
The oracle is pinned against:
- torch's scaled_dot_product_attention in float64, a library routine with its own code;
- closed forms: a constant V, all-zero keys, one dominant key;
- invariants: key order, independence of heads, and the slot order of a cache window.
The shapes are non-square (Tq != Tk != D, H > 1), so a transposed operand or a mixed-up head
index fails at least one pin.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from bit_kv_cache_24_b200 import synth


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _qkv(seed, tq, tk, heads, d):
    q = synth.normal(seed, 0, (tq, heads, d))
    k = synth.normal_with_outliers(seed, 1, (tk, heads, d), 0.02, 15.0)
    v = synth.normal(seed, 2, (tk, heads, d))
    return q, k, v


@pytest.mark.parametrize("tq,tk,heads,d,scale", [(5, 37, 3, 16, 0.25), (1, 1, 1, 16, 1.0), (7, 64, 2, 128, 1 / math.sqrt(128)),
                                                 (3, 130, 4, 32, 0.0371)])
def test_matches_library_sdpa(orc, tq, tk, heads, d, scale):
    q, k, v = _qkv(tq * 31 + tk, tq, tk, heads, d)
    got = orc.attention(q, _bits(k), _bits(v), scale)
    # library routine on [H, T, D] float64 operands, the same FP32 scale value
    qh, kh, vh = (t.to(torch.float64).permute(1, 0, 2) for t in (q, k, v))
    ref = F.scaled_dot_product_attention(qh, kh, vh, scale=float(np.float32(scale))).permute(1, 0, 2).numpy()
    assert got.shape == (tq, heads, d)
    assert np.max(np.abs(got - ref)) <= 1e-12 * max(1.0, np.abs(ref).max())


def test_constant_values_give_the_constant(orc):
    # softmax weights sum to one: with v[j] = c for every token, O = c whatever q and k are
    tq, tk, heads, d = 4, 23, 2, 16
    q, k, _ = _qkv(3, tq, tk, heads, d)
    c = synth.normal(3, 9, (1, heads, d))
    v = c.expand(tk, heads, d).contiguous()
    got = orc.attention(q, _bits(k), _bits(v), 0.5)
    want = np.broadcast_to(c.to(torch.float64).numpy(), got.shape)
    assert np.max(np.abs(got - want)) <= 1e-14 * np.abs(want).max()


def test_zero_keys_give_the_mean_value(orc):
    # every exponent is 0, so the weights are uniform and O is the mean of v over the tokens
    tq, tk, heads, d = 3, 19, 2, 16
    q, _, v = _qkv(4, tq, tk, heads, d)
    k = torch.zeros(tk, heads, d, dtype=torch.bfloat16)
    got = orc.attention(q, _bits(k), _bits(v), 0.7)
    mean = v.to(torch.float64).numpy().mean(axis=0)
    assert np.max(np.abs(got - mean[None])) <= 1e-14 * np.abs(mean).max()


def test_one_dominant_key(orc):
    # q = e0, k[j*] = 32 e0 and every other key 0, scale 1: the exponents are 32 for j* and 0
    # elsewhere, so O = (e^32 v[j*] + sum_{j != j*} v[j]) / (e^32 + tk - 1)
    tq, tk, heads, d, js = 2, 11, 2, 16, 6
    _, _, v = _qkv(5, tq, tk, heads, d)
    q = torch.zeros(tq, heads, d, dtype=torch.bfloat16)
    q[:, :, 0] = 1.0
    k = torch.zeros(tk, heads, d, dtype=torch.bfloat16)
    k[js, :, 0] = 32.0
    got = orc.attention(q, _bits(k), _bits(v), 1.0)
    vf = v.to(torch.float64).numpy()
    e = math.exp(32.0)
    want = (e * vf[js] + vf.sum(axis=0) - vf[js]) / (e + tk - 1)
    assert np.max(np.abs(got - want[None])) <= 1e-14 * np.abs(want).max()


def test_key_order_and_head_independence(orc):
    tq, tk, heads, d = 6, 41, 3, 32
    q, k, v = _qkv(6, tq, tk, heads, d)
    base = orc.attention(q, _bits(k), _bits(v), 0.2)
    perm = torch.from_numpy(np.random.default_rng(0).permutation(tk))
    shuffled = orc.attention(q, _bits(k[perm]), _bits(v[perm]), 0.2)
    assert np.max(np.abs(shuffled - base)) <= 1e-13 * np.abs(base).max()
    # changing head 1's keys moves head 1's output only
    k2 = k.clone()
    k2[:, 1] = synth.normal(6, 7, (tk, d))
    other = orc.attention(q, _bits(k2), _bits(v), 0.2)
    assert np.array_equal(other[:, [0, 2]], base[:, [0, 2]])
    assert np.max(np.abs(other[:, 1] - base[:, 1])) > 1e-3


def test_query_row_selection(orc):
    q, k, v = _qkv(8, 9, 30, 2, 16)
    full = orc.attention(q, _bits(k), _bits(v), 0.3)
    rows = [7, 0, 4]
    assert np.array_equal(orc.attention(q, _bits(k), _bits(v), 0.3, rows=rows), full[rows])


def test_cache_window_attention_is_slot_order_free(orc):
    # the window's tokens form a set: the slot order changes the summation order only
    heads, d = 2, 32
    kv = orc.KVCacheModel(1, heads, d, 3, 40)
    for s, n in enumerate((40, 17, 33)):
        k, v = synth.kv_chunk(0, s, tokens=n)
        kv.append(0, s, k[:, :heads, :d].contiguous(), v[:, :heads, :d].contiguous())
    q = synth.normal(9, 0, (5, heads, d))
    a = kv.attention(0, [0, 1, 2], q, 0.125)
    b = kv.attention(0, [2, 0, 1], q, 0.125)
    assert np.max(np.abs(a - b)) <= 1e-13 * np.abs(a).max()
    # and it is the attention over the restored window
    k, v = kv.dequant(0, [0, 1, 2])
    assert np.array_equal(a, orc.attention(q, k, v, 0.125))
