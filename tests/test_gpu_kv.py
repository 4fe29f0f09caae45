"""GPU parity of kv_quant_append / kv_dequant against the oracle's KV-cache model: in-place
append of a chunk's K and V (own per-tensor scale per slot), bit-exact codes/scales/g, and a
bit-exact BF16 restore of any window of slots."""
import numpy as np
import pytest
import torch

import bit_kv_cache_24_b200 as nv
from bit_kv_cache_24_b200 import synth
from tests.parity_util import gpu_bytes

pytestmark = pytest.mark.gpu


def _slot_bytes(cache, layer, slot):
    row = cache.heads * cache.head_dim
    t0 = (layer * cache.slots + slot) * cache.slot_tokens
    n = cache.slot_len(layer, slot)
    ck = gpu_bytes(cache.codes_k[t0 * row // 2:(t0 + n) * row // 2]).reshape(n, row // 2)
    sk = gpu_bytes(cache.sf_k[t0 * row // 16:(t0 + n) * row // 16]).reshape(n, row // 16)
    cv = gpu_bytes(cache.codes_v[t0 * row // 2:(t0 + n) * row // 2]).reshape(n, row // 2)
    sv = gpu_bytes(cache.sf_v[t0 * row // 16:(t0 + n) * row // 16]).reshape(n, row // 16)
    i = layer * cache.slots + slot
    return ck, sk, float(cache.g_k[i].item()), cv, sv, float(cache.g_v[i].item())


def test_small_cache_append_and_window(orc):
    L, H, D, S, T = 2, 4, 32, 3, 40
    cache = nv.KVCache(L, H, D, S, T)
    model = orc.KVCacheModel(L, H, D, S, T)
    lens = {0: 40, 1: 17, 2: 1}
    for s, n in lens.items():
        k, v = synth.kv_chunk(3, s, tokens=n)
        k, v = k[:, :H, :D].contiguous(), v[:, :H, :D].contiguous()
        nv.kv_quant_append(cache, 1, s, k.cuda(), v.cuda())
        assert model.append(1, s, k, v) == 0
    torch.cuda.synchronize()
    for s in lens:
        ck, sk, gk, cv, sv, gv = _slot_bytes(cache, 1, s)
        qk, qv = model.store[(1, s)]
        assert np.array_equal(ck, qk.codes) and np.array_equal(sk, qk.sf) and gk == float(qk.g)
        assert np.array_equal(cv, qv.codes) and np.array_equal(sv, qv.sf) and gv == float(qv.g)
    for window in ([2, 0, 1], [1], [0, 2]):
        K, V = nv.kv_dequant(cache, 1, window)
        Kw, Vw = model.dequant(1, window)
        assert np.array_equal(K.view(torch.int16).cpu().numpy().view(np.uint16), Kw)
        assert np.array_equal(V.view(torch.int16).cpu().numpy().view(np.uint16), Vw)


def test_append_from_fused_qkv_rows_is_in_place(orc):
    """K and V are strided slices of a QKV GEMM output [ntok, 3*H*D]; appending one slot
    leaves every other slot's bytes untouched."""
    H, D, T = 24, 128, 64
    cache = nv.KVCache(1, H, D, 4, T)
    qkv = synth.ragged(9, T, 3 * H * D, "outliers").cuda()
    row = H * D
    k, v = qkv[:, row:2 * row], qkv[:, 2 * row:]
    nv.kv_quant_append(cache, 0, 0, k, v)
    nv.kv_quant_append(cache, 0, 2, v, k)
    torch.cuda.synchronize()
    before = [t.clone() for t in (cache.codes_k, cache.sf_k, cache.codes_v, cache.sf_v, cache.g_k, cache.g_v)]
    nv.kv_quant_append(cache, 0, 1, k[:50], v[:50])
    torch.cuda.synchronize()
    t1 = 1 * T
    for b, a in zip(before[:4], (cache.codes_k, cache.sf_k, cache.codes_v, cache.sf_v)):
        per_tok = b.numel() // (4 * T)
        assert torch.equal(b[:t1 * per_tok], a[:t1 * per_tok])
        assert torch.equal(b[2 * T * per_tok:], a[2 * T * per_tok:])
    _, qk = orc.quantize(k[:50].contiguous().cpu())
    ck, sk, gk, *_ = _slot_bytes(cache, 0, 1)
    assert np.array_equal(ck, qk.codes) and np.array_equal(sk, qk.sf) and gk == float(qk.g)
    K, V = nv.kv_dequant(cache, 0, [0, 1, 2])
    assert K.shape == (64 + 50 + 64, H, D)


def test_full_cache_one_layer(orc):
    """The KV workload for one layer: 12 appends of 4680 tokens (24 heads x 128, 4 outlier
    channels x15), then the full 56160-token window restored to BF16.  Slots 0, 5 and 11 are
    compared byte for byte with the oracle's quantizer; the whole restore is compared with the
    oracle's dequantizer applied to the cache bytes."""
    H, D, S, T = synth.HEADS, synth.HEAD_DIM, synth.KV_APPENDS, synth.CHUNK_TOKENS
    cache = nv.KVCache(1, H, D, S, T)
    chunks = {}
    for s in range(S):
        k, v = synth.kv_chunk(7, s)
        if s in (0, 5, 11):
            chunks[s] = (k, v)
        nv.kv_quant_append(cache, 0, s, k.cuda(), v.cuda())
    K, V = nv.kv_dequant(cache, 0, list(range(S)))
    torch.cuda.synchronize()
    row = H * D
    for s, (k, v) in chunks.items():
        ck, sk, gk, cv, sv, gv = _slot_bytes(cache, 0, s)
        _, qk = orc.quantize(k.reshape(T, row))
        _, qv = orc.quantize(v.reshape(T, row))
        assert np.array_equal(ck, qk.codes) and np.array_equal(sk, qk.sf) and gk == float(qk.g)
        assert np.array_equal(cv, qv.codes) and np.array_equal(sv, qv.sf) and gv == float(qv.g)
    Kh = K.view(torch.int16).cpu().numpy().view(np.uint16).reshape(S, T, row)
    Vh = V.view(torch.int16).cpu().numpy().view(np.uint16).reshape(S, T, row)
    for s in range(S):
        ck, sk, gk, cv, sv, gv = _slot_bytes(cache, 0, s)
        qk = orc.Quantized(ck, sk, np.float32(gk), T, row)
        qv = orc.Quantized(cv, sv, np.float32(gv), T, row)
        assert np.array_equal(Kh[s], orc.dequant(qk)), s
        assert np.array_equal(Vh[s], orc.dequant(qv)), s


def test_full_cache_all_layers(orc):
    """The whole KV workload geometry: 30 layers x 12 slots of 4680 tokens (24 heads x 128, ~5.8 GB
    of NVFP4 cache; offsets of the last layers pass 2^31 bytes).  Every slot of every layer is
    appended; layers 0, 13 and 29 hold their own chunks (the others reuse a few), their slots 0
    and 11 are compared byte for byte with the oracle's quantizer, and layer 29's full window
    restore with the oracle's dequantizer of the cache bytes."""
    H, D, S, T, L = synth.HEADS, synth.HEAD_DIM, synth.KV_APPENDS, synth.CHUNK_TOKENS, 30
    row = H * D
    cache = nv.KVCache(L, H, D, S, T)
    checked = (0, 13, 29)
    pool = [tuple(t.cuda() for t in synth.kv_chunk(3, s)) for s in range(3)]
    kept = {}
    for layer in range(L):
        for s in range(S):
            if layer in checked:
                k, v = synth.kv_chunk(layer, s)
                if s in (0, S - 1):
                    kept[(layer, s)] = (k, v)
                nv.kv_quant_append(cache, layer, s, k.cuda(), v.cuda())
            else:
                k, v = pool[(layer + s) % 3]
                nv.kv_quant_append(cache, layer, s, k, v)
    K, V = nv.kv_dequant(cache, L - 1, list(range(S)))
    torch.cuda.synchronize()
    for (layer, s), (k, v) in kept.items():
        ck, sk, gk, cv, sv, gv = _slot_bytes(cache, layer, s)
        _, qk = orc.quantize(k.reshape(T, row))
        _, qv = orc.quantize(v.reshape(T, row))
        assert np.array_equal(ck, qk.codes) and np.array_equal(sk, qk.sf) and gk == float(qk.g), (layer, s)
        assert np.array_equal(cv, qv.codes) and np.array_equal(sv, qv.sf) and gv == float(qv.g), (layer, s)
    Kh = K.view(torch.int16).cpu().numpy().view(np.uint16).reshape(S, T, row)
    Vh = V.view(torch.int16).cpu().numpy().view(np.uint16).reshape(S, T, row)
    for s in range(S):
        ck, sk, gk, cv, sv, gv = _slot_bytes(cache, L - 1, s)
        assert np.array_equal(Kh[s], orc.dequant(orc.Quantized(ck, sk, np.float32(gk), T, row))), s
        assert np.array_equal(Vh[s], orc.dequant(orc.Quantized(cv, sv, np.float32(gv), T, row))), s
