"""GPU side of the NVFP4 KV sequence-parallel exchange: shards quantized by kv_quant_append, the
head-group pieces a destination rank receives (cut here by plain slicing, as the all-to-all
delivers them), and sp_exchange.restore through kv_dequant -- bit for bit against the oracle's
dequantization of each source shard's head group.  The exchange itself runs over NCCL with one
rank (the multi-rank transport is tested with gloo in tests/test_sp_exchange.py)."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist

import bit_kv_cache_24_b200 as nv
from bit_kv_cache_24_b200 import synth
from bit_kv_cache_24_b200.sp_exchange import exchange, restore

pytestmark = pytest.mark.gpu

TOKENS, HEADS, HEAD_DIM = 96, 8, 64


def _quantized_shards(P):
    shards = []
    for src in range(P):
        k = synth.ragged(700 + src, TOKENS, HEADS * HEAD_DIM, "outliers")
        v = synth.ragged(800 + src, TOKENS, HEADS * HEAD_DIM, "lognormal")
        c = nv.KVCache(1, HEADS, HEAD_DIM, 1, TOKENS, "cuda")
        nv.kv_quant_append(c, 0, 0, k.cuda(), v.cuda())
        shards.append((k, v, c))
    return shards


@pytest.mark.parametrize("P", [2, 4])
def test_restore_of_received_head_groups(orc, P):
    shards = _quantized_shards(P)
    Hl = HEADS // P
    cw, sw = Hl * HEAD_DIM // 2, Hl * HEAD_DIM // 16
    for r in range(P):                                     # each destination rank
        recv = {}
        for name in ("k", "v"):
            recv[f"codes_{name}"] = torch.stack([getattr(c, f"codes_{name}").view(TOKENS, -1)[:, r * cw:(r + 1) * cw]
                                                 for _, _, c in shards]).contiguous()
            recv[f"sf_{name}"] = torch.stack([getattr(c, f"sf_{name}").view(TOKENS, -1)[:, r * sw:(r + 1) * sw]
                                              for _, _, c in shards]).contiguous()
            recv[f"g_{name}"] = torch.cat([getattr(c, f"g_{name}")[:1] for _, _, c in shards])
        K, V = restore(recv, HEAD_DIM)
        torch.cuda.synchronize()
        for got, w in ((K, 0), (V, 1)):
            want = np.concatenate([orc.dequant(orc.quantize(sh[w])[1])[:, r * Hl * HEAD_DIM:(r + 1) * Hl * HEAD_DIM]
                                   for sh in shards])
            g = got.reshape(P * TOKENS, Hl * HEAD_DIM).view(torch.int16).cpu().numpy().view(np.uint16)
            assert np.array_equal(g, want), (P, r, w)


def test_nccl_exchange_single_rank(orc):
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29561")
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        (k, v, c), = _quantized_shards(1)
        recv = exchange(c.codes_k.view(TOKENS, -1), c.sf_k.view(TOKENS, -1), c.g_k[:1],
                        c.codes_v.view(TOKENS, -1), c.sf_v.view(TOKENS, -1), c.g_v[:1], HEADS, HEAD_DIM)
        K, V = restore(recv, HEAD_DIM)
        torch.cuda.synchronize()
        for got, x in ((K, k), (V, v)):
            want = orc.dequant(orc.quantize(x)[1])
            g = got.reshape(TOKENS, HEADS * HEAD_DIM).view(torch.int16).cpu().numpy().view(np.uint16)
            assert np.array_equal(g, want)
    finally:
        dist.destroy_process_group()
