"""Sequence-parallel exchange of the NVFP4 KV cache (head-split all-to-all of the quantized bytes).

LongLive-2.0 runs sequence-parallel inference where NVFP4 tensor cores are missing and notes that
the quantized KV cache lowers the inter-GPU communication of that SP (arXiv abstract, fugumt.com
mirror).  In a head-split (all-to-all) SP layout every rank holds all heads of its token shard
before attention and all tokens of its head group during attention.  This module moves the K/V
of a chunk between the two layouts in NVFP4: each rank quantizes its token shard once
(kv_quant_append: one g per tensor and shard), and the all-to-all carries, for every destination
rank, that rank's head group of the E2M1 codes and E4M3 block scales (16-blocks never straddle
heads: head_dim % 16 == 0) plus the sources' g -- 0.5625 B per element and 8 B per shard instead
of 2 B per element in BF16 (3.56x fewer bytes).  The receiving rank restores its head group of
all shards with kv_dequant, one slot per source rank, each with that source's g; the bytes are
the source's own, so the restored values equal the source's dequantization bit for bit.

Transport: torch.distributed (NCCL over NVLink between GPUs; gloo for the host tests); no
arithmetic happens in this module.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def _split_heads(t: torch.Tensor, P: int) -> torch.Tensor:
    """[tokens, heads * w] -> [P, tokens, heads/P * w] (head group p of every token row)."""
    tokens, row = t.shape
    return t.reshape(tokens, P, row // P).transpose(0, 1).contiguous()


def exchange(codes_k, sf_k, g_k, codes_v, sf_v, g_v, heads, head_dim, group=None):
    """All-to-all of one quantized K/V shard.

    Inputs on every rank (its token shard of `tokens` rows, the same count on every rank):
    codes [tokens, heads*head_dim/2] u8, sf [tokens, heads*head_dim/16] u8 (linear layout, as
    in the KV cache), g [1] f32, for K and for V.  Returns, for this rank's head group
    (heads/P heads), codes [P, tokens, heads/P*head_dim/2], sf [P, tokens, heads/P*head_dim/16]
    and g [P] for K and V, source ranks in order."""
    P = dist.get_world_size(group)
    if heads % P or head_dim % 16:
        raise ValueError("heads must split evenly over the ranks and head_dim % 16 == 0")
    out = {}
    for name, codes, sf in (("k", codes_k, sf_k), ("v", codes_v, sf_v)):
        for part, t in (("codes", codes), ("sf", sf)):
            send = _split_heads(t, P)
            recv = torch.empty_like(send)
            dist.all_to_all_single(recv, send, group=group)
            out[f"{part}_{name}"] = recv
    g_local = torch.cat([g_k.reshape(1), g_v.reshape(1)]).to(torch.float32)
    gathered = [torch.empty_like(g_local) for _ in range(P)]
    dist.all_gather(gathered, g_local, group=group)
    g = torch.stack(gathered)
    out["g_k"], out["g_v"] = g[:, 0].contiguous(), g[:, 1].contiguous()
    return out


def restore(recv, head_dim):
    """BF16 K, V [P*tokens, heads/P, head_dim] of this rank's head group, all shards in rank order,
    from exchange()'s output (on the GPU): a P-slot KV cache, restored by kv_dequant."""
    import bit_kv_cache_24_b200 as nv
    P, tokens, row_bytes = recv["codes_k"].shape
    local_heads = 2 * row_bytes // head_dim
    cache = nv.KVCache(1, local_heads, head_dim, P, tokens, recv["codes_k"].device)
    cache.codes_k.view(P, tokens, -1).copy_(recv["codes_k"])
    cache.codes_v.view(P, tokens, -1).copy_(recv["codes_v"])
    cache.sf_k.view(P, tokens, -1).copy_(recv["sf_k"])
    cache.sf_v.view(P, tokens, -1).copy_(recv["sf_v"])
    cache.g_k.copy_(recv["g_k"])
    cache.g_v.copy_(recv["g_v"])
    for s in range(P):
        cache.len[s] = tokens
    return nv.kv_dequant(cache, 0, list(range(P)))


def bytes_per_rank(tokens, heads, head_dim, world):
    """Bytes one rank sends for K and V: NVFP4 (codes + scales + g) and BF16, for comparison."""
    elems = tokens * heads * head_dim * (world - 1) // world
    return {"nvfp4": 2 * (elems // 2 + elems // 16) + 8 * (world - 1), "bf16": 2 * 2 * elems}
