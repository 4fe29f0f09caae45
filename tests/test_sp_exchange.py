"""Sequence-parallel exchange of the NVFP4 KV cache (bit_kv_cache_24_b200/sp_exchange.py), on CPU
with two gloo ranks: every rank quantizes its token shard with the oracle, the all-to-all moves
the quantized bytes, and each rank must receive, for its head group, exactly the source shards'
bytes and scales -- so that dequantizing a received piece equals the source's dequantization of
those heads, bit for bit.  (The GPU restore is in tests/test_gpu_sp_exchange.py.)"""
import os

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_kv_cache_24_b200 import synth
from bit_kv_cache_24_b200.sp_exchange import bytes_per_rank, exchange

TOKENS, HEADS, HEAD_DIM = 48, 4, 32


def _shard(src, which):
    return synth.ragged(500 + 10 * src + which, TOKENS, HEADS * HEAD_DIM, "outliers" if which == 0 else "wide")


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle.oracle as orc
    orc.build()
    q = [orc.quantize(_shard(rank, w))[1] for w in (0, 1)]
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))
    recv = exchange(t(q[0].codes), t(q[0].sf), torch.tensor([q[0].g]), t(q[1].codes), t(q[1].sf),
                    torch.tensor([q[1].g]), HEADS, HEAD_DIM)
    P, Hl = world, HEADS // world
    cw, sw = Hl * HEAD_DIM // 2, Hl * HEAD_DIM // 16           # bytes of a head group per row
    ok = True
    for src in range(P):
        for w, name in ((0, "k"), (1, "v")):
            _, qs = orc.quantize(_shard(src, w))               # the source's own quantization
            ok &= np.array_equal(recv[f"codes_{name}"][src].numpy(), qs.codes[:, rank * cw:(rank + 1) * cw])
            ok &= np.array_equal(recv[f"sf_{name}"][src].numpy(), qs.sf[:, rank * sw:(rank + 1) * sw])
            ok &= np.float32(recv[f"g_{name}"][src].item()) == np.float32(qs.g)
            piece = orc.Quantized(recv[f"codes_{name}"][src].numpy(), recv[f"sf_{name}"][src].numpy(),
                                  recv[f"g_{name}"][src].item(), TOKENS, Hl * HEAD_DIM)
            full = orc.dequant(qs)[:, rank * Hl * HEAD_DIM:(rank + 1) * Hl * HEAD_DIM]
            ok &= np.array_equal(orc.dequant(piece), full)
    out[rank] = bool(ok)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_exchange_moves_each_head_group():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, 29531, out), nprocs=world, join=True)
    assert out[0] and out[1]


def test_bytes_moved():
    b = bytes_per_rank(4680, 24, 128, 8)                       # one KV chunk, 8-way SP
    assert b["bf16"] / b["nvfp4"] > 3.5
