"""Save and load NVFP4 tensors and KV caches as raw bytes (host-side, no arithmetic).

Weights are quantized once, offline, and shipped in NVFP4 (LongLive-2.0 distributes NVFP4
checkpoints next to the BF16 ones: yourai.pro report). This module stores a QTensor (codes,
scales and g exactly as the kernels lay them out) or a whole KVCache (its four arrays, both g
arrays and the per-slot token counts), so they can be reloaded onto any device without
re-quantizing.

File layout: the 8-byte magic, a little-endian uint32 header length, a UTF-8 JSON header (kind,
geometry, byte count of each array), then the arrays' raw bytes in header order. On load, the
geometry is checked against the library's own size functions, so a file can never be read into
a mismatched layout.
"""
from __future__ import annotations

import json
import struct

import torch

MAGIC = b"NVFP4IO1"


def _write(path, header: dict, arrays: list[torch.Tensor]):
    header = dict(header, arrays=[int(a.numel() * a.element_size()) for a in arrays])
    h = json.dumps(header, sort_keys=True).encode()
    with open(path, "wb") as f:
        f.write(MAGIC)
        f.write(struct.pack("<I", len(h)))
        f.write(h)
        for a in arrays:
            f.write(a.detach().contiguous().cpu().view(torch.uint8).numpy().tobytes())


def _read(path):
    with open(path, "rb") as f:
        if f.read(len(MAGIC)) != MAGIC:
            raise ValueError(f"{path}: not an NVFP4 file")
        (n,) = struct.unpack("<I", f.read(4))
        header = json.loads(f.read(n).decode())
        blobs = []
        for nbytes in header["arrays"]:
            b = f.read(nbytes)
            if len(b) != nbytes:
                raise ValueError(f"{path}: truncated")
            blobs.append(b)
        if f.read(1):
            raise ValueError(f"{path}: trailing bytes")
    return header, blobs


def _fill(dst: torch.Tensor, blob: bytes, what: str):
    if dst.numel() * dst.element_size() != len(blob):
        raise ValueError(f"{what}: {len(blob)} bytes in the file, {dst.numel() * dst.element_size()} expected")
    src = torch.frombuffer(bytearray(blob), dtype=torch.uint8)
    dst.view(torch.uint8).view(-1).copy_(src)


def save_qtensor(q, path):
    """Write a QTensor (codes, scales, g) to `path`."""
    _write(path, {"kind": "qtensor", "rows": q.rows, "cols": q.cols, "sf_layout": q.sf_layout},
           [q.codes, q.sf, q.g])


def load_qtensor(path, device="cuda"):
    """Read a QTensor written by save_qtensor onto `device`."""
    import bit_kv_cache_24_b200 as nv
    h, blobs = _read(path)
    if h.get("kind") != "qtensor" or len(blobs) != 3:
        raise ValueError(f"{path}: not a saved QTensor")
    q = nv.QTensor(h["rows"], h["cols"], h["sf_layout"], device)
    for dst, blob, what in zip((q.codes, q.sf, q.g), blobs, ("codes", "scales", "g")):
        _fill(dst, blob, what)
    return q


def save_kv_cache(cache, path):
    """Write a KVCache (codes, scales and g of K and V, and the per-slot token counts)."""
    lens = torch.tensor(list(cache.len), dtype=torch.int32)
    _write(path, {"kind": "kv_cache", "layers": cache.layers, "heads": cache.heads, "head_dim": cache.head_dim,
                  "slots": cache.slots, "slot_tokens": cache.slot_tokens},
           [cache.codes_k, cache.codes_v, cache.sf_k, cache.sf_v, cache.g_k, cache.g_v, lens])


def load_kv_cache(path, device="cuda"):
    """Read a KVCache written by save_kv_cache onto `device`."""
    import bit_kv_cache_24_b200 as nv
    h, blobs = _read(path)
    if h.get("kind") != "kv_cache" or len(blobs) != 7:
        raise ValueError(f"{path}: not a saved KV cache")
    c = nv.KVCache(h["layers"], h["heads"], h["head_dim"], h["slots"], h["slot_tokens"], device)
    for dst, blob, what in zip((c.codes_k, c.codes_v, c.sf_k, c.sf_v, c.g_k, c.g_v), blobs[:6],
                               ("codes_k", "codes_v", "sf_k", "sf_v", "g_k", "g_v")):
        _fill(dst, blob, what)
    lens = torch.empty(c.layers * c.slots, dtype=torch.int32)
    _fill(lens, blobs[6], "len")
    if int(lens.min()) < 0 or int(lens.max()) > c.slot_tokens:
        raise ValueError(f"{path}: slot token counts out of range")
    for i, n in enumerate(lens.tolist()):
        c.len[i] = n
    return c
