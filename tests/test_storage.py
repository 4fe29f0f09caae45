"""Save/load of NVFP4 tensors and KV caches (host-side; the arrays live in host memory here, the
same code moves device arrays through the host)."""
import struct

import numpy as np
import pytest
import torch

import bit_kv_cache_24_b200 as nv
from bit_kv_cache_24_b200 import storage, synth


def _random_bytes(t, seed):
    g = torch.Generator().manual_seed(seed)
    t.view(torch.uint8).view(-1).copy_(torch.randint(0, 256, (t.numel() * t.element_size(),), generator=g,
                                                     dtype=torch.uint8))


def test_qtensor_round_trip_is_exact(orc, tmp_path):
    # an oracle quantization of a workload-shaped tensor, stored in a host QTensor
    x = synth.ragged(5, 37, 96, "outliers")
    _, ref = orc.quantize(x)
    q = nv.QTensor(37, 96, nv.SF_LINEAR, "cpu")
    q.codes.copy_(torch.from_numpy(ref.codes.reshape(q.codes.shape)))
    q.sf.copy_(torch.from_numpy(ref.sf.reshape(-1)))
    q.g.fill_(float(ref.g))
    storage.save_qtensor(q, tmp_path / "w.nvfp4")
    r = storage.load_qtensor(tmp_path / "w.nvfp4", "cpu")
    assert (r.rows, r.cols, r.sf_layout) == (37, 96, nv.SF_LINEAR)
    assert torch.equal(r.codes, q.codes) and torch.equal(r.sf, q.sf)
    assert r.g.view(torch.int32).item() == q.g.view(torch.int32).item()
    assert np.array_equal(r.codes.numpy().reshape(-1), ref.codes.reshape(-1))


def test_mma_layout_qtensor_round_trip(tmp_path):
    q = nv.QTensor(300, 512, nv.SF_MMA, "cpu")
    for i, t in enumerate((q.codes, q.sf, q.g)):
        _random_bytes(t, i)
    storage.save_qtensor(q, tmp_path / "a.nvfp4")
    r = storage.load_qtensor(tmp_path / "a.nvfp4", "cpu")
    assert r.sf.numel() == nv.lib().nvfp4_sf_bytes(300, 512, nv.SF_MMA)
    assert all(torch.equal(a.view(torch.uint8), b.view(torch.uint8)) for a, b in
               ((r.codes, q.codes), (r.sf, q.sf), (r.g, q.g)))


def test_kv_cache_round_trip_is_exact(tmp_path):
    c = nv.KVCache(2, 3, 32, 4, 10, "cpu")
    for i, t in enumerate((c.codes_k, c.codes_v, c.sf_k, c.sf_v, c.g_k, c.g_v)):
        _random_bytes(t, 10 + i)
    for i, n in enumerate((10, 0, 7, 3, 1, 10, 0, 2)):
        c.len[i] = n
    storage.save_kv_cache(c, tmp_path / "kv.nvfp4")
    r = storage.load_kv_cache(tmp_path / "kv.nvfp4", "cpu")
    assert (r.layers, r.heads, r.head_dim, r.slots, r.slot_tokens) == (2, 3, 32, 4, 10)
    assert list(r.len) == list(c.len)
    for a, b in ((r.codes_k, c.codes_k), (r.codes_v, c.codes_v), (r.sf_k, c.sf_k), (r.sf_v, c.sf_v),
                 (r.g_k, c.g_k), (r.g_v, c.g_v)):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))


def test_bad_files_are_rejected(tmp_path):
    q = nv.QTensor(16, 32, nv.SF_LINEAR, "cpu")
    for t in (q.codes, q.sf, q.g):
        t.zero_()
    p = tmp_path / "q.nvfp4"
    storage.save_qtensor(q, p)
    raw = p.read_bytes()
    (tmp_path / "magic").write_bytes(b"XXXXXXXX" + raw[8:])
    (tmp_path / "short").write_bytes(raw[:-1])
    (tmp_path / "long").write_bytes(raw + b"\0")
    for name in ("magic", "short", "long"):
        with pytest.raises(ValueError):
            storage.load_qtensor(tmp_path / name, "cpu")
    with pytest.raises(ValueError):
        storage.load_kv_cache(p, "cpu")                            # a QTensor is not a KV cache
    # a header whose geometry disagrees with the array sizes
    n = struct.unpack("<I", raw[8:12])[0]
    h = raw[12:12 + n].replace(b'"rows": 16', b'"rows": 17')
    (tmp_path / "geom").write_bytes(raw[:8] + struct.pack("<I", len(h)) + h + raw[12 + n:])
    with pytest.raises(ValueError):
        storage.load_qtensor(tmp_path / "geom", "cpu")
