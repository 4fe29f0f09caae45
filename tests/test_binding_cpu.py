"""The Python binding on a host without a GPU: it marshals arguments only, so it must reject what
the library cannot take (host tensors, wrong dtype or shape) before any library call, and it
must fail loudly when the compiled library is missing -- there is no fallback path."""
import pytest
import torch

import bit_kv_cache_24_b200 as nv


def test_missing_library_raises(monkeypatch, tmp_path):
    monkeypatch.setattr(nv, "_lib", None)
    monkeypatch.setattr(nv, "LIB_PATH", str(tmp_path / "libnvfp4.so"))
    with pytest.raises(ImportError):
        nv.lib()
    # and so does a product object that needs it
    with pytest.raises(ImportError):
        nv.KVCache(1, 2, 128, 2, 16, "cpu")


def test_host_tensors_are_rejected():
    with pytest.raises(TypeError):
        nv.nvfp4_quantize(torch.zeros(4, 32, dtype=torch.bfloat16))          # host memory
    with pytest.raises(TypeError):
        nv.nvfp4_quantize(torch.zeros(4, 32, dtype=torch.float32))           # not BF16


def test_kv_attention_marshalling_errors():
    cache = nv.KVCache(1, 2, 128, 2, 16, "cpu")                               # storage only; never launched
    with pytest.raises(TypeError):
        nv.kv_attention(cache, 0, [0], torch.zeros(4, 2, 128, dtype=torch.bfloat16), 1.0)


def test_status_word_marshalling(monkeypatch):
    """The caller's status word is passed through; the release build adds none of its own; the
    checked build (here faked, no GPU needed for the release path) is what enables the binding's
    own words."""
    assert nv.checked_build() is False                     # the in-tree release build
    assert nv._status(None) is None
    t = torch.zeros(1, dtype=torch.int32)
    assert nv._status(t).value == t.data_ptr()
    assert nv.checked_status() == 0                        # nothing was ever handed out
    monkeypatch.setattr(nv, "_checked", True)
    assert nv._status(t).value == t.data_ptr()             # an explicit word always wins
