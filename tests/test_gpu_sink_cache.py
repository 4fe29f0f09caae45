"""GPU test of the multi-shot sink cache: chunks appended under the policy (with shot boundaries
and chunks of different lengths) and the restored context, bit for bit against the oracle's
quantize + dequantize of the chunks the brute-force definition puts in the context
(tests/test_sink_policy.py), in context order, for every layer after every chunk."""
import numpy as np
import pytest
import torch

from bit_kv_cache_24_b200 import synth
from bit_kv_cache_24_b200.sink_cache import SinkKVCache
from tests.test_sink_policy import brute_context

pytestmark = pytest.mark.gpu


def test_sink_cache_restore_matches_oracle(orc):
    layers, heads, head_dim, slot_tokens = 2, 2, 16, 64
    G, S, W = 1, 1, 3
    row = heads * head_dim
    cache = SinkKVCache(layers, heads, head_dim, slot_tokens, torch.device("cuda"), G, S, W)
    starts, chunks = {0}, []
    for c in range(12):
        new_shot = c in (5, 9)
        if new_shot:
            starts.add(c)
        ntok = 64 if c % 3 else 40
        kv = [(synth.ragged(1000 + 10 * c + 2 * l, ntok, row, "outliers"),
               synth.ragged(1001 + 10 * c + 2 * l, ntok, row, "wide")) for l in range(layers)]
        chunks.append(kv)
        cache.begin_chunk(new_shot)
        for l, (k, v) in enumerate(kv):
            cache.append(l, k.cuda(), v.cuda())
        want_chunks = brute_context(c + 1, starts, G, S, W)
        assert cache.policy.context_chunks() == want_chunks
        for l in range(layers):
            K, V = cache.restore(l)
            torch.cuda.synchronize()
            for got, which in ((K, 0), (V, 1)):
                want = []
                for cc in want_chunks:
                    st, q = orc.quantize(chunks[cc][l][which])
                    assert st == 0
                    want.append(orc.dequant(q))
                want = np.concatenate(want, axis=0)
                g = got.reshape(got.shape[0], row).view(torch.int16).cpu().numpy().view(np.uint16)
                assert g.shape == want.shape
                assert np.array_equal(g, want), (c, l, which)
