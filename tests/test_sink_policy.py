"""Host-side tests of the multi-shot sink policy (bit_kv_cache_24_b200/sink_cache.py) against a
brute-force definition computed from the chunk history alone:

  global sink = the first G chunks of the video;
  shot sink   = the first S chunks of the current shot that are not global-sink chunks;
  window      = the W most recent chunks that were neither (a chunk that was its own shot's sink
                chunk never enters the window);
  context     = global sink, shot sink, window (oldest -> newest).
Also: a slot, once assigned, is only ever rewritten by a later chunk (in-place updates), global
sink slots never, and the context never exceeds G + S + W slots."""
import random

import pytest

from bit_kv_cache_24_b200.sink_cache import SinkPolicy


def brute_context(n, starts, G, S, W):
    def shot_of(c):
        return max(b for b in starts if b <= c)

    def is_shot_sink(c):
        first = max(shot_of(c), G)
        return c >= G and first <= c < first + S

    glob = list(range(min(G, n)))
    cur = shot_of(n - 1)
    first = max(cur, G)
    shot = [c for c in range(first, min(n, first + S))]
    ring = [c for c in range(n) if c >= G and not is_shot_sink(c)]
    return glob + shot + ring[-W:] if W > 0 else glob + shot


@pytest.mark.parametrize("G,S,W", [(1, 1, 10), (2, 1, 3), (1, 2, 4), (0, 1, 5), (1, 0, 6), (3, 2, 1)])
@pytest.mark.parametrize("seed", range(6))
def test_policy_matches_brute_force(G, S, W, seed):
    rng = random.Random(seed * 100 + G * 10 + S)
    pol = SinkPolicy(G, S, W)
    starts = {0}
    slot_history = {}
    for c in range(60):
        new_shot = c > 0 and rng.random() < 0.15
        if new_shot:
            starts.add(c)
        slot = pol.next_slot(new_shot)
        assert 0 <= slot < G + S + W
        if slot < G:
            assert slot not in slot_history, "a global sink slot was rewritten"
        slot_history[slot] = c
        want = brute_context(c + 1, starts, G, S, W)
        assert pol.context_chunks() == want, (c, sorted(starts), pol.context_chunks(), want)
        assert len(pol.context()) <= G + S + W
        for s in pol.context():
            assert slot_history[s] == pol.slot_chunk[s]


def test_default_geometry_is_the_kv_workload():
    pol = SinkPolicy()
    assert pol.slots == 12                                 # 12 x 4680 tokens = 56160
    for c in range(40):
        pol.next_slot(new_shot=(c in (15, 28)))
    ctx = pol.context_chunks()
    assert ctx[0] == 0 and ctx[1] == 28 and ctx[2:] == list(range(30, 40))   # shots start at 0, 15, 28
