"""Multi-shot attention-sink policy over the NVFP4 KV cache (host-side slot bookkeeping).

LongLive-2.0 keeps a fixed global-level sink that preserves the video's identity, and a shot-level
sink that is re-bound at every shot boundary to hold the scene's appearance (the d9249.github.io
review of the paper, section "핵심 아이디어 / 구조 / 동작 방식"), next to the recent context; its
repository update writes the quantized cache in place (yourai.pro report).  The pages give no
sizes; this module takes the plain reading with parameters:

  - global sink: the first `global_sink` chunks of the video, never replaced;
  - shot sink:   the first `shot_sink` chunks of the current shot (chunks that are not global-sink
                 chunks), replaced in place when a new shot starts;
  - window:      the `window` most recent other chunks, the oldest replaced in place.

Every chunk is quantized once, by kv_quant_append, into the slot this policy assigns; nothing is
re-quantized or moved.  The attention context of a chunk step is the global sink, then the shot
sink, then the window from oldest to newest, restored by one kv_dequant call over that slot list.
With the defaults (1 + 1 + 10 slots of 4680 tokens) the context is the 56160-token window of
the KV-cache workload.

The policy is pure bookkeeping: all arithmetic runs in the library's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass, field



@dataclass
class SinkPolicy:
    """Slot assignment of the multi-shot sink cache (no device state)."""
    global_sink: int = 1
    shot_sink: int = 1
    window: int = 10
    chunks: int = 0                           # chunks appended so far
    shot_start: int = 0                       # first chunk of the current shot
    slot_chunk: dict = field(default_factory=dict)   # slot -> chunk id held
    ring_next: int = 0                        # next window slot to fill (rolling)

    @property
    def slots(self) -> int:
        return self.global_sink + self.shot_sink + self.window

    def next_slot(self, new_shot: bool = False) -> int:
        """Assign the slot of the next chunk (and advance the state).  Chunk 0 starts shot 0."""
        c = self.chunks
        if c == 0 or new_shot:
            self.shot_start = c
            # the previous shot's sink chunks leave the context
            for s in range(self.global_sink, self.global_sink + self.shot_sink):
                self.slot_chunk.pop(s, None)
        if c < self.global_sink:
            slot = c
        elif c - max(self.shot_start, self.global_sink) < self.shot_sink and c >= self.shot_start:
            slot = self.global_sink + (c - max(self.shot_start, self.global_sink))
        else:
            slot = self.global_sink + self.shot_sink + self.ring_next
            self.ring_next = (self.ring_next + 1) % self.window
        self.slot_chunk[slot] = c
        self.chunks = c + 1
        return slot

    def context(self) -> list[int]:
        """Slots of the attention context: global sink, shot sink, window oldest -> newest."""
        sinks = [s for s in range(self.global_sink + self.shot_sink) if s in self.slot_chunk]
        ring = [s for s in range(self.global_sink + self.shot_sink, self.slots) if s in self.slot_chunk]
        ring.sort(key=lambda s: self.slot_chunk[s])
        return sinks + ring

    def context_chunks(self) -> list[int]:
        return [self.slot_chunk[s] for s in self.context()]


class SinkKVCache:
    """An NVFP4 KV cache (all layers) under the multi-shot sink policy.

    Per chunk: begin_chunk(new_shot) picks the slot, append(layer, k, v) quantizes that layer's K
    and V into it (kv_quant_append, in place), restore(layer) dequantizes the layer's context
    (kv_dequant over the context's slots, in context order)."""

    def __init__(self, layers, heads, head_dim, slot_tokens, device, global_sink=1, shot_sink=1, window=10):
        import bit_kv_cache_24_b200 as nv
        self.nv = nv
        self.policy = SinkPolicy(global_sink, shot_sink, window)
        self.cache = nv.KVCache(layers, heads, head_dim, self.policy.slots, slot_tokens, device)
        self.slot = None

    def begin_chunk(self, new_shot: bool = False) -> int:
        self.slot = self.policy.next_slot(new_shot)
        return self.slot

    def append(self, layer, k, v, status=None, stream=None):
        if self.slot is None:
            raise RuntimeError("begin_chunk() first")
        self.nv.kv_quant_append(self.cache, layer, self.slot, k, v, status=status, stream=stream)

    def restore(self, layer, k_out=None, v_out=None, status=None, stream=None):
        return self.nv.kv_dequant(self.cache, layer, self.policy.context(), k_out=k_out, v_out=v_out,
                                  status=status, stream=stream)
