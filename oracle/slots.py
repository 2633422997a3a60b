"""Per-step slot bookkeeping of the compact KV store (oracle simulator).

One decode step at position t, for one (sequence, layer, kv-head), in the
order read from the pages -- delayed eviction retires a flagged token once it
leaves the window ("NVIDIA veröffentlicht Qwen3-8B-DMS-8x ..." (mindverse),
section "Dynamic Memory Sparsification (DMS): Eine innovative Lösung"), and
the compact store reclaims the slot of a physically evicted token ("FastDMS:
vLLM BF16/FP8보다 빠른 6.4x KV cache 압축" (molayo1419.me), opening paragraphs):

1. retire: if t >= w, the ring entry at t mod w holds token t - w; if that
   token is flagged, its slot goes onto the head's free stack (LIFO) and the
   retained count drops by one;
2. allocate: pop the free stack if it is not empty, else take slot n_slots
   and grow n_slots by one;
3. write token t's K/V into that slot;
4. ring[t mod w] = (slot, flag of t); the retained count grows by one.

The simulator follows these steps literally (it keeps the free stack and
the slot -> position map); the closed forms they imply are checked by tests.
"""
from __future__ import annotations

import numpy as np

from .compaction import prefill_ring, prefill_slots


class HeadStore:
    """Logical state of one (sequence, layer, kv-head) of the compact store."""

    def __init__(self, prompt_evict: np.ndarray, w: int):
        self.w = int(w)
        slot = prefill_slots(prompt_evict, w)
        self.pos_of_slot = {s: j for j, s in slot.items()}
        self.n_slots = len(slot)
        self.n_retained = len(slot)
        self.ring = prefill_ring(prompt_evict, w)
        self.free: list[int] = []

    def append(self, t: int, evict_t: int) -> int:
        """Run decode step t; returns the slot that token t was written to."""
        w = self.w
        if t >= w:
            entry = self.ring[t % w]
            if entry is not None and entry[1]:
                s_old = entry[0]
                del self.pos_of_slot[s_old]
                self.free.append(s_old)
                self.n_retained -= 1
        if self.free:
            s = self.free.pop()
        else:
            s = self.n_slots
            self.n_slots += 1
        self.pos_of_slot[s] = t
        self.ring[t % w] = (s, int(evict_t))
        self.n_retained += 1
        return s

    def positions(self) -> np.ndarray:
        """Positions currently held, increasing."""
        return np.array(sorted(self.pos_of_slot.values()), dtype=np.int64)
