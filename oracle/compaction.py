"""Reference prefill compaction into a compact per-head KV store (oracle).

FastDMS keeps a compact KV store that reclaims physically evicted slots
("FastDMS: vLLM BF16/FP8보다 빠른 6.4x KV cache 압축" (molayo1419.me), opening
paragraphs), with per-layer, per-head variable token counts (same page,
table "What's the catch?", row "PagedAttention / KV memory pool").

After a prompt of P tokens the last prompt query sits at t = P - 1 (reading),
so the store holds exactly the positions visible at t = P - 1, in increasing
position order: slot(j) is the rank of j among them.  The window ring keeps,
for each of the last w positions j (j >= P - w), the pair (slot(j), flag(j))
at index j mod w, so that the decode step at position t finds token t - w,
the one leaving the delay window, at index t mod w.
"""
from __future__ import annotations

import numpy as np

from .mask import visible_positions


def prefill_kept_positions(evict: np.ndarray, w: int) -> np.ndarray:
    """Kept prompt positions of one (sequence, layer, kv-head), increasing."""
    P = len(evict)
    if P == 0:
        return np.zeros(0, dtype=np.int64)
    return visible_positions(P - 1, evict, w)


def prefill_slots(evict: np.ndarray, w: int) -> dict:
    """Logical slot of every kept prompt position: {position: slot}."""
    return {int(j): s for s, j in enumerate(prefill_kept_positions(evict, w))}


def prefill_ring(evict: np.ndarray, w: int) -> list:
    """Window ring after prefill: list of w entries, (slot, flag) or None."""
    P = len(evict)
    slot = prefill_slots(evict, w)
    ring = [None] * w
    for j in range(max(0, P - w), P):
        ring[j % w] = (slot[j], int(evict[j]))
    return ring
