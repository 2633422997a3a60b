"""Visibility rule of DMS delayed eviction (oracle; test infrastructure only).

Source: "NVIDIA veröffentlicht Qwen3-8B-DMS-8x ..." (mindverse), section
"Dynamic Memory Sparsification (DMS): Eine innovative Lösung" -- a token
marked for eviction is kept for a while after the mark (delayed eviction),
and the policy interpolates between a sliding window of the last w = 512
tokens (every token flagged) and full attention (no token flagged).  Also
"Nvidia DMS: сжатие памяти LLM в 8 раз ..." (stiva.ai), section
"Ключевое изобретение: delayed eviction".

Reading taken where the pages leave the edge open: the window is the w most
recent positions including the query's own, so key j is hidden from the
query at position t exactly when it is flagged and t - j >= w.
"""
from __future__ import annotations

import numpy as np


def is_visible(t: int, j: int, evict_j: int, w: int) -> bool:
    """True when key position j can be attended by the query at position t."""
    if j > t:
        return False
    return not (bool(evict_j) and t - j >= w)


def visible_positions(t: int, evict: np.ndarray, w: int) -> np.ndarray:
    """Increasing positions j in [0, t] visible at t; ``evict[j]`` is token j's flag."""
    return np.array([j for j in range(t + 1) if is_visible(t, j, int(evict[j]), w)],
                    dtype=np.int64)


def visible_mask(t: int, evict: np.ndarray, w: int) -> np.ndarray:
    """Boolean mask over positions 0..t."""
    m = np.zeros(t + 1, dtype=bool)
    m[visible_positions(t, evict, w)] = True
    return m
