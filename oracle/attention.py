"""Dense fp64 masked GQA decode attention (oracle; test infrastructure only).

DMS changes which keys a query sees, not how attention is computed: for the
query at position t the output is plain softmax attention over the keys that
the delayed-eviction rule leaves visible ("NVIDIA veröffentlicht
Qwen3-8B-DMS-8x ..." (mindverse), section "Dynamic Memory Sparsification
(DMS): Eine innovative Lösung").  The compact KV store only skips the hidden
keys, so it reaches this result up to rounding order.

Readings: query head hq reads kv head hq // g with g = Hq / Hkv (contiguous
GQA groups); scores are scaled by ``sm_scale`` (1/sqrt(D) unless given).
"""
from __future__ import annotations

import numpy as np

from .mask import visible_positions


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, sm_scale: float) -> np.ndarray:
    """softmax(sm_scale * q K^T) V in fp64.  q [g, D], K/V [n, D] -> [g, D]."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    s = (q @ K.T) * float(sm_scale)                # [g, n]
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ V


def decode_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, evict: np.ndarray,
                     t: int, w: int, sm_scale: float | None = None) -> np.ndarray:
    """Output of the query at position t for one sequence of one layer.

    q      [Hq, D]        query of position t
    K, V   [t+1, Hkv, D]  stored keys / values of positions 0..t
    evict  [t+1, Hkv]     eviction flags
    returns [Hq, D] fp64
    """
    Hq, D = q.shape
    Hkv = K.shape[1]
    g = Hq // Hkv
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(D)
    out = np.zeros((Hq, D), dtype=np.float64)
    for hkv in range(Hkv):
        vis = visible_positions(t, evict[:, hkv], w)
        rows = slice(hkv * g, (hkv + 1) * g)
        out[rows] = attend(q[rows], K[vis, hkv], V[vis, hkv], sm_scale)
    return out


def prefill_attention(Q: np.ndarray, K: np.ndarray, V: np.ndarray, evict: np.ndarray, w: int,
                      sm_scale: float | None = None) -> np.ndarray:
    """Outputs of every prompt query of one sequence of one layer.

    The delayed-eviction mask applies to every query, not only to decode
    steps: query i sees key j <= i unless j is flagged and i - j >= w (the
    same rule as decode_attention with t = i).
    Q [P, Hq, D], K / V [P, Hkv, D], evict [P, Hkv] -> [P, Hq, D] fp64.
    """
    P = Q.shape[0]
    out = np.zeros(Q.shape, dtype=np.float64)
    for i in range(P):
        out[i] = decode_attention(Q[i], K[:i + 1], V[:i + 1], evict[:i + 1], i, w, sm_scale)
    return out
