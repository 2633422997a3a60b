"""K/V projection and eviction decision of one decode token (oracle; test
infrastructure only).

DMS is retrofitted onto a model: each attention layer's projection gives the
token's keys and values, and a learned predictor gives, per kv-head, the
decision whether the token will be evicted once it leaves the delayed
window ("NVIDIA veröffentlicht Qwen3-8B-DMS-8x ..." (mindverse), section
"Dynamic Memory Sparsification (DMS): Eine innovative Lösung"; "Nvidia DMS
..." (stiva.ai), section "Ключевое изобретение: delayed eviction").  The
predictor's weights are an input here (training them needs data).

Readings: k[h] = x @ W_kv[:, h*D:(h+1)*D], v[h] = x @ W_kv[:, (Hkv+h)*D:
(Hkv+h+1)*D]; the eviction logit of head h is x @ w_evict[:, h] + b_evict[h]
and the token is flagged when the logit exceeds the threshold (a logistic
decision at probability 1/2 is threshold 0).  k and v are rounded to bf16,
the precision the store's inputs have.
"""
from __future__ import annotations

import numpy as np


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Correctly rounded bf16 of fp64 values (nearest, ties to even), as fp64.

    The two bf16 neighbours of x are found from its fp32 value truncated to
    bf16 (the bf16 grid is part of the fp32 grid, so fp32 rounding cannot
    step over one of them); the nearer one wins, ties go to the even one."""
    x = np.asarray(x, dtype=np.float64)
    f = x.astype(np.float32)
    lo_bits = f.view(np.uint32) & np.uint32(0xFFFF0000)
    lo = lo_bits.view(np.float32).astype(np.float64)                 # toward zero
    hi = (lo_bits + np.uint32(0x10000)).view(np.float32).astype(np.float64)  # away from zero
    d_lo, d_hi = np.abs(x - lo), np.abs(hi - x)
    lo_even = ((lo_bits >> 16) & 1) == 0
    pick_lo = (d_lo < d_hi) | ((d_lo == d_hi) & lo_even)
    return np.where(pick_lo, lo, hi)


def project_token(x: np.ndarray, W_kv: np.ndarray, w_evict: np.ndarray, b_evict: np.ndarray,
                  n_kv_heads: int, head_dim: int):
    """x [d_model] -> (k [Hkv, D] fp64 exact, v [Hkv, D] fp64 exact, logit [Hkv] fp64)."""
    x = np.asarray(x, dtype=np.float64)
    kv = x @ np.asarray(W_kv, dtype=np.float64)                 # [2 * Hkv * D]
    Hkv, D = n_kv_heads, head_dim
    k = kv[:Hkv * D].reshape(Hkv, D)
    v = kv[Hkv * D:].reshape(Hkv, D)
    logit = x @ np.asarray(w_evict, dtype=np.float64) + np.asarray(b_evict, dtype=np.float64)
    return k, v, logit


def evict_flags(logit: np.ndarray, threshold: float) -> np.ndarray:
    return (np.asarray(logit) > threshold).astype(np.uint8)
