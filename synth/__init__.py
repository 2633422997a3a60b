"""Seeded synthetic workloads for compact-KV decode (NumPy side).

This module draws random numbers and nothing else: it holds none of the
attention, eviction, compaction or quantisation arithmetic.  Both the CPU
oracle and the CUDA tests take their inputs from here; the CUDA library
carries a twin of `hash64` / `normal` / `evict_flags` (``dms_synth_*``) that
must reproduce these values bit for bit, which a test checks.

Generator
---------
Every value is a pure function of its coordinates, so any element can be
regenerated alone (which is what lets a CPU test sample a 100 GB workload).

* ``hash64(key, n)`` is the n-th output of a SplitMix64 stream whose state
  starts at ``key``:  ``mix64(key + n * GAMMA)`` with the SplitMix64 increment
  ``GAMMA = 0x9E3779B97F4A7C15`` and the finaliser ``mix64`` of Steele, Lea and
  Flood, "Fast splittable pseudorandom number generators" (OOPSLA 2014),
  variant "Mix13" (shifts 30/27/31).
* ``stream_key(seed, stream) = mix64(seed XOR (stream << 56))``.  Streams:
  0 = K, 1 = V, 2 = Q, 3 = eviction flags.
* The counter packs the coordinates of one draw:
  ``layer << 52 | b << 44 | pos << 20 | head << 12 | d << 2 | k``
  (k < 4 selects one of the hash words of an element; pos < 2**24,
  head < 256, d < 1024, b < 256, layer < 4096).
* "~N(0,1)" values: three hash words give twelve 16-bit uniforms u_i; the
  Irwin-Hall sum gives ``x = (sum(u_i) - 393210) * 2**-16``, computed as one
  exact int->fp32 conversion times a power of two (mean exactly 0, variance
  1 - 2**-32, bounded by 6).  bf16 tensors take ``x`` rounded to nearest even.
* Eviction flags: one hash word per (layer, b, pos, kv-head); its top 24 bits
  ``u`` give ``keep = u < thr`` with ``thr = rint(p_keep * 2**24)`` from the
  host, and ``evict = not keep``.
"""
from __future__ import annotations

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

STREAM_K, STREAM_V, STREAM_Q, STREAM_FLAGS = 0, 1, 2, 3
IRWIN_HALL_CENTER = 393210  # 12 * (2**16 - 1) / 2

# counter bit positions
SH_K, SH_D, SH_HEAD, SH_POS, SH_B, SH_LAYER = 0, 2, 12, 20, 44, 52


def mix64(z):
    """SplitMix64 finaliser (Mix13 constants) on uint64 arrays, wrapping mod 2**64."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, stream: int) -> np.uint64:
    return mix64(np.uint64(seed) ^ (np.uint64(stream) << np.uint64(56)))[()]


def hash64(key, counter):
    """n-th output of a SplitMix64 stream seeded with ``key`` (n = counter)."""
    with np.errstate(over="ignore"):
        return mix64(np.uint64(key) + np.asarray(counter, dtype=np.uint64) * GAMMA)


def counter(layer, b, pos, head, d, k=0):
    """Pack coordinates into the 64-bit counter (broadcasting)."""
    u = lambda x: np.asarray(x, dtype=np.uint64)  # noqa: E731
    return ((u(layer) << np.uint64(SH_LAYER)) | (u(b) << np.uint64(SH_B))
            | (u(pos) << np.uint64(SH_POS)) | (u(head) << np.uint64(SH_HEAD))
            | (u(d) << np.uint64(SH_D)) | (u(k) << np.uint64(SH_K)))


def normal_f32(seed, stream, layer, b, pos, head, d):
    """Irwin-Hall ~N(0,1) draws as float32 (exact: integer sum times 2**-16)."""
    key = stream_key(seed, stream)
    base = counter(layer, b, pos, head, d, 0)
    total = np.zeros(np.shape(base), dtype=np.int64)
    for k in range(3):
        h = hash64(key, base | np.uint64(k))
        for i in range(4):
            total += ((h >> np.uint64(16 * i)) & np.uint64(0xFFFF)).astype(np.int64)
    return (total - IRWIN_HALL_CENTER).astype(np.float32) * np.float32(2.0 ** -16)


def f32_to_bf16_bits(x):
    """Round float32 to bfloat16 (nearest, ties to even); returns uint16 bits.

    Inputs here are finite by construction (|x| <= 6)."""
    bits = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (bits + np.uint64(0x7FFF) + ((bits >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(bits):
    return (np.asarray(bits, dtype=np.uint32) << np.uint32(16)).view(np.float32)


def normal(seed, stream, layer, b, pos, head, d, dtype):
    """Draws in storage precision, returned as float32 values.

    dtype "f32" keeps the Irwin-Hall float32; "bf16" rounds it to bfloat16."""
    x = normal_f32(seed, stream, layer, b, pos, head, d)
    if dtype == "f32":
        return x
    if dtype == "bf16":
        return bf16_bits_to_f32(f32_to_bf16_bits(x))
    raise ValueError(dtype)


def keep_threshold(p_keep):
    """Host-side 24-bit threshold for a keep probability (array or scalar)."""
    p = np.clip(np.asarray(p_keep, dtype=np.float64), 0.0, 1.0)
    return np.rint(p * float(1 << 24)).astype(np.int64)


def evict_flags(seed, layer, b, pos, head, thr):
    """uint8 eviction flags: 1 = flagged for (delayed) eviction."""
    h = hash64(stream_key(seed, STREAM_FLAGS), counter(layer, b, pos, head, 0, 0))
    u24 = (h >> np.uint64(40)).astype(np.int64)
    return (u24 >= np.asarray(thr, dtype=np.int64)).astype(np.uint8)


# --------------------------------------------------------------------------
# Whole-tensor helpers (small cases; large ones are generated on the device)
# --------------------------------------------------------------------------

def kv_tokens(seed, stream, layer, batch, pos0, n_pos, n_kv_heads, head_dim, dtype):
    """K or V rows for positions [pos0, pos0+n_pos): float32 array [B, n_pos, Hkv, D]."""
    b = np.arange(batch)[:, None, None, None]
    p = (pos0 + np.arange(n_pos))[None, :, None, None]
    h = np.arange(n_kv_heads)[None, None, :, None]
    d = np.arange(head_dim)[None, None, None, :]
    return normal(seed, stream, layer, b, p, h, d, dtype)


def q_tokens(seed, layer, batch, pos, n_q_heads, head_dim, dtype):
    """Decode query for position ``pos``: float32 array [B, Hq, D]."""
    b = np.arange(batch)[:, None, None]
    h = np.arange(n_q_heads)[None, :, None]
    d = np.arange(head_dim)[None, None, :]
    return normal(seed, STREAM_Q, layer, b, pos, h, d, dtype)


def flag_tokens(seed, layer, batch, pos0, n_pos, n_kv_heads, thr_layer):
    """Eviction flags for positions [pos0, pos0+n_pos): uint8 [B, n_pos, Hkv].

    ``thr_layer`` holds one 24-bit keep threshold per kv-head of this layer."""
    b = np.arange(batch)[:, None, None]
    p = (pos0 + np.arange(n_pos))[None, :, None]
    h = np.arange(n_kv_heads)[None, None, :]
    thr = np.asarray(thr_layer, dtype=np.int64)[None, None, :]
    return evict_flags(seed, layer, b, p, h, thr)
