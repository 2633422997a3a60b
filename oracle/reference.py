"""Per-head expected values for a seeded synthetic workload (oracle).

Glue between ``synth`` (inputs, drawn by its C twin ``synth.fast`` for speed)
and the oracle's definitions: it regenerates the inputs of one (layer,
sequence, kv-head) from the seed, forms the values
the store holds (the model's K/V in their input precision, for an FP8 store
their E4M3 codes times the per-head scale, for a 4-bit store their group
codes times the group scales) and evaluates the oracle's
mask, compaction, slot simulator and attention on them.  Everything is fp64
except where the stored precision is the point (bf16 rounding, fp32 quotient
before E4M3 rounding).
"""
from __future__ import annotations

import numpy as np

import synth
from synth import fast as synth_fast

from .attention import attend
from .fp8 import dequantize, fp8_scale, quantize
from .int4 import stored as int4_stored
from .mask import visible_positions


def head_flags(wl, layer: int, b: int, h: int, n_pos: int) -> np.ndarray:
    """uint8 eviction flags of positions 0..n_pos-1 for one kv-head."""
    thr = wl.thresholds()[layer, h]
    return synth.evict_flags(wl.seed, layer, b, np.arange(n_pos), h, thr)


def head_input(wl, stream: int, layer: int, b: int, h: int, pos0: int, n_pos: int) -> np.ndarray:
    """float32 [n_pos, D]: the model's K (stream 0) or V (stream 1) rows in input precision."""
    return synth_fast.normal(wl.seed, stream, layer, b, pos0 + np.arange(n_pos), h, wl.head_dim,
                             wl.in_dtype)


def fp8_layer_scales(wl, layer: int) -> list:
    """[(scale_K, scale_V)] of every kv-head of a layer: amax/448 over the
    whole prompt of every sequence, before eviction."""
    amax = [synth_fast.amax(wl.seed, stream, layer, wl.batch, 0, wl.prompt, wl.n_kv_heads,
                            wl.head_dim, wl.in_dtype) for stream in (synth.STREAM_K, synth.STREAM_V)]
    return [(fp8_scale(amax[0][h]), fp8_scale(amax[1][h])) for h in range(wl.n_kv_heads)]


def fp8_head_scales(wl, layer: int, h: int, chunk: int = 4096) -> tuple:
    """(scale_K, scale_V) of one (layer, kv-head): amax/448 over the whole
    prompt and batch, taken chunk by chunk of positions."""
    scales = []
    for stream in (synth.STREAM_K, synth.STREAM_V):
        amax = np.float32(0.0)
        for b in range(wl.batch):
            for p0 in range(0, wl.prompt, chunk):
                n = min(chunk, wl.prompt - p0)
                x = head_input(wl, stream, layer, b, h, p0, n)
                amax = max(amax, np.float32(np.abs(x).max()))
        scales.append(fp8_scale(amax))
    return scales[0], scales[1]


def stored_rows(wl, layer: int, b: int, h: int, pos: np.ndarray, scales=None):
    """(K, V) fp64 [len(pos), D] as held by the store for the given positions."""
    pos = np.asarray(pos, dtype=np.int64)
    out = []
    for i, stream in enumerate((synth.STREAM_K, synth.STREAM_V)):
        x = synth_fast.normal(wl.seed, stream, layer, b, pos, h, wl.head_dim, wl.in_dtype)
        if wl.kv_dtype == "fp8":
            out.append(dequantize(quantize(x, scales[i]), scales[i]))
        elif wl.kv_dtype == "int4":
            out.append(int4_stored(x))
        else:
            out.append(x.astype(np.float64))
    return out[0], out[1]


def head_query(wl, layer: int, b: int, h_kv: int, t: int) -> np.ndarray:
    """float32 [g, D]: queries of the GQA group of kv-head h_kv at position t."""
    g = wl.group
    heads = np.arange(h_kv * g, (h_kv + 1) * g)[:, None]
    return synth.normal(wl.seed, synth.STREAM_Q, layer, b, t, heads,
                        np.arange(wl.head_dim)[None, :], wl.in_dtype)


def expected_output(wl, layer: int, b: int, h_kv: int, t: int, sm_scale: float | None = None,
                    scales=None) -> np.ndarray:
    """fp64 [g, D] decode output of the query heads of kv-head h_kv at position t."""
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(wl.head_dim)
    flags = head_flags(wl, layer, b, h_kv, t + 1)
    vis = visible_positions(t, flags, wl.window)
    K, V = stored_rows(wl, layer, b, h_kv, vis, scales)
    q = head_query(wl, layer, b, h_kv, t).astype(np.float64)
    return attend(q, K, V, sm_scale)
