"""4-bit K/V with per-group scales (oracle; test infrastructure only).

DMS composes with quantisation of what it keeps: FastDMS decides eviction
before FP8 quantisation ("FastDMS: vLLM BF16/FP8보다 빠른 6.4x KV cache 압축"
(molayo1419.me), paragraph after the speed table), and the pages place
sparsification next to lower-bit KV (the same page's comparison with
TurboQuant 4-bit KV, and the memory table).  The pages give no 4-bit format;
the reading taken here is the plain symmetric one:

* each stored row (one token of one kv-head, K or V) is cut into groups of
  GROUP = 32 consecutive elements;
* a group's scale is amax / 7 computed in IEEE fp32, rounded to the nearest
  fp16 (ties to even; 65504 at most); a group of zeros has scale 0;
* each value is stored as q = clamp(rint(x / scale), -7, 7), the quotient in
  IEEE fp32 and rint rounding half to even; scale 0 gives q = 0;
* the stored value is q * scale (exact in fp32: 4 x 11 significant bits).
"""
from __future__ import annotations

import numpy as np

GROUP = 32
QMAX = 7


def group_scales(x: np.ndarray) -> np.ndarray:
    """fp16 scales (as float32) of the groups of each row of x [..., D]."""
    x = np.asarray(x, dtype=np.float32)
    g = x.reshape(x.shape[:-1] + (x.shape[-1] // GROUP, GROUP))
    amax = np.abs(g).max(axis=-1).astype(np.float32)
    s = (amax / np.float32(QMAX)).astype(np.float32)
    return np.minimum(s.astype(np.float16), np.float16(65504.0)).astype(np.float32)


def quantize(x: np.ndarray):
    """x [..., D] float32 -> (q int8 [..., D] in [-7, 7], scales float32 [..., D / 32])."""
    x = np.asarray(x, dtype=np.float32)
    s = group_scales(x)
    sx = np.repeat(s, GROUP, axis=-1)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(sx > 0, np.rint(x / np.where(sx > 0, sx, np.float32(1))), 0)
    q = np.clip(r, -QMAX, QMAX).astype(np.int8)
    return q, s


def dequantize(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Stored values q * scale in fp64 (exact)."""
    return np.asarray(q, np.float64) * np.repeat(np.asarray(s, np.float64), GROUP, axis=-1)


def stored(x: np.ndarray) -> np.ndarray:
    """The values a 4-bit store holds for x, fp64."""
    return dequantize(*quantize(x))
