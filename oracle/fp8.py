"""Software FP8-E4M3 codec and per-head scale (oracle; test infrastructure only).

Storage composition: eviction decides which tokens stay, and FP8 then
quantises what stays ("FastDMS: vLLM BF16/FP8보다 빠른 6.4x KV cache 압축"
(molayo1419.me), the paragraph after the speed table).  The format itself is
the OCP 8-bit floating point E4M3 ("fn") encoding: 1 sign bit, 4 exponent
bits with bias 7, 3 mantissa bits; exponent field 0 holds subnormals
(m/8 * 2^-6); S.1111.111 is NaN; there is no infinity; the largest finite
magnitude is 1.75 * 2^8 = 448.

Readings (the pages give no quantisation detail): one fp32 scale per
(layer, kv-head) for K and one for V, shared by the batch, equal to
amax/448 over every prompt token of that head before eviction (1 when amax
is 0); a value is stored as e4m3(x / scale) with the quotient taken in IEEE
fp32 and rounded to nearest even, saturating to +-448.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_NAN = 0x7F


def e4m3_decode(codes) -> np.ndarray:
    """Exact value of each E4M3 code as float64 (NaN for S.1111.111)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


_POS_CODES = np.arange(0x7F, dtype=np.uint8)          # 0x00 .. 0x7E, all finite
_POS_VALUES = e4m3_decode(_POS_CODES)                  # increasing


def e4m3_encode(x) -> np.ndarray:
    """Round float values to E4M3 codes: nearest, ties to even, saturating to +-448.

    The rounding grid of |x| in the binade [2^e, 2^(e+1)) (e >= -6) is
    2^(e-3); below 2^-6 it is the subnormal step 2^-9."""
    a = np.asarray(x, dtype=np.float64)
    nan = np.isnan(a)
    neg = np.signbit(a)
    mag = np.abs(np.where(nan, 0.0, a))
    _, ex = np.frexp(mag)                      # mag = f * 2^ex, f in [0.5, 1)
    e = np.maximum(ex - 1, -6)                 # floor(log2 mag), clamped to the subnormal range
    step = np.exp2(e - 3.0)
    r = np.rint(mag / step) * step             # np.rint rounds half to even
    r = np.minimum(r, E4M3_MAX)
    idx = np.searchsorted(_POS_VALUES, r)
    assert np.all(_POS_VALUES[idx] == r), "rounded value off the E4M3 grid"
    codes = _POS_CODES[idx] | np.where(neg, 0x80, 0).astype(np.uint8)
    return np.where(nan, np.uint8(E4M3_NAN), codes).astype(np.uint8)


def fp8_scale(amax) -> np.float32:
    """Per-head scale amax/448 in IEEE fp32 (1 when amax is 0)."""
    a = np.float32(amax)
    if a == 0:
        return np.float32(1.0)
    return np.float32(a / np.float32(E4M3_MAX))


def quantize(x, scale) -> np.ndarray:
    """E4M3 codes of x / scale, the quotient in IEEE fp32."""
    y = np.asarray(x, dtype=np.float32) / np.float32(scale)
    return e4m3_encode(y.astype(np.float64))


def dequantize(codes, scale) -> np.ndarray:
    """Stored value decode(code) * scale in fp64 (exact: 4 x 24 significant bits)."""
    return e4m3_decode(codes) * np.float64(np.float32(scale))
