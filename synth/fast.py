"""ctypes loader of ``hostgen.c``, the C twin of this package's generator,
for host draws too large for NumPy (test infrastructure and the oracle's
inputs; the CUDA library has its own device twin).

``normal`` and ``amax`` return exactly what the NumPy functions of
``synth`` return for the same coordinates (a CPU test compares them bit for
bit).  The shared library is built with gcc next to the source on first use
when it is missing or older than the source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hostgen.c")
_LIB = os.path.join(_HERE, "libhostgen.so")
_lib = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp"
        subprocess.run(["gcc", "-O3", "-shared", "-fPIC", "-o", tmp, _SRC, "-lpthread", "-lm"],
                       check=True, capture_output=True)
        os.replace(tmp, _LIB)
    return _LIB


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        h = ctypes.CDLL(build())
        P, I, I64, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64
        h.hostgen_normal.argtypes = [U64, I, I, I, P, I64, I, I, I, P, I]
        h.hostgen_normal.restype = None
        h.hostgen_amax.argtypes = [U64, I, I, I, I64, I64, I, I, I, P, I]
        h.hostgen_amax.restype = None
        _lib = h
    return _lib


def threads() -> int:
    """Threads per call: SYNTH_THREADS if set (e.g. 1 in worker processes
    that already run in parallel), else the CPUs this process may use."""
    env = os.environ.get("SYNTH_THREADS")
    if env:
        return max(1, min(64, int(env)))
    try:
        return max(1, min(64, len(os.sched_getaffinity(0))))
    except AttributeError:
        return max(1, min(64, os.cpu_count() or 1))


def _bf16(dtype: str) -> int:
    if dtype not in ("f32", "bf16"):
        raise ValueError(dtype)
    return int(dtype == "bf16")


def normal(seed: int, stream: int, layer: int, b: int, pos, head: int, head_dim: int,
           dtype: str) -> np.ndarray:
    """float32 [len(pos), head_dim]: synth.normal(seed, stream, layer, b,
    pos[:, None], head, arange(head_dim)[None, :], dtype)."""
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int64).reshape(-1))
    out = np.empty((len(pos), head_dim), dtype=np.float32)
    lib().hostgen_normal(seed, stream, layer, b, pos.ctypes.data, len(pos), head, head_dim,
                         _bf16(dtype), out.ctypes.data, threads())
    return out


def amax(seed: int, stream: int, layer: int, batch: int, pos0: int, n_pos: int, n_heads: int,
         head_dim: int, dtype: str) -> np.ndarray:
    """float32 [n_heads]: max |x| over sequences 0..batch-1, positions pos0 ..
    pos0+n_pos-1 and every element of each head's rows."""
    out = np.zeros(n_heads, dtype=np.float32)
    lib().hostgen_amax(seed, stream, layer, batch, pos0, n_pos, n_heads, head_dim, _bf16(dtype),
                       out.ctypes.data, threads())
    return out
