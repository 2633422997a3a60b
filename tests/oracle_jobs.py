"""Oracle evaluations run in worker processes (test infrastructure).

The full-size parity tests compare every head of a decode step with the fp64
oracle; the heads are independent, so they are spread over a process pool
started with the "spawn" method (safe after the parent has initialised
CUDA: the workers import only NumPy, the generator and the oracle)."""
from __future__ import annotations

import multiprocessing as mp
import os

_POOL = None


def _init():
    os.environ["SYNTH_THREADS"] = "1"


def _expected(args):
    from synth import configs
    from oracle import reference as oref
    name, l, b, h, t, scales = args
    return oref.expected_output(configs.BY_NAME[name], l, b, h, t, scales=scales)


def pool():
    """A shared spawn pool with one worker per usable CPU (at most 32)."""
    global _POOL
    if _POOL is None:
        n = max(1, min(32, len(os.sched_getaffinity(0))))
        _POOL = mp.get_context("spawn").Pool(n, initializer=_init)
    return _POOL


def expected_outputs(wl, heads, t, scales=None):
    """fp64 oracle outputs [len(heads), g, D] of heads (layer, seq, kv-head) at position t."""
    jobs = [(wl.name, l, b, h, t, None if scales is None else scales[l][h]) for (l, b, h) in heads]
    return pool().map(_expected, jobs, chunksize=max(1, len(jobs) // (8 * pool()._processes)))
