"""Drive a seeded synthetic workload through the C ABI on one GPU.

Plumbing around ``dms``: sizes a pool for a workload, draws the prompt and
per-step inputs on the device with the generator twin (``dms_synth_*``),
runs prefill compaction layer by layer and the decode steps
(``dms_append_evict_layers`` then ``dms_decode_attn_layers`` over all
layers).  No method arithmetic lives here.
"""
from __future__ import annotations

import math

import numpy as np

from . import dms

STREAM_K, STREAM_V, STREAM_Q = 0, 1, 2


def _dtype_code(name: str) -> int:
    return {"f32": dms.DMS_F32, "bf16": dms.DMS_BF16, "fp8": dms.DMS_FP8_E4M3, "int4": dms.DMS_INT4}[name]


def expected_blocks(wl, steps: int, sigmas: float = 8.0) -> int:
    """Pool blocks for a workload: expected kept tokens per head plus a
    binomial margin, plus the decode steps, rounded up to blocks."""
    probs = wl.keep_probs()
    P, w = wl.prompt, wl.window
    older = max(0, P - w)
    total = 0
    for p in probs.reshape(-1):
        n = min(P, w) + p * older + sigmas * math.sqrt(max(p * (1 - p), 0.0) * older) + 1
        n = min(n, P) + steps
        total += math.ceil(n / dms.BLOCK_TOKENS) + 1
    return int(total * wl.batch + 16)


class DeviceWorkload:
    """A workload's pool plus its on-device inputs."""

    def __init__(self, wl, steps: int, device="cuda", max_blocks: int | None = None,
                 pregenerate_steps: bool = True, batch: int | None = None):
        import torch
        self.torch = torch
        self.wl = wl
        self.steps = steps
        self.device = torch.device(device)
        self.batch = batch or wl.batch
        self.L, self.Hq, self.Hkv, self.D = wl.n_layers, wl.n_q_heads, wl.n_kv_heads, wl.head_dim
        self.in_dtype = torch.float32 if wl.in_dtype == "f32" else torch.bfloat16
        self.in_code = _dtype_code(wl.in_dtype)
        self.thr = torch.tensor(wl.thresholds().astype(np.int32), device=self.device)
        self.pool = dms.Pool(self.L, self.batch, self.Hq, self.Hkv, self.D, wl.window,
                             _dtype_code(wl.kv_dtype),
                             max_blocks or expected_blocks(wl, steps), wl.prompt + steps + 1,
                             device=self.device)
        self.out = torch.empty(self.L, self.batch, self.Hq, self.D, dtype=self.in_dtype,
                               device=self.device)
        self.step_inputs = None
        if pregenerate_steps and steps > 0:
            self.step_inputs = self.make_step_inputs(wl.prompt, steps)

    # ---- generation -------------------------------------------------------
    def _stream(self):
        return int(self.torch.cuda.current_stream().cuda_stream)

    def normal(self, stream_id, layer0, n_layers, pos0, n_pos, n_heads, out=None):
        t = self.torch
        shape = (n_layers, self.batch, n_pos, n_heads, self.D)
        if out is None:
            out = t.empty(shape, dtype=self.in_dtype, device=self.device)
        dms.dms_synth_normal(self.wl.seed, stream_id, layer0, n_layers, self.batch, pos0, n_pos,
                             n_heads, self.D, self.in_code, out.data_ptr(), self._stream())
        return out

    def flags(self, layer0, n_layers, pos0, n_pos, out=None):
        t = self.torch
        shape = (n_layers, self.batch, n_pos, self.Hkv)
        if out is None:
            out = t.empty(shape, dtype=t.uint8, device=self.device)
        thr = self.thr[layer0:layer0 + n_layers].contiguous()
        dms.dms_synth_flags(self.wl.seed, layer0, n_layers, self.batch, pos0, n_pos, self.Hkv,
                            thr.data_ptr(), out.data_ptr(), self._stream())
        return out

    def make_step_inputs(self, pos0: int, n_steps: int) -> dict:
        """k, v [n_steps, L, B, Hkv, D]; q [n_steps, L, B, Hq, D]; evict [n_steps, L, B, Hkv]."""
        t = self.torch
        S = n_steps
        k = t.empty(S, self.L, self.batch, self.Hkv, self.D, dtype=self.in_dtype, device=self.device)
        v = t.empty_like(k)
        q = t.empty(S, self.L, self.batch, self.Hq, self.D, dtype=self.in_dtype, device=self.device)
        e = t.empty(S, self.L, self.batch, self.Hkv, dtype=t.uint8, device=self.device)
        for s in range(S):
            self.normal(STREAM_K, 0, self.L, pos0 + s, 1, self.Hkv, out=k[s])
            self.normal(STREAM_V, 0, self.L, pos0 + s, 1, self.Hkv, out=v[s])
            self.normal(STREAM_Q, 0, self.L, pos0 + s, 1, self.Hq, out=q[s])
            self.flags(0, self.L, pos0 + s, 1, out=e[s])
        return {"k": k, "v": v, "q": q, "evict": e, "pos0": pos0}

    # ---- the path ---------------------------------------------------------
    def prefill(self, layers=None, timed=False):
        """Compact every layer's prompt (inputs drawn on the device, one layer at a
        time).  With timed=True the first layer runs eagerly (it loads the
        kernels), the others are captured once into a CUDA graph and replayed
        once, and the device milliseconds of each layer's compaction call alone
        (CUDA events, event nodes in the graph) are returned."""
        t = self.torch
        P = self.wl.prompt
        kbuf = t.empty(1, self.batch, P, self.Hkv, self.D, dtype=self.in_dtype, device=self.device)
        vbuf = t.empty_like(kbuf)
        fbuf = t.empty(1, self.batch, P, self.Hkv, dtype=t.uint8, device=self.device)
        layers = list(range(self.L) if layers is None else layers)
        events = [(t.cuda.Event(enable_timing=True, external=True),
                   t.cuda.Event(enable_timing=True, external=True)) for _ in layers] if timed else None

        def run(first, last):
            for i in range(first, last):
                layer = layers[i]
                self.normal(STREAM_K, layer, 1, 0, P, self.Hkv, out=kbuf)
                self.normal(STREAM_V, layer, 1, 0, P, self.Hkv, out=vbuf)
                self.flags(layer, 1, 0, P, out=fbuf)
                if timed:
                    events[i][0].record()
                self.pool.compact_prefill(layer, kbuf[0], vbuf[0], fbuf[0])
                if timed:
                    events[i][1].record()

        if timed:
            run(0, min(1, len(layers)))
            t.cuda.synchronize(self.device)
            if len(layers) > 1:
                graph = t.cuda.CUDAGraph()
                with t.cuda.graph(graph):
                    run(1, len(layers))
                graph.replay()
                t.cuda.synchronize(self.device)
                del graph
        else:
            run(0, len(layers))
            t.cuda.synchronize(self.device)
        del kbuf, vbuf, fbuf
        if timed:
            return [float(a.elapsed_time(b)) for a, b in events]
        return None

    def step(self, s: int, out=None):
        """Decode step s (position prompt + s): append/evict all layers, then attention."""
        si = self.step_inputs
        pos = si["pos0"] + s
        self.pool.append_evict_layers(0, pos, si["k"][s], si["v"][s], si["evict"][s])
        self.pool.decode_attn_layers(0, si["q"][s], self.out if out is None else out)

    def retained_bytes(self) -> int:
        """Bytes of held K/V rows right now (device stats; synchronises)."""
        return int(self.pool.stats().kv_bytes_retained)
