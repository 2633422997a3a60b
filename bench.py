#!/usr/bin/env python
"""Benchmark: compact-KV DMS decode on B200.

One step = one decode position of the whole hot path over every layer of the
workload: dms_append_evict_layers (retire / reclaim / append) then
dms_decode_attn_layers (split-K attention over each head's held rows).
The default workload is Qwen3-8B attention shapes at ctx 8192 (36 layers,
32 q / 8 kv heads, head_dim 128, bf16 K/V, window 512, per-head keep
probability U[0.02, 0.30], seed 2).

value      retained-KV GB/s of the whole step (held K/V bytes read per step,
           summed over steps and ranks, / max-over-ranks device time)
roofline   the attention kernel alone: algorithmic bytes / its CUDA-event time
e2e        the same metric through the Python/C API with pinned host inputs
           copied in and outputs copied out inside the timed region
cpu_baseline  the CPU oracle timed on a bounded sample (rank 0, N = 1)

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
(for N > 1 launch with torch.distributed.run; each rank runs a replica).
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402
from synth import configs  # noqa: E402

METRIC = "compact-KV decode attn: retained-KV GB/s vs HBM peak; decode steps/s at ctx 8K"
DEFAULT_WORKLOAD = configs.QWEN8B_CTX8K.name
ATTN_KERNEL_SRC = os.path.join(ROOT, "compact_decode_attention_b200", "csrc", "attn.cu")
PROFILES = os.path.join(ROOT, "profiles")
L2_BYTES = 126 * 1024 * 1024
L2_FLUSH_BYTES = 512 * 1024 * 1024   # written between timed steps when the held K/V fits in L2


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(configs.BY_NAME))
    ap.add_argument("--kv-dtype", default=None, choices=["f32", "bf16", "fp8", "int4"],
                    help="store the workload's K/V in this dtype instead of its own")
    ap.add_argument("--e2e-steps", type=int, default=256)
    ap.add_argument("--no-numa-bind", action="store_true",
                    help="do not pin the process to the CPUs local to its GPU")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill-attention measurement")
    ap.add_argument("--prefill-only", action="store_true",
                    help="run only the prefill-attention measurement and print it")
    ap.add_argument("--projection-only", action="store_true",
                    help="run only the fused K/V projection + append measurement and print it")
    ap.add_argument("--prefill-prompt", type=int, default=0,
                    help="prompt length for --prefill-only (default: the workload's)")
    ap.add_argument("--cpu-heads", type=int, default=72)
    ap.add_argument("--cpu-steps", type=int, default=90)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case", action="store_true",
                    help="run a short fixed case for kernel captures (prefill, 4 all-layer steps, "
                         "2 steps as per-layer fused calls) and exit; prints no bench line")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# measured peaks, clocks
# ---------------------------------------------------------------------------

KV_TAGS = {"f32": "fp32", "bf16": "bf16", "fp8": "fp8e4m3", "int4": "int4g32"}


def with_kv_dtype(wl, kv_dtype):
    """The workload with its K/V stored in another dtype (the name's dtype
    tag follows)."""
    if not kv_dtype or kv_dtype == wl.kv_dtype:
        return wl
    import dataclasses
    old, new = "_" + KV_TAGS[wl.kv_dtype], "_" + KV_TAGS[kv_dtype]
    i = wl.name.rfind(old)
    name = wl.name[:i] + new + wl.name[i + len(old):] if i >= 0 else wl.name + new
    return dataclasses.replace(wl, name=name, kv_dtype=kv_dtype)


def parse_cpulist(text: str) -> set:
    """The CPUs of a sysfs cpu list such as "0-15,32-47"."""
    cpus = set()
    for part in text.strip().split(","):
        if "-" in part:
            a, b = part.split("-")
            cpus.update(range(int(a), int(b) + 1))
        elif part:
            cpus.add(int(part))
    return cpus


def bind_to_gpu_numa_node(device_index: int):
    """Pin this process to the CPUs the GPU's PCI function reports as local
    (sysfs local_cpulist), so that pinned host buffers are allocated on the
    GPU's NUMA node.  Returns the CPU list, or None when it is unknown."""
    import torch
    prop = torch.cuda.get_device_properties(device_index)
    path = "/sys/bus/pci/devices/%04x:%02x:%02x.0/local_cpulist" % (
        prop.pci_domain_id, prop.pci_bus_id, prop.pci_device_id)
    try:
        text = open(path).read().strip()
    except OSError:
        return None
    cpus = parse_cpulist(text) & os.sched_getaffinity(0)
    if not cpus:
        return None
    os.sched_setaffinity(0, cpus)
    return text


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def measured_bf16_tflops():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return float(json.load(open(p))["bf16_tflops"]), "measured burst cuBLAS bf16 (MEASURED_PEAKS.json bf16_tflops)"
    return 1590.0, "fallback 1.59 PFLOP/s"


def projection_line(wl, device, n_calls=8):
    """dms_project_append (K/V projection + eviction decision + append, fused)
    for one layer and the workload's batch, d_model = Hq * D (4096 for the
    Qwen3-8B shapes), synthetic bf16 weights: n_calls decode steps captured
    in a CUDA graph, mean time per call.  Bytes = weights read (W_kv and the predictor) + x + rows written;
    the kernel streams the weights once, so HBM bandwidth bounds it."""
    import torch
    from compact_decode_attention_b200 import dms
    if wl.head_dim != 128 or wl.kv_dtype == "f32":
        return None
    B, Hq, Hkv, D = wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim
    dm = Hq * D
    g = torch.Generator(device=device).manual_seed(wl.seed)
    w_kv = (torch.randn(dm, 2 * Hkv * D, device=device, generator=g) / dm ** 0.5).to(torch.bfloat16)
    w_ev = (torch.randn(dm, Hkv, device=device, generator=g) / dm ** 0.5).to(torch.bfloat16)
    x = torch.randn(n_calls + 1, B, dm, device=device, generator=g).to(torch.bfloat16)
    code = {"bf16": dms.DMS_BF16, "fp8": dms.DMS_FP8_E4M3, "int4": dms.DMS_INT4}[wl.kv_dtype]
    pool = dms.Pool(1, B, Hq, Hkv, D, wl.window, code, B * Hkv * 4, n_calls + 2, device=device)
    pos = [torch.full((B,), c, dtype=torch.int64, device=device) for c in range(n_calls + 1)]
    pool.project_append(0, None, pos[0], x[0], w_kv, w_ev)      # module load, workspace
    torch.cuda.synchronize()
    # the timed calls are captured once into a graph and replayed once, so the
    # host's issue time cannot leave the GPU idle inside the timed region
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for c in range(1, n_calls + 1):
            pool.project_append(0, None, pos[c], x[c], w_kv, w_ev)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    graph.replay()
    e1.record()
    torch.cuda.synchronize()
    if pool.stats(check=False).error_flags:
        raise SystemExit("the projection set the device error word")
    ms = e0.elapsed_time(e1) / n_calls
    nbytes = (w_kv.numel() + w_ev.numel() + B * dm) * 2 + B * Hkv * 2 * wl.kv_row_bytes()
    peak, kind = measured_peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"value": gbs, "unit": "GB/s", "us_per_layer": ms * 1e3, "d_model": dm, "batch": B,
            "algorithmic_bytes": nbytes,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak},
            "kernel": "project_append_kernel<128> (split-K over d_model, epilogue appends)"}


def prefill_tiles(flags: np.ndarray, P: int, w: int, tile: int = 128):
    """Key tiles per (sequence, kv-head) that the prefill attention kernel
    computes, summed over its query tiles: (dense, sparse).  flags uint8
    [B, P, Hkv].  Dense: every causal tile.  Sparse: a query tile
    [i0, i0 + 128) reads the band of prompt tiles from the one holding
    i0 - w + 1 to the diagonal, plus ceil(n_far / 128) tiles of older
    unflagged keys from the store (n_far of them), unless those tiles' slots
    run past the head's kept rows (then all causal tiles)."""
    B, _, Hkv = flags.shape
    n = (P + tile - 1) // tile
    dense = n * (n + 1) // 2
    sparse = np.zeros((B, Hkv), dtype=np.int64)
    for b in range(B):
        for h in range(Hkv):
            f = flags[b, :, h]
            unfl = np.concatenate([[0], np.cumsum(f == 0)])
            kept = int(unfl[P]) + int(np.sum(f[max(0, P - w):] != 0))
            tot = 0
            for qt in range(n):
                lo = qt * tile - w + 1
                kl = lo // tile if lo > 0 else 0
                nf = (int(unfl[kl * tile]) + tile - 1) // tile
                if kl > 0 and nf * tile <= kept:
                    tot += nf + qt - kl + 1
                else:
                    tot += qt + 1
            sparse[b, h] = tot
    return dense, sparse


def prefill_attention_line(wl, device, n_layers=3):
    """dms_prefill_attn (prompt attention under the DMS mask on the tensor
    cores, with compaction) at the workload's prompt shapes: one layer per
    call, the median of n_layers calls, each into an empty layer of a small
    pool; the default reading (old kept keys from the store) and the dense
    one (every causal tile from the prompt).  FLOPs = 4 D 128^2 per key tile
    computed (QK and PV, 2 flops per multiply-add); the visible (query, key)
    pairs give the method's own count."""
    import torch
    from compact_decode_attention_b200 import dms
    from compact_decode_attention_b200.workload import DeviceWorkload, STREAM_K, STREAM_Q, STREAM_V
    if wl.kv_dtype != "bf16" or wl.head_dim not in (64, 128):
        return None
    P, B, Hq, Hkv, D = wl.prompt, wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim
    g = Hq // Hkv
    gen = DeviceWorkload(wl, 0, device=device, max_blocks=16)
    k = gen.normal(STREAM_K, 0, 1, 0, P, Hkv)[0]
    v = gen.normal(STREAM_V, 0, 1, 0, P, Hkv)[0]
    q = gen.normal(STREAM_Q, 0, 1, 0, P, Hq)[0]
    f = gen.flags(0, 1, 0, P)[0]
    out = torch.empty_like(q)

    def time_mode(mode):
        pool = dms.Pool(n_layers + 1, B, Hq, Hkv, D, wl.window, dms.DMS_BF16,
                        (n_layers + 1) * B * Hkv * (P // 64 + 2), P + 1, device=device)
        pool.set_prefill_mode(mode)
        pool.prefill_attn(0, 0, q, k, v, f, out)          # warm-up (module load, attributes)
        torch.cuda.synchronize()
        ts = []
        for layer in range(1, n_layers + 1):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            pool.prefill_attn(layer, 0, q, k, v, f, out)
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        if pool.stats(check=False).error_flags:
            raise SystemExit("prefill attention set the device error word")
        return float(np.median(ts))

    ms = time_mode(dms.PREFILL_SPARSE)
    ms_dense = time_mode(dms.PREFILL_DENSE)
    fl = f.cpu().numpy()
    dense_tiles, sparse_tiles = prefill_tiles(fl, P, wl.window)
    tile_flops = 4.0 * D * 128 * 128
    flops = tile_flops * float(sparse_tiles.sum()) * g
    flops_dense = tile_flops * dense_tiles * Hq * B
    # visible (query, key) pairs: min(i + 1, w) + unflagged keys older than the window
    pairs = 0
    for b in range(B):
        for h in range(Hkv):
            unfl = np.concatenate([[0], np.cumsum(fl[b, :, h] == 0)])
            i = np.arange(P)
            pairs += int(np.sum(np.minimum(i + 1, wl.window) + unfl[np.maximum(i - wl.window + 1, 0)])) * g
    peak, kind = measured_bf16_tflops()
    tf = flops / (ms * 1e-3) / 1e12
    return {"value": tf, "unit": "TFLOP/s", "ms_per_layer": ms, "prompt": P,
            "roofline": {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s",
                         "frac": tf / peak, "peak_kind": kind},
            "flops_basis": "128x128 key tiles computed (QK^T and PV), per layer: prompt tiles from the "
                           "window band to the diagonal plus tiles of older kept keys read from the store",
            "tiles_per_layer": int(sparse_tiles.sum()) * g, "dense_tiles_per_layer": int(dense_tiles) * Hq * B,
            "visible_pair_tflops": 4.0 * D * pairs / (ms * 1e-3) / 1e12,
            "dense": {"ms_per_layer": ms_dense, "value": flops_dense / (ms_dense * 1e-3) / 1e12,
                      "frac": flops_dense / (ms_dense * 1e-3) / 1e12 / peak,
                      "mode": "every causal tile from the prompt, kept rows stored by the attention kernel"},
            "speedup_vs_dense": ms_dense / ms,
            "timing": "CUDA events around each layer's dms_prefill_attn call (compaction included), median",
            "kernel": (f"prefill_pair_kernel<{D}>" if g % 2 == 0 else f"prefill_attn_kernel<{D}>") +
                      " (tcgen05), old kept keys from the store"}


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read only)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks",
               0x1: "gpu_idle"}

    def __init__(self, index: int, period_s: float = 0.0002):
        self.samples, self.reasons = [], 0
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report no clocks rather than guess
            self.err = str(e)
        self.period = period_s
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(get_reasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "NVML unavailable"}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ---------------------------------------------------------------------------

def cpu_baseline(wl, t0: int, n_heads: int, n_steps: int, bytes_per_step: float):
    """Time the oracle (as it stands, one thread) on a sample of (head, step)
    pairs of the workload; scale to a whole step by the number of heads."""
    os.environ.setdefault("OMP_NUM_THREADS", "1")
    from oracle import attention as oatt
    from oracle import reference as oref
    from oracle import slots as oslots
    H = wl.n_layers * wl.batch * wl.n_kv_heads
    picks = []
    rng = np.random.Generator(np.random.PCG64(12345))
    for i in rng.choice(H, size=min(n_heads, H), replace=False):
        h = int(i % wl.n_kv_heads)
        b = int((i // wl.n_kv_heads) % wl.batch)
        layer = int(i // (wl.n_kv_heads * wl.batch))
        picks.append((layer, b, h))
    if wl.keep == "heavy_tail":
        # the sample always holds two keep-all heads (they dominate the bytes)
        full = [(int(l), 0, int(h)) for l, h in np.argwhere(wl.keep_probs() >= 1.0)[:2]]
        picks = full + [p for p in picks if p not in full][:max(0, len(picks) - len(full))]
    # untimed: inputs of each sampled head (flags, the rows it may see, queries)
    prep = []
    for (layer, b, h) in picks:
        T = t0 + n_steps
        flags = oref.head_flags(wl, layer, b, h, T)
        need = np.unique(np.concatenate([oracle_visible(t, flags, wl.window) for t in (t0, T - 1)]))
        need = np.unique(np.concatenate([need, np.arange(max(0, t0 - wl.window), T)]))
        K, V = oref.stored_rows(wl, layer, b, h, need,
                                oref.fp8_head_scales(wl, layer, h) if wl.kv_dtype == "fp8" else None)
        Kf = np.zeros((T, wl.head_dim))
        Vf = np.zeros((T, wl.head_dim))
        Kf[need], Vf[need] = K, V
        qs = [oref.head_query(wl, layer, b, h, t).astype(np.float64) for t in range(t0, T)]
        store = oslots.HeadStore(flags[:wl.prompt], wl.window)
        for t in range(wl.prompt, t0):
            store.append(t, int(flags[t]))
        prep.append((flags, Kf, Vf, qs, store))
    # timed: the oracle's decode step for each sampled head, step by step
    # (one step = every sampled head's step), and the bytes those heads hold
    row_bytes = 2 * wl.kv_row_bytes()
    sample_bytes = 0
    start = time.perf_counter()
    for s in range(n_steps):
        t = t0 + s
        for (flags, Kf, Vf, qs, store) in prep:
            store.append(t, int(flags[t]))
            oatt.decode_attention(qs[s], Kf[:t + 1, None, :], Vf[:t + 1, None, :], flags[:t + 1, None],
                                  t, wl.window)
            sample_bytes += store.n_retained * row_bytes
    elapsed = time.perf_counter() - start
    per_head_step = elapsed / (len(prep) * n_steps)
    step_time = per_head_step * H
    return {
        "value": bytes_per_step / step_time / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
        "sample": (f"{len(prep)} of {H} (layer, seq, kv-head) heads x {n_steps} decode steps from "
                   f"t={t0}: slot bookkeeping + fp64 masked attention per head, {elapsed:.1f} s; "
                   f"per-step time = mean head-step time x {H} heads"),
        "seconds": elapsed, "step_seconds_extrapolated": step_time,
        "sample_heads": len(prep), "sample_steps": n_steps, "sample_bytes": sample_bytes,
        "sample_value": sample_bytes / elapsed / 1e9,
        "compaction": oracle_compaction(wl, picks[:4 if wl.prompt <= 32768 else 1]),
    }


def oracle_compaction(wl, picks):
    """Time the oracle's prefill compaction (one thread) of the given heads:
    kept positions, slots and window ring, the kept K/V rows gathered (FP8:
    the head's maximum over its prompt rows and the kept rows quantised);
    scaled to a layer by its head count."""
    from oracle import compaction as ocomp
    from oracle import fp8 as ofp8
    from oracle import reference as oref
    prep = []
    for (layer, b, h) in picks:          # untimed: the head's inputs
        prep.append((oref.head_flags(wl, layer, b, h, wl.prompt),
                     oref.head_input(wl, 0, layer, b, h, 0, wl.prompt),
                     oref.head_input(wl, 1, layer, b, h, 0, wl.prompt)))
    in_row = 2 * wl.head_dim * (4 if wl.in_dtype == "f32" else 2)
    nbytes = 0
    start = time.perf_counter()
    for flags, K, V in prep:
        kept = ocomp.prefill_kept_positions(flags, wl.window)
        ocomp.prefill_slots(flags, wl.window)
        ocomp.prefill_ring(flags, wl.window)
        Kc, Vc = K[kept], V[kept]
        if wl.kv_dtype == "fp8":
            ofp8.quantize(Kc, ofp8.fp8_scale(np.abs(K).max()))
            ofp8.quantize(Vc, ofp8.fp8_scale(np.abs(V).max()))
            nbytes += wl.prompt * in_row
        nbytes += wl.prompt + len(kept) * (in_row + 2 * wl.kv_row_bytes())
    elapsed = time.perf_counter() - start
    heads_per_layer = wl.batch * wl.n_kv_heads
    per_head = elapsed / max(1, len(prep))
    return {"ms_per_layer": per_head * heads_per_layer * 1e3,
            "value": nbytes / elapsed / 1e9 if elapsed > 0 else None, "unit": "GB/s", "cores": 1,
            "sample": (f"{len(prep)} (sequence, kv-head) prompts of {wl.prompt} tokens, {elapsed:.2f} s; "
                       f"per-layer time = mean head time x {heads_per_layer} heads")}


def oracle_visible(t, flags, w):
    from oracle import mask
    return mask.visible_positions(t, flags, w)


def expected_bytes_per_step(wl):
    """Expected retained K/V bytes per step from the workload's keep probabilities."""
    p = wl.keep_probs()
    n = np.minimum(wl.prompt, wl.window) + p * max(0, wl.prompt - wl.window)
    return float(n.sum() * wl.batch * 2 * wl.kv_row_bytes())


# ---------------------------------------------------------------------------
# roofline helpers
# ---------------------------------------------------------------------------

def attn_source_hash() -> str:
    h = hashlib.sha256()
    for f in sorted(os.listdir(os.path.dirname(ATTN_KERNEL_SRC))):
        if f in ("attn.cu", "attn_warp.cuh", "step.cu", "dms_internal.cuh"):
            h.update(open(os.path.join(os.path.dirname(ATTN_KERNEL_SRC), f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic_ratio(workload: str):
    """DRAM bytes (read + write) per algorithmic byte of the attention kernel
    from the committed ncu summary of this workload, when it was taken on the
    current kernel source; else None.  The captured launch held fewer tokens
    than the timed ones, so traffic is scaled by held bytes (read traffic
    tracks them 1:1)."""
    for f in sorted(glob.glob(os.path.join(PROFILES, "decode_attn_*.md"))):
        txt = open(f).read()
        m_wl = re.search(r"^workload:\s*(\S+)", txt, re.M)
        m_src = re.search(r"kernel source hash:\s*([0-9a-f]+)", txt)
        m_tr = re.search(r"dram bytes per algorithmic byte:\s*([0-9.eE+]+)", txt)
        if m_wl and m_src and m_tr and m_wl.group(1) == workload and m_src.group(1) == attn_source_hash():
            return float(m_tr.group(1)), m_src.group(1)
    return None, None


# ---------------------------------------------------------------------------
# ranks
# ---------------------------------------------------------------------------

def reduce_over_ranks(ms: float, nbytes: float, device="cpu"):
    """(max of the device times, sum of the bytes) over all ranks of the
    default process group; (ms, nbytes) when not distributed.  Every rank
    makes the same two collective calls in the same order."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(ms), float(nbytes)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    b = torch.tensor([float(nbytes)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(b, op=dist.ReduceOp.SUM)
    return float(t.item()), float(b.item())


# ---------------------------------------------------------------------------
# the benchmark
# ---------------------------------------------------------------------------

def needs_l2_flush(wl) -> bool:
    """True when a step's held K/V (expected) fits in L2, so that timed steps
    must start after an L2 flush."""
    return expected_bytes_per_step(wl) <= L2_BYTES


def bench_config(wl, world: int) -> dict:
    """The `config` of a bench line (the same for both arms)."""
    held = expected_bytes_per_step(wl)
    l2 = (f"flush: {L2_FLUSH_BYTES >> 20} MB written then read before each timed step, outside its events "
          f"({held / 1e6:.0f} MB of held K/V per step fits in the 126 MB L2)" if needs_l2_flush(wl) else
          f"no flush: {held / 1e6:.0f} MB of held K/V read per step > 126 MB L2")
    return {"workload": wl.name, "layers": wl.n_layers, "batch": wl.batch, "q_heads": wl.n_q_heads,
            "kv_heads": wl.n_kv_heads, "head_dim": wl.head_dim, "prompt": wl.prompt, "window": wl.window,
            "kv_dtype": wl.kv_dtype, "seed": wl.seed, "parallelism": f"replicas x{world}", "l2": l2}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = with_kv_dtype(configs.BY_NAME[args.workload], args.kv_dtype)
    bps = expected_bytes_per_step(wl)
    steps = max(1, args.steps)
    n_heads = max(8, args.cpu_heads // 3)
    H = wl.n_layers * wl.batch * wl.n_kv_heads
    t0 = time.perf_counter()
    if args.warmup > 0:   # untimed warm-up steps of the same sample
        cpu_baseline(wl, wl.prompt, n_heads, min(args.warmup, 3), bps)
    cb = cpu_baseline(wl, wl.prompt + args.warmup, n_heads, steps, bps)
    wall = time.perf_counter() - t0
    line = {
        "impl": "reference", "metric": METRIC, "value": cb["sample_value"], "unit": "GB/s",
        "n_gpus": args.gpus, "steps": steps, "warmup": args.warmup,
        "ms_per_step": cb["seconds"] / steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(wl, args.gpus),
        "timing": (f"host wall clock around the {steps} timed steps; each step is the oracle's decode step of "
                   f"the same {cb['sample_heads']} sampled (layer, sequence, kv-head) heads of {H}, and the value "
                   f"is the K/V those heads hold over that time"),
        "sampled": {"heads": cb["sample_heads"], "of_heads": H, "steps": steps,
                    "ms_per_full_step_extrapolated": cb["step_seconds_extrapolated"] * 1e3,
                    "extrapolation": f"mean head-step time x {H} heads (not what was timed)"},
        "cpu_baseline": {k: cb[k] for k in ("unit", "cores", "kind", "sample", "compaction")} |
                        {"value": cb["sample_value"]},
        "e2e": {"value": cb["sample_value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "note": ("the reference arm is the CPU oracle (the pages ship no code), timed on a bounded sample "
                 "of each decode step"),
        "wall_s": wall,
    }
    print(json.dumps(line))
    return 0


def profile_case(wl, device):
    """Prefill, then steps 0-3 as all-layer steps (attention in one launch
    per step) and steps 4-5 as per-layer fused calls (append + attention in
    one launch per layer): the case the kernel captures under profiles/ use."""
    import torch
    from compact_decode_attention_b200.workload import DeviceWorkload
    dw = DeviceWorkload(wl, 6, device=device)
    dw.prefill()
    si, P, L = dw.step_inputs, wl.prompt, wl.n_layers
    for s in range(4):
        dw.step(s)
    for s in range(4, 6):
        for layer in range(L):
            sl = slice(layer, layer + 1)
            dw.pool.decode_step_layers(layer, P + s, si["k"][s][sl], si["v"][s][sl], si["evict"][s][sl],
                                       si["q"][s][sl], dw.out[sl])
    torch.cuda.synchronize()
    flags = dw.pool.stats().error_flags
    print(json.dumps({"profile_case": wl.name, "error_flags": flags}))
    return 0 if flags == 0 else 1


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist
    from compact_decode_attention_b200 import dms
    from compact_decode_attention_b200.workload import DeviceWorkload

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    numa = None if args.no_numa_bind else bind_to_gpu_numa_node(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    def barrier():
        if world > 1:
            dist.barrier()

    wl = with_kv_dtype(configs.BY_NAME[args.workload], args.kv_dtype)
    if args.projection_only:       # the fused projection measurement alone (one GPU)
        line = projection_line(wl, f"cuda:{local}")
        if rank == 0:
            print(json.dumps({"workload": wl.name, "kv_projection_append": line}))
        return 0
    if args.prefill_only:          # the prefill-attention measurement alone (one GPU)
        import dataclasses
        if args.prefill_prompt:
            wl = dataclasses.replace(wl, prompt=args.prefill_prompt)
        line = prefill_attention_line(wl, f"cuda:{local}")
        if rank == 0:
            print(json.dumps({"workload": wl.name, "prompt": wl.prompt, "prefill_attention": line}))
        return 0
    if args.profile_case:          # a short case for profiler captures (one GPU)
        return profile_case(wl, f"cuda:{local}")
    W, K, E = args.warmup, args.steps, args.e2e_steps
    R = min(K, 64)                 # instrumented steps for the attention-kernel timing
    RL = min(K, 16)                # steps issued as per-layer calls (each of the two forms)
    assert W >= 3 and K >= 1
    dw = DeviceWorkload(wl, W + K + R + 2 * RL + E, device=f"cuda:{local}")
    compact_ms_layers = dw.prefill(timed=True)
    # median layer: the first call of each kernel also pays its module load
    compact_ms = float(np.median(compact_ms_layers)) * len(compact_ms_layers)
    torch.cuda.synchronize()

    L, B, Hkv, D, w, P = wl.n_layers, wl.batch, wl.n_kv_heads, wl.head_dim, wl.window, wl.prompt
    H = L * B * Hkv
    row_bytes = 2 * wl.kv_row_bytes()                # K row + V row of one token

    # exact held tokens after each step: +1 per head, -1 per head whose token
    # t - w carried a flag (flags drawn by the same device generator)
    NT = W + K + R + 2 * RL + E
    fl = dw.flags(0, L, P - w, NT) if P - w >= 0 else None
    retired = fl.sum(dim=(0, 1, 3)).cpu().numpy().astype(np.int64) if fl is not None else \
        np.zeros(NT, np.int64)
    base = int(dw.pool.stats().retained_tokens)
    # compaction (prefill) bytes: flags + kept rows read in input precision and
    # written in the store's precision (+ every prompt row once more for the
    # FP8 scale pass)
    in_row = 2 * D * (4 if wl.in_dtype == "f32" else 2)
    compact_bytes = L * B * P * Hkv + base * (in_row + row_bytes)
    if wl.kv_dtype == "fp8":
        compact_bytes += L * B * P * Hkv * in_row
    # the same rate counted as if every prompt row were read (the full-read variant)
    full_read_bytes = L * B * P * Hkv * (1 + in_row) + base * row_bytes
    hbm_peak, hbm_kind = measured_peaks()
    compaction = {"value": compact_bytes / (compact_ms * 1e-3) / 1e9, "unit": "GB/s",
                  "frac": compact_bytes / (compact_ms * 1e-3) / 1e9 / hbm_peak,
                  "peak_kind": f"{hbm_kind} copy bandwidth",
                  "ms_per_layer": compact_ms / L, "algorithmic_bytes_per_layer": compact_bytes / L,
                  "full_read_value": full_read_bytes / (compact_ms * 1e-3) / 1e9,
                  "kernels": ("prefill_cluster_kernel (one launch a layer)"
                              if wl.kv_dtype in ("bf16", "f32") and P <= 16384 else
                              "prefill_plan_kernel + prefill_scatter_kernel (two launches a layer)"),
                  "timing": "CUDA events around each layer's dms_compact_prefill call, layers after "
                            "the first captured in one CUDA graph replayed once; median layer"}
    held = base + np.cumsum(H - retired)                  # after step s
    bytes_step = held.astype(np.float64) * row_bytes

    stream = torch.cuda.current_stream()
    for s in range(W):
        dw.step(s)
    torch.cuda.synchronize()

    # ---- device-timed region: exactly K steps, captured once into a CUDA graph
    # (so host issue time cannot leave the GPU idle between kernels) and
    # replayed once; positions advance every step, so each graph runs once ----
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    si = dw.step_inputs
    # a held K/V that fits in L2 would be read from L2 by the next step: then
    # every timed step starts after an L2 flush (a write of L2_FLUSH_BYTES,
    # then a read of it, so that no dirty line is left for the step to write
    # back), outside the event pair that times it, and the step times are summed
    flush = needs_l2_flush(wl)
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=f"cuda:{local}") if flush else None
    flush_sink = torch.empty((), dtype=torch.int32, device=f"cuda:{local}")

    def l2_flush(j):
        flush_buf.fill_(j & 0xff)
        torch.amax(flush_buf.view(torch.int32), dim=0, out=flush_sink)

    step_ev = [(torch.cuda.Event(enable_timing=True, external=True),
                torch.cuda.Event(enable_timing=True, external=True)) for _ in range(K if flush else 0)]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for j in range(K):
            s = W + j
            if flush:
                l2_flush(j)
                step_ev[j][0].record()
            dw.pool.append_evict_layers(0, P + s, si["k"][s], si["v"][s], si["evict"][s])
            dw.pool.decode_attn_layers(0, si["q"][s], dw.out)
            if flush:
                step_ev[j][1].record()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        barrier()
        torch.cuda.synchronize()
        t_start.record(stream)
        graph.replay()
        t_end.record(stream)
        torch.cuda.synchronize()
        barrier()
    ms = sum(a.elapsed_time(b) for a, b in step_ev) if flush else t_start.elapsed_time(t_end)
    del graph

    # ---- the attention kernel alone: a second graph of R steps with event
    # nodes around each attention launch (an event between the kernels stops
    # the programmatic overlap of append and attention, so the headline graph
    # above carries none) ----
    ev = [(torch.cuda.Event(enable_timing=True, external=True),
           torch.cuda.Event(enable_timing=True, external=True)) for _ in range(R)]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for j in range(R):
            s = W + K + j
            if flush:
                l2_flush(j)
            dw.pool.append_evict_layers(0, P + s, si["k"][s], si["v"][s], si["evict"][s])
            ev[j][0].record()
            dw.pool.decode_attn_layers(0, si["q"][s], dw.out)
            ev[j][1].record()
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()
    attn_ms = np.array([a.elapsed_time(b) for a, b in ev])
    del graph

    # ---- the same decode step as 2 L launches (append, then attention, one
    # layer per call), captured and replayed like the headline steps ----
    dw.pool.workspace(1, B, dw.out.device)   # allocated before the capture
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for j in range(RL):
            s = W + K + R + j
            for layer in range(L):
                dw.pool.append_evict_layers(layer, P + s, si["k"][s][layer:layer + 1],
                                            si["v"][s][layer:layer + 1], si["evict"][s][layer:layer + 1])
                dw.pool.decode_attn_layers(layer, si["q"][s][layer:layer + 1], dw.out[layer:layer + 1])
    torch.cuda.synchronize()
    pl0, pl1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pl0.record(stream)
    graph.replay()
    pl1.record(stream)
    torch.cuda.synchronize()
    pl_ms = pl0.elapsed_time(pl1) / RL
    del graph
    # ---- the same decode step as L fused calls (dms_decode_step_layers: the
    # append and the attention of one layer in one launch), layer after layer ----
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for j in range(RL):
            s = W + K + R + RL + j
            for layer in range(L):
                dw.pool.decode_step_layers(layer, P + s, si["k"][s][layer:layer + 1], si["v"][s][layer:layer + 1],
                                           si["evict"][s][layer:layer + 1], si["q"][s][layer:layer + 1],
                                           dw.out[layer:layer + 1])
    torch.cuda.synchronize()
    pf0, pf1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pf0.record(stream)
    graph.replay()
    pf1.record(stream)
    torch.cuda.synchronize()
    pf_ms = pf0.elapsed_time(pf1) / RL
    del graph
    fused_bytes = float(bytes_step[W + K + R + RL:W + K + R + 2 * RL].mean())
    per_layer_calls = {"ms_per_step": pl_ms, "decode_steps_per_s": 1e3 / pl_ms,
                       "value": float(bytes_step[W + K + R:W + K + R + RL].mean()) / (pl_ms * 1e-3) / 1e9,
                       "unit": "GB/s", "launches_per_step": 2 * L, "steps": RL,
                       "timing": "CUDA events around one replay of a captured graph of the steps, "
                                 "each step one append and one attention call per layer",
                       "fused_step": {"ms_per_step": pf_ms, "decode_steps_per_s": 1e3 / pf_ms,
                                      "value": fused_bytes / (pf_ms * 1e-3) / 1e9, "unit": "GB/s",
                                      "frac": fused_bytes / (pf_ms * 1e-3) / 1e9 / measured_peaks()[0],
                                      "launches_per_step": L, "steps": RL,
                                      "call": "dms_decode_step_layers, one layer per call (append/evict and "
                                              "attention in one launch: decode_cluster_kernel)"}}
    st = dw.pool.stats()
    if st.error_flags:
        raise SystemExit(f"device error word 0x{st.error_flags:x}")

    my_bytes = float(bytes_step[W:W + K].sum())
    ms_max, total_bytes = reduce_over_ranks(ms, my_bytes, device=f"cuda:{local}")
    value = total_bytes / (ms_max * 1e-3) / 1e9

    # ---- roofline of the attention kernel ----
    plan_kind, plan_c = dms.dms_decode_attn_plan(dw.pool.handle, L, B)
    attn_kernel_name = (f"decode_cluster_kernel<{wl.kv_dtype},{D}> ({plan_c} CTAs per head)"
                        if plan_kind == dms.ATTN_CLUSTER else f"decode_attn_kernel<{wl.kv_dtype},{D}> (stream-K)")
    peak, peak_kind = measured_peaks()
    rbytes = bytes_step[W + K:W + K + R]
    achieved = float(rbytes.sum() / (attn_ms.sum() * 1e-3) / 1e9)
    ratio, _ = profiled_traffic_ratio(wl.name)
    traffic = None if ratio is None else ratio * float(rbytes.mean())
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": traffic,
                "kernel": attn_kernel_name,
                "peak_kind": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback 6.65 TB/s",
                "algorithmic_bytes_per_launch": float(rbytes.mean()),
                "attn_us_per_launch": float(attn_ms.mean() * 1e3),
                "timed_launches": R, "timing": "CUDA event nodes around each attention launch in "
                                                "a captured graph of R steps, replayed once"}

    # ---- end to end through the C ABI from host memory: dms_stepper_step per
    # step (packed pinned input -> device, append/evict, attention, output ->
    # pinned host), copies inside the timed region ----
    e2e = None
    if E > 0:
        e0s = W + K + R + 2 * RL
        stp = dms.Stepper(dw.pool, 0, L, B, stream=stream)
        hin = stp.host_inputs(E)
        hout = torch.empty(E, stp.layout.out_bytes, dtype=torch.uint8).pin_memory()
        for j in range(E):
            s = e0s + j
            stp.pack(hin[j], si["k"][s], si["v"][s], si["q"][s], si["evict"][s])
        flush_ms = 0.0
        if flush:      # the flushes alone, subtracted from the timed loop below
            f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            f0.record(stream)
            for j in range(E):
                l2_flush(j)
            f1.record(stream)
            torch.cuda.synchronize()
            flush_ms = f0.elapsed_time(f1)
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        h0 = time.perf_counter()
        for j in range(E):
            if flush:
                l2_flush(j)
            stp.step(P + e0s + j, hin[j], hout[j])
        host_issue_s = time.perf_counter() - h0
        stp.join(stream)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e_ms, e_bytes = reduce_over_ranks(e0.elapsed_time(e1) - flush_ms, float(bytes_step[e0s:e0s + E].sum()),
                                          device=f"cuda:{local}")
        e2e = {"value": e_bytes / (e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": int(stp.layout.in_bytes), "d2h_bytes_per_step": int(stp.layout.out_bytes),
               "steps": E, "ms_per_step": e_ms / E,
               "host_cpus": numa or "not bound",
               "host_issue_us_per_step": host_issue_s / E * 1e6,
               "path": "dms_stepper_step: one packed pinned-host input copy, append/evict, decode "
                       "attention, one pinned-host output copy per step; copies on their own streams, "
                       "four buffers deep against the neighbouring steps' kernels"}
        if flush:
            e2e["l2"] = (f"an L2 flush ({L2_FLUSH_BYTES >> 20} MB written then read) on the compute stream before each "
                         f"step; their time alone ({flush_ms / E * 1e3:.1f} us per flush) is subtracted")
        stp.close()

    prefill = prefill_attention_line(wl, f"cuda:{local}") if not args.no_prefill else None
    projection = projection_line(wl, f"cuda:{local}") if not args.no_prefill else None

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, P + W, args.cpu_heads, args.cpu_steps, float(bytes_step[W]))
        cpu = {k: cpu[k] for k in ("value", "unit", "cores", "kind", "sample", "compaction")}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": W,
            "ms_per_step": ms_max / K,
            "timing": ("sum of CUDA event pairs around each step in one replay of a captured graph of "
                       "the K steps (an L2 flush between steps, outside the pairs)" if flush else
                       "CUDA events around one replay of a captured graph of the K steps"), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if wl.kv_dtype == "bf16" else wl.kv_dtype, "data": "synthetic",
            "config": bench_config(wl, world),
            "decode_steps_per_s": world * K / (ms_max * 1e-3),
            "per_layer_calls": per_layer_calls,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "compaction": compaction,
            "prefill_attention": prefill, "kv_projection_append": projection,
            "gpu_launches": 2 * K, "clocks": clk.summary(),
            "kernels_per_step": ["append_evict_kernel (1 launch, all layers)",
                                 f"{attn_kernel_name} (1 launch, all layers)"],
            "pool": {"blocks_in_use": int(st.blocks_in_use), "kv_bytes_in_use": int(st.kv_bytes_in_use),
                     "retained_tokens": int(st.retained_tokens),
                     "min_retained": int(st.min_retained), "max_retained": int(st.max_retained)},
        }
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
