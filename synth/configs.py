"""The five synthetic workloads, named by what they are.

Shapes follow the attention geometry of Llama-3.2-1B (16 layers, 32 query /
8 KV heads, head_dim 64) and Qwen3-8B (36 layers, 32 / 8, head_dim 128); the
context lengths follow the pages' ctx_len=8192 / gen_len=128 benchmark
setting and Qwen3-8B's 131072-token YaRN context.  The 512-token delay window
is the DMS default of the Qwen3-8B-DMS-8x model card.

Per-head keep probabilities are host draws from ``numpy.random.Generator(
PCG64(seed))``; they become 24-bit thresholds (``synth.keep_threshold``) that
both the oracle and the device generator read as an input array.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import keep_threshold


@dataclass(frozen=True)
class Workload:
    name: str
    n_layers: int
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    prompt: int
    decode: int
    window: int
    kv_dtype: str          # storage dtype in the pool: "f32" | "bf16" | "fp8" | "int4"
    in_dtype: str          # dtype of the K/V/Q the model hands over: "f32" | "bf16"
    seed: int
    keep: str              # "const" | "uniform" | "heavy_tail"
    p_keep: float = 0.0
    extra: dict = field(default_factory=dict)

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def keep_probs(self) -> np.ndarray:
        """float64 [n_layers, n_kv_heads] keep probability per (layer, kv-head).

        The draw is shared by every sequence of the batch."""
        L, H = self.n_layers, self.n_kv_heads
        if self.keep == "const":
            return np.full((L, H), self.p_keep, dtype=np.float64)
        rng = np.random.Generator(np.random.PCG64(self.seed))
        if self.keep == "uniform":
            lo, hi = self.extra["lo"], self.extra["hi"]
            return rng.uniform(lo, hi, size=(L, H))
        if self.keep == "heavy_tail":
            n = L * H
            n_all = int(round(self.extra["frac_keep_all"] * n))
            keep_all = rng.choice(n, size=n_all, replace=False)
            p = rng.beta(self.extra["a"], self.extra["b"], size=n)
            p[keep_all] = 1.0
            return p.reshape(L, H)
        raise ValueError(self.keep)

    def thresholds(self) -> np.ndarray:
        """int64 [n_layers, n_kv_heads] 24-bit keep thresholds."""
        return keep_threshold(self.keep_probs())

    def kv_row_bytes(self) -> int:
        """Bytes of one stored K (or V) row: 4-bit rows carry 4 bits per
        element plus one fp16 scale per group of 32."""
        if self.kv_dtype == "int4":
            return self.head_dim // 2 + self.head_dim // 16
        return self.head_dim * {"f32": 4, "bf16": 2, "fp8": 1}[self.kv_dtype]

    def in_elem_bytes(self) -> int:
        return {"f32": 4, "bf16": 2}[self.in_dtype]


TINY_FP32 = Workload("tiny_fp32_l1_b1_h4x2_d64_p256_s16_w32", 1, 1, 4, 2, 64, 256, 16, 32,
                     "f32", "f32", 0, "const", p_keep=0.15)
LLAMA1B_CTX8K = Workload("llama3.2-1b_l16_b1_ctx8192_s128_w512_bf16", 16, 1, 32, 8, 64, 8192, 128,
                         512, "bf16", "bf16", 1, "const", p_keep=0.10)
QWEN8B_CTX8K = Workload("qwen3-8b_l36_b1_ctx8192_s128_w512_bf16", 36, 1, 32, 8, 128, 8192, 128,
                        512, "bf16", "bf16", 2, "uniform", extra={"lo": 0.02, "hi": 0.30})
QWEN8B_FP8_B8_CTX32K = Workload("qwen3-8b_l36_b8_ctx32768_s256_w512_fp8e4m3", 36, 8, 32, 8, 128,
                                32768, 256, 512, "fp8", "bf16", 3, "const", p_keep=0.067)
QWEN8B_B16_CTX128K = Workload("qwen3-8b_l36_b16_ctx131072_s1024_w512_bf16_stress", 36, 16, 32, 8,
                              128, 131072, 1024, 512, "bf16", "bf16", 4, "heavy_tail",
                              extra={"frac_keep_all": 0.10, "a": 0.5, "b": 8.0})

ALL = [TINY_FP32, LLAMA1B_CTX8K, QWEN8B_CTX8K, QWEN8B_FP8_B8_CTX32K, QWEN8B_B16_CTX128K]
BY_NAME = {w.name: w for w in ALL}
