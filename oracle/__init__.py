"""CPU oracle for compact-KV DMS decode: TEST INFRASTRUCTURE ONLY.

Plain, slow, fp64 NumPy restatement of what the hot path computes, written
from the pages' description of Dynamic Memory Sparsification (DMS) and
FastDMS.  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline may import it; the product path (the CUDA library and its Python
binding) never does, and it imports nothing from the product.  Its inputs
come from the seeded generator in ``synth`` (which holds no method
arithmetic).

Sources (page title and section):

* "NVIDIA veröffentlicht Qwen3-8B-DMS-8x mit innovativer Speicherkompression
  für verbesserte Inferenzzeiten" (mindverse), section "Dynamic Memory
  Sparsification (DMS): Eine innovative Lösung": per-head eviction policies
  that interpolate between a sliding window over the last 512 tokens and
  full attention; delayed eviction keeps a flagged token for a while.
* "Nvidia DMS: сжатие памяти LLM в 8 раз — модели думают лучше" (stiva.ai),
  section "Ключевое изобретение: delayed eviction": a flagged token remains
  available for further steps and is removed afterwards.
* "FastDMS: vLLM BF16/FP8보다 빠른 6.4x KV cache 압축" (molayo1419.me),
  opening paragraphs: FastDMS is DMS with a compact KV store that reclaims
  physically evicted slots; the FP8 paragraph after the speed table:
  eviction is decided before FP8 quantisation; table "What's the catch?",
  row "PagedAttention / KV memory pool": per-layer, per-head variable token
  counts with partial block release.

Modules:
  mask        visibility rule of delayed eviction
  attention   dense fp64 masked GQA decode attention
  compaction  reference prefill compaction and window ring
  slots       per-step slot bookkeeping simulator (retire, reclaim, append)
  fp8         software FP8-E4M3 codec and per-head scale
  reference   per-head expected values for a seeded workload

Every function here is pinned by a ``-m "not gpu"`` test against something
other than itself (closed forms, library routines, brute force, page
figures): the per-head glue of ``reference`` (flags, inputs, query rows,
FP8 scales, stored rows, expected outputs) against whole tensors drawn from
the generator, torch's fp64 scaled_dot_product_attention under the
operational eviction mask and torch's float8 cast, for every (layer,
sequence, kv-head) of a small workload; none is "parity unpinned".
"""
