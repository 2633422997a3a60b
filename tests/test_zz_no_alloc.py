"""dms_decode_attn_layers_noalloc: decode attention for callers that cannot
allocate device memory (an engine that has given all free HBM to its KV pool,
a plugin with no allocator, a path that must not pay cudaMalloc's
synchronisation).  Its split-K scratch is a fixed array inside the library.

These tests call it through the C ABI and compare it with the entry point
that takes a caller workspace.  The file is named so that pytest collects it
last; it builds its own pool, so it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import synth
from compact_decode_attention_b200 import dms

pytestmark = pytest.mark.gpu

TOL_BF16 = 2e-2


def _filled_pool(B=2, Hq=16, Hkv=4, D=128, P=3000, w=128, seed=77):
    """A pool holding one bf16 layer after prefill and one decode step."""
    K = synth.kv_tokens(seed, 0, 0, B, 0, P + 1, Hkv, D, "bf16")
    V = synth.kv_tokens(seed, 1, 0, B, 0, P + 1, Hkv, D, "bf16")
    flags = synth.flag_tokens(seed, 0, B, 0, P + 1, Hkv, [synth.keep_threshold(0.3)] * Hkv)
    pool = dms.Pool(1, B, Hq, Hkv, D, w, dms.DMS_BF16, 4 * B * Hkv * ((P + 64) // 64), P + 2)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).cuda()  # noqa: E731
    pool.compact_prefill(0, dev(K[:, :P]), dev(V[:, :P]), torch.from_numpy(flags[:, :P].copy()).cuda())
    pool.append_evict_layers(0, P, dev(K[None, :, P]), dev(V[None, :, P]),
                             torch.from_numpy(flags[None, :, P].copy()).cuda())
    q = dev(synth.q_tokens(seed, 0, B, P, Hq, D, "bf16")[None])
    return pool, q


def test_noalloc_matches_workspace_entry_on_two_calls():
    pool, q = _filled_pool()
    stream = torch.cuda.current_stream().cuda_stream
    ref = torch.empty_like(q)
    ws = pool.workspace(1, q.shape[1])
    dms.dms_decode_attn_layers(pool.handle, 0, 1, q.shape[1], q.data_ptr(), dms.DMS_BF16,
                               ref.data_ptr(), 0.0, ws.data_ptr(), ws.numel(), stream)
    outs = []
    for _ in range(2):   # the second call reuses scratch the first one left behind
        out = torch.full_like(q, float("nan"))
        dms.dms_decode_attn_layers_noalloc(pool.handle, 0, 1, q.shape[1], q.data_ptr(), dms.DMS_BF16,
                                           out.data_ptr(), 0.0, stream)
        outs.append(out.float().cpu().numpy())
    r = ref.float().cpu().numpy()
    for o in outs:
        assert np.isfinite(o).all()
        assert np.abs(o - r).max() < TOL_BF16
    assert pool.stats().error_flags == 0


def test_noalloc_rejects_calls_larger_than_its_scratch():
    # 64 layers x 8 sequences x 8 kv-heads, g = 8, D = 128 needs ~18 MB of scratch
    pool = dms.Pool(64, 8, 64, 8, 128, 16, dms.DMS_BF16, 8, 64)
    q = torch.zeros(64, 8, 64, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    with pytest.raises(dms.DmsError) as e:
        dms.dms_decode_attn_layers_noalloc(pool.handle, 0, 64, 8, q.data_ptr(), dms.DMS_BF16,
                                           out.data_ptr(), 0.0, torch.cuda.current_stream().cuda_stream)
    assert e.value.status == dms.DMS_ERR_CAPACITY
    assert "fixed workspace" in str(e.value)
