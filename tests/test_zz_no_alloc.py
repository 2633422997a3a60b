"""dms_decode_attn_layers_noalloc: decode attention for callers that cannot
allocate device memory (an engine that has given all free HBM to its KV pool,
a plugin with no allocator, a path that must not pay cudaMalloc's
synchronisation).  Its split-K scratch is a fixed array inside the library.

These tests call it through the C ABI and compare it with the entry point
that takes a caller workspace: the same kernel runs on the same inputs and
merges split partials in a fixed order, so the outputs must be identical bit
for bit, on two calls in a row (the second finds the first call's partials
in the shared array).  Both are also checked against the fp64 oracle.  The
file is named so that pytest collects it last; it builds its own pools, so it
also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import attention as oatt
from oracle import fp8 as ofp8
from compact_decode_attention_b200 import dms

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-2, "fp8": 6e-2}
CODE = {"f32": dms.DMS_F32, "bf16": dms.DMS_BF16, "fp8": dms.DMS_FP8_E4M3}


def _filled_pool(kind, L, B=2, Hq=16, Hkv=4, D=128, P=3000, w=128, seed=77):
    """A pool holding L layers after prefill and one decode step, its query,
    and the oracle's outputs [L, B, Hq, D]."""
    in_kind = "f32" if kind == "f32" else "bf16"
    dt = torch.float32 if in_kind == "f32" else torch.bfloat16
    pool = dms.Pool(L, B, Hq, Hkv, D, w, CODE[kind], 4 * L * B * Hkv * ((P + 64) // 64), P + 2)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dt).cuda()  # noqa: E731
    ks, vs, fs, qs, exp = [], [], [], [], np.zeros((L, B, Hq, D))
    for layer in range(L):
        K = synth.kv_tokens(seed, 0, layer, B, 0, P + 1, Hkv, D, in_kind)
        V = synth.kv_tokens(seed, 1, layer, B, 0, P + 1, Hkv, D, in_kind)
        F = synth.flag_tokens(seed, layer, B, 0, P + 1, Hkv, [synth.keep_threshold(0.3)] * Hkv)
        Q = synth.q_tokens(seed, layer, B, P, Hq, D, in_kind)
        pool.compact_prefill(layer, dev(K[:, :P]), dev(V[:, :P]), torch.from_numpy(F[:, :P].copy()).cuda())
        ks.append(K[:, P])
        vs.append(V[:, P])
        fs.append(F[:, P])
        qs.append(Q)
        Ks, Vs = K.astype(np.float64), V.astype(np.float64)
        if kind == "fp8":
            for h in range(Hkv):
                sk, sv = ofp8.fp8_scale(np.abs(K[:, :P, h]).max()), ofp8.fp8_scale(np.abs(V[:, :P, h]).max())
                Ks[:, :, h] = ofp8.dequantize(ofp8.quantize(K[:, :, h], sk), sk)
                Vs[:, :, h] = ofp8.dequantize(ofp8.quantize(V[:, :, h], sv), sv)
        for b in range(B):
            exp[layer, b] = oatt.decode_attention(Q[b].astype(np.float64), Ks[b], Vs[b], F[b], P, w)
    pool.append_evict_layers(0, P, dev(np.stack(ks)), dev(np.stack(vs)),
                             torch.from_numpy(np.ascontiguousarray(np.stack(fs))).cuda())
    return pool, dev(np.stack(qs)), exp


@pytest.mark.parametrize("kind,L", [("bf16", 1), ("bf16", 3), ("fp8", 2), ("f32", 1)])
def test_noalloc_matches_workspace_entry_on_two_calls(kind, L):
    pool, q, exp = _filled_pool(kind, L)
    B = q.shape[1]
    code = dms.DMS_F32 if kind == "f32" else dms.DMS_BF16
    stream = torch.cuda.current_stream().cuda_stream
    ref = torch.empty_like(q)
    ws = pool.workspace(L, B)
    dms.dms_decode_attn_layers(pool.handle, 0, L, B, q.data_ptr(), code, ref.data_ptr(), 0.0,
                               ws.data_ptr(), ws.numel(), stream)
    for call in range(2):   # the second call reuses scratch the first one left behind
        out = torch.full_like(q, float("nan"))
        dms.dms_decode_attn_layers_noalloc(pool.handle, 0, L, B, q.data_ptr(), code, out.data_ptr(),
                                           0.0, stream)
        torch.cuda.synchronize()
        assert torch.equal(out, ref), f"call {call}: differs from the workspace entry point"
        assert np.abs(out.float().cpu().numpy() - exp).max() < TOL[kind]
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
