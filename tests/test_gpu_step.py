"""The fused decode step (dms_decode_step_layers) and the cluster attention
kernel, through the C ABI, against the fp64 oracle.

A fused step must leave the store exactly as dms_append_evict does
(bookkeeping and stored bytes bit-exact against the oracle's slot simulator)
and return the attention over exactly the rows the two separate calls would
see, within the attention tolerances: 1e-5 (fp32 store), 2e-2 (bf16),
6e-2 (FP8 and 4-bit).  The cases cover retired slots reused by the new token
(the masked hole), new slots and new blocks, windows of one token, every
token flagged and none, every store and input dtype, heads long enough that a
CTA of a cluster runs more blocks than it has stages and more than 32
block-table entries, and the cluster kernel forced onto calls with more
heads than fit (clusters of one CTA in waves)."""
import numpy as np
import pytest
import torch

import synth
from oracle import attention as oatt
from oracle import fp8 as ofp8
from oracle import int4 as oint4
from compact_decode_attention_b200 import dms

from gpu_util import check_block_invariants, check_head_store, head_id, int4_rows, oracle_store, read_state

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-2, "fp8": 6e-2, "int4": 6e-2}
CODE = {"f32": dms.DMS_F32, "bf16": dms.DMS_BF16, "fp8": dms.DMS_FP8_E4M3, "int4": dms.DMS_INT4}


def _inputs(seed, L, B, P, S, Hq, Hkv, D, in_kind, p_keep=0.3, flags=None):
    """K, V [L, B, P+S, Hkv, D], flags [L, B, P+S, Hkv], Q [S, L, B, Hq, D] (fp32 arrays in input precision)."""
    K = np.stack([synth.kv_tokens(seed, 0, l, B, 0, P + S, Hkv, D, in_kind) for l in range(L)])
    V = np.stack([synth.kv_tokens(seed, 1, l, B, 0, P + S, Hkv, D, in_kind) for l in range(L)])
    if flags is None:
        flags = np.stack([synth.flag_tokens(seed, l, B, 0, P + S, Hkv, [synth.keep_threshold(p_keep)] * Hkv)
                          for l in range(L)])
    qk = "f32" if in_kind == "f32" else "bf16"
    Q = np.stack([np.stack([synth.q_tokens(seed, l, B, P + s, Hq, D, qk) for l in range(L)]) for s in range(S)]) \
        if S else np.zeros((0, L, B, Hq, D), np.float32)
    return K, V, flags, Q


def _stored_values(K, V, P, kind):
    """Values the store holds for every position (fp64), with the FP8 scales
    of each (layer, kv-head) taken over the prompt rows of every sequence."""
    if kind in ("f32", "bf16"):
        return K.astype(np.float64), V.astype(np.float64), None
    if kind == "int4":
        return oint4.stored(K), oint4.stored(V), None
    L, B, T, Hkv, D = K.shape
    Ks, Vs = np.empty(K.shape), np.empty(V.shape)
    scales = {}
    for l in range(L):
        for h in range(Hkv):
            sk = ofp8.fp8_scale(np.abs(K[l, :, :P, h]).max())
            sv = ofp8.fp8_scale(np.abs(V[l, :, :P, h]).max())
            scales[(l, h)] = (sk, sv)
            Ks[l, :, :, h] = ofp8.dequantize(ofp8.quantize(K[l, :, :, h], sk), sk)
            Vs[l, :, :, h] = ofp8.dequantize(ofp8.quantize(V[l, :, :, h], sv), sv)
    return Ks, Vs, scales


def _run_steps(kind, in_kind, L, B, Hq, Hkv, D, P, S, w, seed, p_keep=0.3, flags=None, attn=dms.ATTN_AUTO,
               per_layer=False):
    K, V, F, Q = _inputs(seed, L, B, P, S, Hq, Hkv, D, in_kind, p_keep, flags)
    T = P + S
    pool = dms.Pool(L, B, Hq, Hkv, D, w, CODE[kind], L * B * Hkv * ((T + 63) // 64 + 1), T + 1)
    pool.set_attn_kernel(attn)
    dt = torch.float32 if in_kind == "f32" else torch.bfloat16
    qdt = torch.float32 if kind == "f32" else torch.bfloat16
    dev = lambda a, t=dt: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(t).cuda()  # noqa: E731
    if P > 0:
        for l in range(L):
            pool.compact_prefill(l, dev(K[l, :, :P]), dev(V[l, :, :P]),
                                 torch.from_numpy(np.ascontiguousarray(F[l, :, :P])).cuda())
    Ks, Vs, scales = _stored_values(K, V, P, kind)
    worst = 0.0
    for s in range(S):
        t = P + s
        k1, v1 = dev(K[:, :, t]), dev(V[:, :, t])
        f1 = torch.from_numpy(np.ascontiguousarray(F[:, :, t])).cuda()
        q1 = dev(Q[s], qdt)
        out = torch.full((L, B, Hq, D), float("nan"), dtype=qdt, device="cuda")
        if per_layer:
            for l in range(L):
                pool.decode_step_layers(l, t, k1[l:l + 1], v1[l:l + 1], f1[l:l + 1], q1[l:l + 1], out[l:l + 1])
        else:
            pool.decode_step_layers(0, t, k1, v1, f1, q1, out)
        got = out.float().cpu().numpy()
        for l in range(L):
            for b in range(B):
                exp = oatt.decode_attention(Q[s, l, b].astype(np.float64), Ks[l, b, :t + 1], Vs[l, b, :t + 1],
                                            F[l, b, :t + 1], t, w)
                err = np.abs(got[l, b] - exp).max()
                worst = max(worst, err)
                assert err < TOL[kind], (kind, s, l, b, err)
    # the store after the last step, bit-exact against the slot simulator
    state = read_state(pool)
    assert state["error"] == 0
    for l in range(L):
        for b in range(B):
            for h in range(Hkv):
                store = oracle_store(F[l, b, :P, h], F[l, b, P:, h], w, P)
                hd = head_id(pool.cfg, l, b, h)
                if kind == "int4":
                    assert state["n_slots"][hd] == store.n_slots and state["n_retained"][hd] == store.n_retained
                    pos = np.array([store.pos_of_slot[x] for x in range(store.n_slots)])
                    ck, sk, cv, sv = int4_rows(pool, state, hd, store.n_slots)
                    qk, ek = oint4.quantize(K[l, b, pos, h])
                    qv, ev = oint4.quantize(V[l, b, pos, h])
                    assert np.array_equal(ck, qk) and np.array_equal(sk, ek), (l, b, h)
                    assert np.array_equal(cv, qv) and np.array_equal(sv, ev), (l, b, h)
                else:
                    check_head_store(pool, state, hd, store, {j: K[l, b, j, h] for j in range(T)},
                                     {j: V[l, b, j, h] for j in range(T)}, kind,
                                     None if scales is None else scales[(l, h)])
    check_block_invariants(pool, state)
    assert pool.stats().error_flags == 0
    return worst


@pytest.mark.parametrize("kind,in_kind,D,g", [
    ("bf16", "bf16", 128, 4), ("bf16", "bf16", 64, 4), ("bf16", "bf16", 128, 8), ("bf16", "bf16", 64, 1),
    ("fp8", "bf16", 128, 4), ("fp8", "f32", 128, 4), ("int4", "bf16", 128, 4), ("int4", "f32", 128, 2),
    ("f32", "f32", 64, 2), ("f32", "f32", 128, 4)])
def test_fused_step_every_head_every_step(kind, in_kind, D, g):
    """Two layers in one call, ragged prompts over several blocks, 70 steps
    with w = 100: retired slots reused (holes) and new slots and blocks."""
    Hkv = 3
    _run_steps(kind, in_kind, 2, 2, Hkv * g, Hkv, D, 700, 70, 100, seed=101 + D + g)


@pytest.mark.parametrize("P,w,S,pattern", [(20, 64, 60, None), (1, 8, 30, None), (130, 1, 20, None),
                                           (300, 32, 40, "all"), (300, 32, 40, "none"), (64, 16, 70, None)])
def test_fused_step_edges(P, w, S, pattern):
    """Prompts shorter than the window, one-token prompts, w = 1 (every step
    reuses the previous token's slot when it was flagged), every token
    flagged (a pure sliding window: every step reuses a slot), none flagged
    (every step takes a new slot), a prompt ending on a block edge."""
    B, Hkv, L = 2, 2, 1
    flags = None
    if pattern is not None:
        flags = np.full((L, B, P + S, Hkv), 1 if pattern == "all" else 0, np.uint8)
    _run_steps("bf16", "bf16", L, B, 8, Hkv, 64, P, S, w, seed=7 + P + w, p_keep=0.2, flags=flags)


def test_fused_step_per_layer_calls():
    """The form a model issues: one call per layer, layer after layer."""
    _run_steps("bf16", "bf16", 4, 1, 16, 4, 128, 900, 20, 64, seed=55, per_layer=True)


def test_fused_step_falls_back_to_two_kernels_for_many_heads():
    """Too many heads for one resident cluster each (the stream-K kernel and
    the append kernel run), and the same forced onto stream-K."""
    _run_steps("bf16", "bf16", 1, 48, 16, 4, 64, 150, 6, 32, seed=56)
    _run_steps("bf16", "bf16", 1, 2, 8, 2, 128, 400, 10, 32, seed=57, attn=dms.ATTN_STREAM_K)


def _attn_paths(B, Hkv, g, D, P, w, flags, seed):
    """One decode step's attention by the cluster and by the stream-K kernel,
    and the oracle's."""
    K, V, F, Q = _inputs(seed, 1, B, P + 1, 0, Hkv * g, Hkv, D, "bf16", flags=flags)
    Q = synth.q_tokens(seed, 0, B, P, Hkv * g, D, "bf16")
    pool = dms.Pool(1, B, Hkv * g, Hkv, D, w, dms.DMS_BF16, B * Hkv * ((P + 64) // 64 + 1), P + 2)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).cuda()  # noqa: E731
    pool.compact_prefill(0, dev(K[0, :, :P]), dev(V[0, :, :P]), torch.from_numpy(np.ascontiguousarray(F[0, :, :P])).cuda())
    pool.append_evict_layers(0, P, dev(K[:, :, P]), dev(V[:, :, P]), torch.from_numpy(np.ascontiguousarray(F[:, :, P])).cuda())
    outs = {}
    for kind in (dms.ATTN_CLUSTER, dms.ATTN_STREAM_K):
        pool.set_attn_kernel(kind)
        out = torch.full((1, B, Hkv * g, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        pool.decode_attn_layers(0, dev(Q[None]), out)
        outs[kind] = out[0].float().cpu().numpy()
    exp = np.stack([oatt.decode_attention(Q[b].astype(np.float64), K[0, b, :P + 1], V[0, b, :P + 1],
                                          F[0, b, :P + 1], P, w) for b in range(B)])
    assert pool.stats().error_flags == 0
    return outs, exp


@pytest.mark.parametrize("B,Hkv,P,keep_all_head", [(1, 2, 40000, 0), (1, 4, 20000, 1), (30, 8, 300, None)])
def test_cluster_and_stream_k_kernels_agree(B, Hkv, P, keep_all_head):
    """A head of 625 blocks (39 per CTA of a 16-CTA cluster: more than its
    stages and than one batch of 32 block-table entries) next to short ones,
    and 240 heads with the cluster kernel forced (clusters of one CTA)."""
    flags = None
    if keep_all_head is not None:
        flags = np.ones((1, B, P + 1, Hkv), np.uint8)
        flags[:, :, :, keep_all_head] = 0
    outs, exp = _attn_paths(B, Hkv, 4, 128, P, 16, flags, seed=88 + P)
    for kind, got in outs.items():
        assert np.abs(got - exp).max() < TOL["bf16"], kind


def test_cluster_attention_of_an_empty_sequence_is_zero():
    """A sequence with nothing held (never prefilled) next to a filled one:
    its outputs are zero, like the stream-K kernel's."""
    B, Hkv, g, D, P, w = 2, 2, 4, 64, 300, 32
    K, V, F, _ = _inputs(9, 1, 1, P, 0, Hkv * g, Hkv, D, "bf16")
    pool = dms.Pool(1, B, Hkv * g, Hkv, D, w, dms.DMS_BF16, 64, P + 2)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).cuda()  # noqa: E731
    pool.compact_prefill_seqs(0, 0, dev(K[0]), dev(V[0]), torch.from_numpy(np.ascontiguousarray(F[0])).cuda())
    Q = synth.q_tokens(9, 0, B, P - 1, Hkv * g, D, "bf16")
    for kind in (dms.ATTN_CLUSTER, dms.ATTN_STREAM_K):
        pool.set_attn_kernel(kind)
        out = torch.full((1, B, Hkv * g, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        pool.decode_attn_layers(0, dev(Q[None]), out)
        got = out[0].float().cpu().numpy()
        assert np.all(got[1] == 0), kind
        exp = oatt.decode_attention(Q[0].astype(np.float64), K[0, 0], V[0, 0], F[0, 0], P - 1, w)
        assert np.abs(got[0] - exp).max() < TOL["bf16"], kind


def test_attn_kernel_setting_is_checked():
    pool = dms.Pool(1, 1, 4, 2, 64, 16, dms.DMS_BF16, 8, 64)
    with pytest.raises(dms.DmsError) as e:
        pool.set_attn_kernel(7)
    assert e.value.status == dms.DMS_ERR_INVALID_ARG
