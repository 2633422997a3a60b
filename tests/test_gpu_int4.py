"""4-bit K/V store (DMS_INT4): compaction, append and decode attention
against the oracle, through the C ABI.

Stored codes and group scales must equal the oracle's quantisation of the
rows the slot simulator says are held (bit-exact, like all bookkeeping);
attention over the stored values must be within the FP8 tolerance, 6e-2
max-abs, of the fp64 oracle run on the dequantised rows.  Only the test whose
groups are scaled far from unit size (values up to a few thousand) widens it,
by the two roundings that grow with the values: the bf16 output (half an
ulp, 2^-9 of |out|, taken as 2^-8) and the f16 probabilities times f16 group
scales of the P.V product (2^-11 of each weight twice, so at most 2^-10 of
max |v|)."""
import numpy as np
import pytest
import torch

import synth
from oracle import attention as oatt
from oracle import int4 as oint4
from oracle import projection as oproj
from compact_decode_attention_b200 import dms

from gpu_util import (check_block_invariants, head_id, int4_rows, oracle_store, read_state)

pytestmark = pytest.mark.gpu

TOL = 6e-2


def _dev(a, dt):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dt).cuda()


def _stored(X):
    """[..., T, Hkv, D] rows -> the values a 4-bit store holds for them."""
    return oint4.stored(np.asarray(X, np.float32))


def _check_store(pool, K, V, flags, P, w):
    state = read_state(pool)
    assert state["error"] == 0
    B, T, Hkv, D = K.shape
    for b in range(B):
        for h in range(Hkv):
            store = oracle_store(flags[b, :P, h], flags[b, P:, h], w, P)
            hd = head_id(pool.cfg, 0, b, h)
            assert state["n_slots"][hd] == store.n_slots
            assert state["n_retained"][hd] == store.n_retained
            assert state["free_top"][hd] == len(store.free)
            for idx, e in enumerate(store.ring):
                if e is not None:
                    assert state["ring"][hd, idx] == (e[0] | (e[1] << 31)), (hd, idx)
            n = store.n_slots
            pos = np.array([store.pos_of_slot[s] for s in range(n)])
            ck, sk, cv, sv = int4_rows(pool, state, hd, n)
            qk, ek = oint4.quantize(K[b, pos, h])
            qv, ev = oint4.quantize(V[b, pos, h])
            assert np.array_equal(ck, qk), f"K codes differ for head {hd}"
            assert np.array_equal(sk, ek), f"K scales differ for head {hd}"
            assert np.array_equal(cv, qv), f"V codes differ for head {hd}"
            assert np.array_equal(sv, ev), f"V scales differ for head {hd}"
    check_block_invariants(pool, state)


def _run(seed, B, P, S, Hq, Hkv, w, in_kind, p_keep=0.3, edit=None, widen=False):
    D = 128
    K = synth.kv_tokens(seed, 0, 0, B, 0, P + S, Hkv, D, in_kind)
    V = synth.kv_tokens(seed, 1, 0, B, 0, P + S, Hkv, D, in_kind)
    if edit is not None:
        edit(K, V)
    Q = np.stack([synth.q_tokens(seed, 0, B, P + s, Hq, D, "bf16") for s in range(S)])
    flags = synth.flag_tokens(seed, 0, B, 0, P + S, Hkv, [synth.keep_threshold(p_keep)] * Hkv)
    dt = torch.float32 if in_kind == "f32" else torch.bfloat16
    T = P + S
    pool = dms.Pool(1, B, Hq, Hkv, D, w, dms.DMS_INT4, B * Hkv * ((T + 63) // 64 + 1), T + 1)
    if P > 0:
        pool.compact_prefill(0, _dev(K[:, :P], dt), _dev(V[:, :P], dt),
                             torch.from_numpy(np.ascontiguousarray(flags[:, :P])).cuda())
    Ks, Vs = _stored(K), _stored(V)
    worst = 0.0
    for s in range(S):
        t = P + s
        pool.append_evict_layers(0, t, _dev(K[None, :, t], dt), _dev(V[None, :, t], dt),
                                 torch.from_numpy(np.ascontiguousarray(flags[None, :, t])).cuda())
        out = torch.empty(1, B, Hq, D, dtype=torch.bfloat16, device="cuda")
        pool.decode_attn_layers(0, _dev(Q[None, s], torch.bfloat16), out)
        got = out[0].float().cpu().numpy()
        for b in range(B):
            exp = oatt.decode_attention(Q[s, b].astype(np.float64), Ks[b, :t + 1], Vs[b, :t + 1],
                                        flags[b, :t + 1], t, w)
            bound = TOL
            if widen:     # values far from unit scale: the roundings that grow with them
                bound = TOL + np.abs(exp) * 2.0 ** -8 + np.abs(Vs[b, :t + 1]).max() * 2.0 ** -10
            worst = max(worst, float((np.abs(got[b] - exp) / bound).max()))
    assert worst < 1.0, worst
    _check_store(pool, K, V, flags, P, w)
    return pool


@pytest.mark.parametrize("in_kind", ["bf16", "f32"])
def test_int4_store_every_step(in_kind):
    """Prompt over several blocks with a ragged tail, then decode steps that
    retire window tokens into reused slots (V nibbles shared by 8 tokens)."""
    _run(81, 2, 300, 70, 8, 2, 32, in_kind, p_keep=0.3)


def test_int4_gqa_and_block_boundaries():
    """GQA 4 with a prompt that ends exactly on a block edge, so the first
    decode token opens a fresh block (its V tile is cleared)."""
    _run(82, 3, 128, 80, 12, 3, 16, "bf16", p_keep=0.5)


def test_int4_zero_and_large_groups():
    """A group of zeros (scale 0, codes 0) and groups with amax near the f16
    range limit of the dequantised values."""
    def edit(K, V):
        K[0, :, 0, 32:64] = 0.0
        V[1, :, 1, 96:128] = 0.0
        K[1, ::7, 0, 0:32] *= 512.0        # |k| up to a few thousand
        V[0, ::5, 1, 64:96] *= 1024.0
        K[:] = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(K))
        V[:] = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(V))
    _run(83, 2, 150, 40, 8, 2, 24, "bf16", p_keep=0.4, edit=edit, widen=True)


def test_int4_all_layers_fused_call_and_release():
    """Several layers in one append / attention call, then one sequence
    released and its slot filled again from a new prompt."""
    L, B, Hq, Hkv, D, w, P, S = 3, 2, 8, 2, 128, 16, 90, 30
    rng_seed = 84
    pool = dms.Pool(L, B, Hq, Hkv, D, w, dms.DMS_INT4, 64, P + S + 1)
    Ks, Vs, Fs = [], [], []
    for layer in range(L):
        K = synth.kv_tokens(rng_seed, 0, layer, B, 0, P + S, Hkv, D, "bf16")
        V = synth.kv_tokens(rng_seed, 1, layer, B, 0, P + S, Hkv, D, "bf16")
        F = synth.flag_tokens(rng_seed, layer, B, 0, P + S, Hkv, [synth.keep_threshold(0.3)] * Hkv)
        pool.compact_prefill(layer, _dev(K[:, :P], torch.bfloat16), _dev(V[:, :P], torch.bfloat16),
                             torch.from_numpy(np.ascontiguousarray(F[:, :P])).cuda())
        Ks.append(K)
        Vs.append(V)
        Fs.append(F)
    K, V, F = np.stack(Ks), np.stack(Vs), np.stack(Fs)          # [L, B, T, Hkv, D]
    SK, SV = _stored(K), _stored(V)
    for s in range(S):
        t = P + s
        q = np.stack([synth.q_tokens(rng_seed + layer, 0, B, t, Hq, D, "bf16") for layer in range(L)])
        pool.append_evict_layers(0, t, _dev(K[:, :, t], torch.bfloat16), _dev(V[:, :, t], torch.bfloat16),
                                 torch.from_numpy(np.ascontiguousarray(F[:, :, t])).cuda())
        out = torch.empty(L, B, Hq, D, dtype=torch.bfloat16, device="cuda")
        pool.decode_attn_layers(0, _dev(q, torch.bfloat16), out)
        got = out.float().cpu().numpy()
        for layer in range(L):
            for b in range(B):
                exp = oatt.decode_attention(q[layer, b].astype(np.float64), SK[layer, b, :t + 1],
                                            SV[layer, b, :t + 1], F[layer, b, :t + 1], t, w)
                assert np.abs(got[layer, b] - exp).max() < TOL, (s, layer, b)
    # release sequence 1 and prefill it again: its blocks come back from the free stack
    pool.release_seqs(torch.tensor([1], dtype=torch.int32, device="cuda"))
    K2 = synth.kv_tokens(rng_seed + 9, 0, 0, 1, 0, P, Hkv, D, "bf16")
    V2 = synth.kv_tokens(rng_seed + 9, 1, 0, 1, 0, P, Hkv, D, "bf16")
    F2 = synth.flag_tokens(rng_seed + 9, 0, 1, 0, P, Hkv, [synth.keep_threshold(0.3)] * Hkv)
    pool.compact_prefill_seqs(0, 1, _dev(K2, torch.bfloat16), _dev(V2, torch.bfloat16),
                              torch.from_numpy(np.ascontiguousarray(F2)).cuda())
    state = read_state(pool)
    assert state["error"] == 0
    for h in range(Hkv):
        store = oracle_store(F2[0, :, h], np.zeros(0, np.uint8), w, P)
        hd = head_id(pool.cfg, 0, 1, h)
        n = store.n_slots
        assert state["n_slots"][hd] == n
        pos = np.array([store.pos_of_slot[i] for i in range(n)])
        ck, sk, cv, sv = int4_rows(pool, state, hd, n)
        qk, ek = oint4.quantize(K2[0, pos, h])
        qv, ev = oint4.quantize(V2[0, pos, h])
        assert np.array_equal(ck, qk) and np.array_equal(sk, ek)
        assert np.array_equal(cv, qv) and np.array_equal(sv, ev)
    check_block_invariants(pool, state)


def test_int4_projected_tokens():
    """The fused projection epilogue quantises into a 4-bit store too."""
    L, Bmax, Hq, Hkv, D, w, dm, P, S = 1, 2, 8, 2, 128, 16, 256, 40, 12
    rng = np.random.default_rng(85)
    pool = dms.Pool(L, Bmax, Hq, Hkv, D, w, dms.DMS_INT4, 32, P + S + 1)
    W = oproj.bf16_round(rng.standard_normal((dm, 2 * Hkv * D)) / np.sqrt(dm))
    we = oproj.bf16_round(rng.standard_normal((dm, Hkv)) / np.sqrt(dm))
    be = np.zeros(Hkv, np.float32)
    K = synth.kv_tokens(86, 0, 0, Bmax, 0, P, Hkv, D, "bf16")
    V = synth.kv_tokens(86, 1, 0, Bmax, 0, P, Hkv, D, "bf16")
    F = synth.flag_tokens(86, 0, Bmax, 0, P, Hkv, [synth.keep_threshold(0.4)] * Hkv)
    pool.compact_prefill(0, _dev(K, torch.bfloat16), _dev(V, torch.bfloat16),
                         torch.from_numpy(np.ascontiguousarray(F)).cuda())
    Wd, wed, bed = _dev(W, torch.bfloat16), _dev(we, torch.bfloat16), torch.from_numpy(be).cuda()
    ids = torch.arange(Bmax, dtype=torch.int32, device="cuda")
    last = {}
    for step in range(S):
        t = P + step
        X = oproj.bf16_round(rng.standard_normal((Bmax, dm)))
        pool.project_append(0, ids, torch.full((Bmax,), t, dtype=torch.int64, device="cuda"),
                            _dev(X, torch.bfloat16), Wd, wed, bed, 0.0)
        for b in range(Bmax):
            k, v, _ = oproj.project_token(X[b], W, we, be, Hkv, D)
            last[b] = (oproj.bf16_round(k), oproj.bf16_round(v), t)
    # the last token's row of each head: codes within one step of the
    # oracle's (the kernel's fp32 sum may round k to the neighbouring bf16)
    state = read_state(pool)
    assert state["error"] == 0
    for b in range(Bmax):
        k, v, t = last[b]
        for h in range(Hkv):
            hd = head_id(pool.cfg, 0, b, h)
            slot = int(state["ring"][hd, t % w] & 0x7fffffff)
            n = int(state["n_slots"][hd])
            ck, sk, cv, sv = int4_rows(pool, state, hd, n)
            got_k = ck[slot].astype(np.float64) * np.repeat(sk[slot], 32)
            got_v = cv[slot].astype(np.float64) * np.repeat(sv[slot], 32)
            ek, ev = _stored(k[h][None])[0], _stored(v[h][None])[0]
            assert np.abs(got_k - ek).max() <= np.repeat(sk[slot], 32).max() * 1.01
            assert np.abs(got_v - ev).max() <= np.repeat(sv[slot], 32).max() * 1.01
