"""dms_prefill_attn: prompt attention under the delayed-eviction mask on the
tensor cores, fused with compaction (through the C ABI).  Outputs are
compared with the fp64 oracle (every query on small prompts, sampled queries
on a long one, max-abs 2e-2 as for every bf16 path); the pool the fused
kernel fills must hold exactly what the oracle's compaction keeps (FP8 and
4-bit pools: compacted first, codes and scales bit-exact)."""
import numpy as np
import pytest
import torch

import synth
from oracle import attention as oatt
from compact_decode_attention_b200 import dms

from oracle import fp8 as ofp8
from oracle import int4 as oint4

from gpu_util import check_block_invariants, check_head_store, head_id, int4_rows, oracle_store, read_state

pytestmark = pytest.mark.gpu
TOL = 2e-2


def _inputs(seed, B, P, Hq, Hkv, D, p_keep):
    K = synth.kv_tokens(seed, 0, 0, B, 0, P, Hkv, D, "bf16")
    V = synth.kv_tokens(seed, 1, 0, B, 0, P, Hkv, D, "bf16")
    Q = np.stack([synth.q_tokens(seed, 0, B, i, Hq, D, "bf16") for i in range(P)], axis=1)  # [B, P, Hq, D]
    F = synth.flag_tokens(seed, 0, B, 0, P, Hkv, [synth.keep_threshold(p_keep)] * Hkv)
    return Q, K, V, F


def _run(pool, seq0, Q, K, V, F, layer=0):
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).cuda()  # noqa: E731
    out = torch.full(Q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    pool.prefill_attn(layer, seq0, dev(Q), dev(K), dev(V), torch.from_numpy(np.ascontiguousarray(F)).cuda(), out)
    return out.float().cpu().numpy()


def _check_store(pool, seq0, K, V, F, P, w):
    state = read_state(pool)
    assert state["error"] == 0
    B, _, Hkv, _ = K.shape
    for b in range(B):
        for h in range(Hkv):
            store = oracle_store(F[b, :, h], np.zeros(0, np.uint8), w, P)
            check_head_store(pool, state, head_id(pool.cfg, 0, seq0 + b, h), store,
                             {j: K[b, j, h] for j in range(P)}, {j: V[b, j, h] for j in range(P)}, "bf16")
    check_block_invariants(pool, state)


@pytest.mark.parametrize("D,P,w,p_keep", [(128, 300, 64, 0.3), (64, 300, 64, 0.3), (128, 200, 512, 0.1),
                                          (128, 129, 1, 0.0), (64, 77, 16, 0.5)])
def test_every_query_matches_the_oracle_and_the_store_matches_compaction(D, P, w, p_keep):
    B, Hq, Hkv = 2, 8, 2
    Q, K, V, F = _inputs(7 + D + P, B, P, Hq, Hkv, D, p_keep)
    pool = dms.Pool(1, B, Hq, Hkv, D, w, dms.DMS_BF16, B * Hkv * (P // 64 + 2), P + 1)
    got = _run(pool, 0, Q, K, V, F)
    assert np.isfinite(got).all()
    for b in range(B):
        exp = oatt.prefill_attention(Q[b].astype(np.float64), K[b], V[b], F[b], w)
        err = np.abs(got[b] - exp).max()
        assert err < TOL, (b, err)
    _check_store(pool, 0, K, V, F, P, w)


def test_long_prompt_sampled_queries_and_sequence_offset():
    B, P, Hq, Hkv, D, w = 1, 2048, 32, 8, 128, 512
    Q, K, V, F = _inputs(91, B, P, Hq, Hkv, D, 0.15)
    pool = dms.Pool(1, 3, Hq, Hkv, D, w, dms.DMS_BF16, 3 * Hkv * (P // 64 + 2), P + 1)
    got = _run(pool, 2, Q, K, V, F)             # into sequence slot 2
    rng = np.random.default_rng(5)
    for i in sorted(set(rng.integers(0, P, 40).tolist()) | {0, 127, 128, 1023, P - 1}):
        exp = oatt.decode_attention(Q[0, i].astype(np.float64), K[0, :i + 1], V[0, :i + 1], F[0, :i + 1], i, w)
        assert np.abs(got[0, i] - exp).max() < TOL, i
    _check_store(pool, 2, K, V, F, P, w)


@pytest.mark.parametrize("kind,P", [("fp8", 333), ("int4", 333), ("fp8", 1500), ("int4", 1500)])
def test_quantised_pools_compact_first_then_attend(kind, P):
    """FP8 and 4-bit stores: the layer is compacted as by
    dms_compact_prefill_seqs (codes and scales bit-exact against the
    oracle), and every query's output matches the oracle on the bf16 inputs
    (the old kept keys are gathered from the prompt by the positions the
    compaction recorded; at P = 1500 several such tiles per query tile)."""
    B, Hq, Hkv, D, w = 2, 8, 2, 128, 64
    Q, K, V, F = _inputs(41, B, P, Hq, Hkv, D, 0.3)
    code = dms.DMS_FP8_E4M3 if kind == "fp8" else dms.DMS_INT4
    pool = dms.Pool(1, B, Hq, Hkv, D, w, code, B * Hkv * (P // 64 + 2), P + 1)
    got = _run(pool, 0, Q, K, V, F)
    for b in range(B):
        exp = oatt.prefill_attention(Q[b].astype(np.float64), K[b], V[b], F[b], w)
        assert np.abs(got[b] - exp).max() < TOL, b
    state = read_state(pool)
    assert state["error"] == 0
    for b in range(B):
        for h in range(Hkv):
            store = oracle_store(F[b, :, h], np.zeros(0, np.uint8), w, P)
            hd = head_id(pool.cfg, 0, b, h)
            assert state["n_slots"][hd] == store.n_slots
            pos = np.array([store.pos_of_slot[x] for x in range(store.n_slots)])
            if kind == "fp8":
                scales = (ofp8.fp8_scale(np.abs(K[:, :, h]).max()), ofp8.fp8_scale(np.abs(V[:, :, h]).max()))
                assert state["scales"][0, h, 0] == scales[0] and state["scales"][0, h, 1] == scales[1]
                check_head_store(pool, state, hd, store, {j: K[b, j, h] for j in range(P)},
                                 {j: V[b, j, h] for j in range(P)}, "fp8", scales)
            else:
                ck, sk, cv, sv = int4_rows(pool, state, hd, store.n_slots)
                qk, ek = oint4.quantize(K[b, pos, h])
                qv, ev = oint4.quantize(V[b, pos, h])
                assert np.array_equal(ck, qk) and np.array_equal(sk, ek)
                assert np.array_equal(cv, qv) and np.array_equal(sv, ev)
    check_block_invariants(pool, state)


def test_unsupported_pools_are_refused():
    pool = dms.Pool(1, 1, 8, 2, 128, 16, dms.DMS_F32, 16, 256)
    x = torch.zeros(1, 64, 8, 128, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(1, 64, 2, 128, dtype=torch.bfloat16, device="cuda")
    f = torch.zeros(1, 64, 2, dtype=torch.uint8, device="cuda")
    with pytest.raises(dms.DmsError) as e:
        pool.prefill_attn(0, 0, x, kv, kv, f, x)
    assert e.value.status == dms.DMS_ERR_UNSUPPORTED


def _sampled_check(got, Q, K, V, F, w, idx, b=0):
    for i in idx:
        exp = oatt.decode_attention(Q[b, i].astype(np.float64), K[b, :i + 1], V[b, :i + 1], F[b, :i + 1], i, w)
        err = np.abs(got[b, i] - exp).max()
        assert err < TOL, (i, err)


@pytest.mark.parametrize("D,w,p_keep,Hq", [(128, 128, 0.15, 8), (64, 128, 0.15, 8), (128, 256, 0.0, 8),
                                           (128, 128, 1.0, 8), (64, 200, 0.4, 8), (128, 128, 0.2, 6)])
def test_sparse_and_dense_reading_agree_with_the_oracle(D, w, p_keep, Hq):
    """Old kept keys read back from the store (default) against every key
    tile read from the prompt: the same store bit for bit, outputs within
    the bf16 bound of the oracle and of each other.  Keep rates 0 (far keys
    all evicted: no far tile), 1 (every old key kept) and in between, ragged
    far counts (not multiples of 128), a window that is not a tile multiple;
    an even group size runs two query heads per CTA, an odd one (g = 3) one."""
    B, P, Hkv = 2, 1500, 2
    Q, K, V, F = _inputs(300 + D + w, B, P, Hq, Hkv, D, p_keep)
    outs, states = {}, {}
    for mode in (dms.PREFILL_SPARSE, dms.PREFILL_DENSE):
        pool = dms.Pool(1, B, Hq, Hkv, D, w, dms.DMS_BF16, B * Hkv * (P // 64 + 2), P + 1)
        pool.set_prefill_mode(mode)
        outs[mode] = _run(pool, 0, Q, K, V, F)
        _check_store(pool, 0, K, V, F, P, w)
        states[mode] = read_state(pool)
    assert np.isfinite(outs[dms.PREFILL_SPARSE]).all()
    for key in ("n_slots", "n_retained", "ring"):
        assert np.array_equal(states[0][key], states[1][key]), key
    assert np.abs(outs[0] - outs[1]).max() < TOL
    idx = sorted(set(np.random.default_rng(D + w).integers(0, P, 24).tolist()) | {0, w, 383, 384, P - 1})
    for b in range(B):
        _sampled_check(outs[dms.PREFILL_SPARSE], Q, K, V, F, w, idx, b)


def test_sparse_reading_falls_back_when_far_blocks_are_missing():
    """A window shorter than a key tile with few kept keys: the far tiles'
    second block may not exist, so those query tiles read the prompt."""
    B, P, Hq, Hkv, D, w = 1, 700, 8, 2, 128, 16
    Q, K, V, F = _inputs(55, B, P, Hq, Hkv, D, 0.05)
    pool = dms.Pool(1, B, Hq, Hkv, D, w, dms.DMS_BF16, B * Hkv * (P // 64 + 2), P + 1)
    got = _run(pool, 0, Q, K, V, F)
    exp = oatt.prefill_attention(Q[0].astype(np.float64), K[0], V[0], F[0], w)
    assert np.abs(got[0] - exp).max() < TOL
    _check_store(pool, 0, K, V, F, P, w)


def test_a_layer_that_is_not_empty_still_gets_correct_outputs():
    """The second prompt into the same layer is refused by the compaction
    (DMS_DEVERR_LAYER_NOT_EMPTY); the store still holds the first prompt,
    so the attention must read every key from the second prompt."""
    B, P, Hq, Hkv, D, w = 1, 900, 8, 2, 128, 128
    Q, K, V, F = _inputs(61, B, P, Hq, Hkv, D, 0.2)
    Q2, K2, V2, F2 = _inputs(62, B, P, Hq, Hkv, D, 0.2)
    pool = dms.Pool(1, B, Hq, Hkv, D, w, dms.DMS_BF16, 2 * B * Hkv * (P // 64 + 2), P + 1)
    _run(pool, 0, Q, K, V, F)
    got = _run(pool, 0, Q2, K2, V2, F2)
    assert read_state(pool)["error"] & dms.DEVERR_LAYER_NOT_EMPTY
    _sampled_check(got, Q2, K2, V2, F2, w, [0, 200, 511, 512, 640, 777, P - 1])


@pytest.mark.parametrize("P", [16384, 16384 + 500])
def test_store_reading_on_either_side_of_the_one_launch_compaction(P):
    """Prompts up to 16384 tokens are compacted in one launch, longer ones by
    the plan and scatter launches; the prompt attention takes the far-key
    counts from either one's chunk prefix counts.  Sampled queries (every
    query tile is a different far/band split) against the oracle."""
    B, Hq, Hkv, D, w = 1, 4, 2, 64, 512
    Q, K, V, F = _inputs(70 + P, B, P, Hq, Hkv, D, 0.2)
    pool = dms.Pool(1, B, Hq, Hkv, D, w, dms.DMS_BF16, B * Hkv * (P // 64 + 2), P + 1)
    got = _run(pool, 0, Q, K, V, F)
    assert np.isfinite(got).all()
    rng = np.random.default_rng(P)
    idx = sorted(set(rng.integers(0, P, 10).tolist()) | {w + 127, 4096, P - 129, P - 1})
    _sampled_check(got, Q, K, V, F, w, idx)
    _check_store(pool, 0, K, V, F, P, w)


@pytest.mark.parametrize("kind", ["fp8", "int4"])
def test_quantised_pools_both_readings_agree(kind):
    """The gathered old-key tiles against every causal tile from the prompt
    (DMS_PREFILL_DENSE): the same store, outputs within the bf16 bound."""
    B, P, Hq, Hkv, D, w = 1, 1200, 8, 2, 128, 128
    Q, K, V, F = _inputs(83, B, P, Hq, Hkv, D, 0.2)
    code = dms.DMS_FP8_E4M3 if kind == "fp8" else dms.DMS_INT4
    outs, states = [], []
    for mode in (dms.PREFILL_SPARSE, dms.PREFILL_DENSE):
        pool = dms.Pool(1, B, Hq, Hkv, D, w, code, B * Hkv * (P // 64 + 2), P + 1)
        pool.set_prefill_mode(mode)
        outs.append(_run(pool, 0, Q, K, V, F))
        states.append(read_state(pool))
    assert states[0]["error"] == 0 and states[1]["error"] == 0
    for key in ("n_slots", "n_retained", "ring"):
        assert np.array_equal(states[0][key], states[1][key]), key
    assert np.isfinite(outs[0]).all()
    assert np.abs(outs[0] - outs[1]).max() < TOL
    _sampled_check(outs[0], Q, K, V, F, w, [0, 127, 128, 300, 640, 900, P - 1])
