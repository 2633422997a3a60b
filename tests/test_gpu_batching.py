"""Continuous batching over the pool (through the C ABI): sequences are
prefilled into any free slot, decode at their own positions, and give their
blocks back when they finish; a later sequence reuses the slot and the
blocks.  Every output is compared with the fp64 oracle on that request's own
token history, the head stores bit for bit with the oracle's slot simulator,
and block ownership with the pool invariants."""
import numpy as np
import pytest
import torch

import synth
from oracle import attention as oatt
from oracle import fp8 as ofp8
from compact_decode_attention_b200 import dms

from gpu_util import check_block_invariants, check_head_store, head_id, oracle_store, read_state

pytestmark = pytest.mark.gpu


class Request:
    """One sequence's synthetic stream: prompt + decode tokens per layer."""

    def __init__(self, seed, P, S, L, Hq, Hkv, D, p_keep, in_kind="bf16"):
        self.seed, self.P, self.t = seed, P, P
        self.Hq, self.in_kind = Hq, in_kind
        thr = [synth.keep_threshold(p_keep)] * Hkv
        self.K = [synth.kv_tokens(seed, 0, l, 1, 0, P + S, Hkv, D, in_kind)[0] for l in range(L)]
        self.V = [synth.kv_tokens(seed, 1, l, 1, 0, P + S, Hkv, D, in_kind)[0] for l in range(L)]
        self.F = [synth.flag_tokens(seed, l, 1, 0, P + S, Hkv, thr)[0] for l in range(L)]

    def q(self, layer, t):
        return synth.q_tokens(self.seed, layer, 1, t, self.Hq, self.K[0].shape[-1], self.in_kind)[0]


def _dev(a, dt=torch.bfloat16):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dt).cuda()


def prefill(pool, req, slot, L):
    for l in range(L):
        pool.compact_prefill_seqs(l, slot, _dev(req.K[l][None, :req.P]), _dev(req.V[l][None, :req.P]),
                                  torch.from_numpy(np.ascontiguousarray(req.F[l][None, :req.P])).cuda())


def step(pool, active, L, kv_of=None):
    """One decode step of the active (slot, request) list; returns outputs [L, n, Hq, D]."""
    slots = torch.tensor([s for s, _ in active], dtype=torch.int32, device="cuda")
    pos = torch.tensor([r.t for _, r in active], dtype=torch.int64, device="cuda")
    k = _dev(np.stack([[r.K[l][r.t] for _, r in active] for l in range(L)]))
    v = _dev(np.stack([[r.V[l][r.t] for _, r in active] for l in range(L)]))
    f = torch.from_numpy(np.stack([[r.F[l][r.t] for _, r in active] for l in range(L)]).astype(np.uint8)).cuda()
    q_np = np.stack([[r.q(l, r.t) for _, r in active] for l in range(L)])
    out = torch.empty(q_np.shape, dtype=torch.bfloat16, device="cuda")
    pool.append_evict_seqs(0, slots, pos, k, v, f)
    pool.decode_attn_seqs(0, slots, _dev(q_np), out)
    got = out.float().cpu().numpy()
    for j, (_, r) in enumerate(active):
        for l in range(L):
            K, V = (r.K[l], r.V[l]) if kv_of is None else kv_of(r, l)
            exp = oatt.decode_attention(q_np[l, j].astype(np.float64), K[:r.t + 1], V[:r.t + 1],
                                        r.F[l][:r.t + 1], r.t, pool.cfg.window)
            err = np.abs(got[l, j] - exp).max()
            assert err < (6e-2 if kv_of is not None else 2e-2), (l, j, r.seed, r.t, err)
        r.t += 1
    return got


def check_stores(pool, active, L, kind="bf16", scales=None):
    state = read_state(pool)
    assert state["error"] == 0
    Hkv = pool.cfg.n_kv_heads
    for slot, r in active:
        for l in range(L):
            for h in range(Hkv):
                store = oracle_store(r.F[l][:r.P, h], r.F[l][r.P:r.t, h], pool.cfg.window, r.P)
                rk = {j: r.K[l][j, h] for j in range(r.t)}
                rv = {j: r.V[l][j, h] for j in range(r.t)}
                check_head_store(pool, state, head_id(pool.cfg, l, slot, h), store, rk, rv, kind,
                                 None if scales is None else scales[l][h])
    check_block_invariants(pool, state)
    return state


def test_sequences_join_finish_and_reuse_slots_and_blocks():
    L, Bmax, Hq, Hkv, D, w = 2, 4, 8, 2, 128, 32
    S = 24
    pool = dms.Pool(L, Bmax, Hq, Hkv, D, w, dms.DMS_BF16, 400, 400)
    r0 = Request(101, 200, S, L, Hq, Hkv, D, 0.3)
    r1 = Request(102, 90, S, L, Hq, Hkv, D, 0.3)
    r2 = Request(103, 150, S, L, Hq, Hkv, D, 0.3)
    r3 = Request(104, 64, S, L, Hq, Hkv, D, 0.5)
    prefill(pool, r0, 0, L)
    prefill(pool, r1, 1, L)
    active = [(0, r0), (1, r1)]
    for _ in range(6):
        step(pool, active, L)
    prefill(pool, r3, 2, L)                       # a request joins mid-way
    active = [(2, r3), (0, r0), (1, r1)]          # batch rows in any slot order
    for _ in range(4):
        step(pool, active, L)
    check_stores(pool, active, L)
    before = read_state(pool)
    pool.release_seqs(torch.tensor([0], dtype=torch.int32, device="cuda"))   # r0 finishes
    after = read_state(pool)
    assert np.all(after["n_slots"][[head_id(pool.cfg, l, 0, h) for l in range(L) for h in range(Hkv)]] == 0)
    freed = sum(-(-before["n_slots"][head_id(pool.cfg, l, 0, h)] // 64) for l in range(L) for h in range(Hkv))
    assert after["block_stack_top"] == before["block_stack_top"] + freed > 0
    prefill(pool, r2, 0, L)                       # a new request takes the slot
    mid = read_state(pool)
    need = sum(-(-mid["n_slots"][head_id(pool.cfg, l, 0, h)] // 64) for l in range(L) for h in range(Hkv))
    stack = after["block_stack_top"]
    assert mid["block_stack_top"] == stack - min(need, stack), "released blocks were not reused first"
    assert mid["next_block"] - after["next_block"] == max(0, need - stack)
    active = [(2, r3), (1, r1), (0, r2)]
    for _ in range(8):
        step(pool, active, L)
    state = check_stores(pool, active, L)
    held = sum(-(-state["n_slots"][head_id(pool.cfg, l, s, h)] // 64)
               for s, _ in active for l in range(L) for h in range(Hkv))
    st = pool.stats()
    assert st.blocks_in_use == held and st.error_flags == 0


def test_fp8_later_prefill_reuses_the_layer_scales():
    L, Bmax, Hq, Hkv, D, w = 1, 2, 8, 2, 128, 16
    pool = dms.Pool(L, Bmax, Hq, Hkv, D, w, dms.DMS_FP8_E4M3, 64, 300)
    r0 = Request(201, 100, 6, L, Hq, Hkv, D, 0.4)
    r1 = Request(202, 120, 6, L, Hq, Hkv, D, 0.4)
    prefill(pool, r0, 0, L)
    sc = read_state(pool)["scales"].copy()
    exp_sc = [[(ofp8.fp8_scale(np.abs(r0.K[0][:r0.P, h]).max()), ofp8.fp8_scale(np.abs(r0.V[0][:r0.P, h]).max()))
               for h in range(Hkv)]]
    for h in range(Hkv):
        assert sc[0, h, 0] == exp_sc[0][h][0] and sc[0, h, 1] == exp_sc[0][h][1]
    prefill(pool, r1, 1, L)
    assert np.array_equal(read_state(pool)["scales"], sc), "a later prefill changed the layer's scales"

    def stored(r, l):    # the values the store holds: E4M3 of x / scale, times the scale
        K = np.stack([ofp8.dequantize(ofp8.quantize(r.K[l][:, h], exp_sc[l][h][0]), exp_sc[l][h][0])
                      for h in range(Hkv)], axis=1)
        V = np.stack([ofp8.dequantize(ofp8.quantize(r.V[l][:, h], exp_sc[l][h][1]), exp_sc[l][h][1])
                      for h in range(Hkv)], axis=1)
        return K, V

    active = [(1, r1), (0, r0)]
    for _ in range(6):
        step(pool, active, L, kv_of=stored)
    check_stores(pool, active, L, kind="fp8", scales=exp_sc)


def test_bad_sequence_id_is_reported_and_other_rows_are_served():
    L, Bmax, Hq, Hkv, D, w = 1, 4, 8, 2, 64, 16
    pool = dms.Pool(L, Bmax, Hq, Hkv, D, w, dms.DMS_BF16, 64, 300)
    r0 = Request(301, 80, 2, L, Hq, Hkv, D, 0.3)
    prefill(pool, r0, 0, L)
    step(pool, [(0, r0)], L)
    ids = torch.tensor([0, Bmax], dtype=torch.int32, device="cuda")      # slot 4 does not exist
    q = _dev(np.stack([[r0.q(0, r0.t - 1), r0.q(0, r0.t - 1)]]))
    out = torch.zeros(1, 2, Hq, D, dtype=torch.bfloat16, device="cuda")
    pool.decode_attn_seqs(0, ids, q, out)
    st = pool.stats(check=False)
    assert st.error_flags & dms.DEVERR_BAD_SEQUENCE
    exp = oatt.decode_attention(r0.q(0, r0.t - 1).astype(np.float64), r0.K[0][:r0.t], r0.V[0][:r0.t],
                                r0.F[0][:r0.t], r0.t - 1, w)
    assert np.abs(out[0, 0].float().cpu().numpy() - exp).max() < 2e-2
    assert torch.all(out[0, 1] == 0)
