"""Prefill compaction at both piece sizes of the scatter kernel.

The scatter kernel gives a CTA 64 prompt tokens when a layer would have fewer
than 16 x SMs CTAs of 256 tokens, else 256.  For each store (bf16, FP8, 4-bit;
the quantised stores from bf16 and from fp32 inputs) the same prompts are compacted at a batch size that selects each span, into
pools whose blocks were filled with
0xFF bytes first (NaN in bf16, FP8 and the f16 scales), with per-head keep
probabilities from window-only to keep-all and a ragged last chunk.  Every
checked head's counters, ring and stored rows must equal the oracle's bit for
bit; in the quantised stores the V rows past a head's last slot must read zero
(the attention reads whole V tiles); one decode step over every head must
match the fp64 oracle."""
import numpy as np
import pytest
import torch

import synth
from oracle import attention as oatt
from oracle import fp8 as ofp8
from oracle import int4 as oint4
from compact_decode_attention_b200 import dms

from gpu_util import (BT, check_block_invariants, check_head_store, head_id, int4_rows, oracle_store,
                      read_state)

pytestmark = pytest.mark.gpu

CODE = {"bf16": dms.DMS_BF16, "fp8": dms.DMS_FP8_E4M3, "int4": dms.DMS_INT4}
TOL = {"bf16": 2e-2, "fp8": 6e-2, "int4": 6e-2}
KEEP = [0.3, 1.0, 0.0, 0.05, 0.5, 0.3, 0.9, 0.15] * 2   # per kv-head


def _dev(a, dt=torch.bfloat16):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dt).cuda()


def _v_tail_bytes(pool, state, hd, n, kind):
    """Bytes of the V rows r0..63 of the block holding slot n - 1 (r0 = n mod 64)."""
    r0 = n % BT
    blk = int(state["bt"][hd, (n - 1) // BT])
    lay, D = pool.layout, pool.cfg.head_dim
    o = int(lay.blocks + blk * lay.block_bytes)
    rows = np.arange(r0, BT)
    d = np.arange(D)
    if kind == "fp8":
        vt = pool.buffer[o + BT * D:o + 2 * BT * D].cpu().numpy()
        f = (((rows & 7) >> 1) << 4) | ((rows >> 4) << 2) | (((rows >> 3) & 1) << 1) | (rows & 1)
        return vt[d[:, None] * 64 + f[None, :]]
    tile = BT * (D // 2 + D // 16)
    vt = pool.buffer[o + tile:o + 2 * tile].cpu().numpy()
    words = vt[:BT * D // 2].view(np.uint32)
    wi = (d[:, None] * 32 + ((rows[None, :] & 7) >> 1) * 8 + (rows[None, :] >> 5) * 4) // 4
    sh = 8 * ((rows >> 4) & 1) + 4 * ((rows >> 3) & 1) + 16 * (rows & 1)
    nib = (words[wi] >> sh[None, :].astype(np.uint32)) & 0xF
    scales = vt[BT * D // 2:].view(np.uint16).reshape(D // 32, BT)[:, rows]
    return np.concatenate([nib.reshape(-1), scales.reshape(-1).astype(np.uint32)])


def _device_inputs(seed, B, n_pos, Hkv, D, thr, in_kind="bf16"):
    """K, V [B, n_pos, Hkv, D] (bf16 or fp32) and flags [B, n_pos, Hkv] drawn on
    the device by the generator's device twin."""
    st = torch.cuda.current_stream().cuda_stream
    dt, code = (torch.float32, dms.DMS_F32) if in_kind == "f32" else (torch.bfloat16, dms.DMS_BF16)
    K = torch.empty(1, B, n_pos, Hkv, D, dtype=dt, device="cuda")
    V = torch.empty_like(K)
    F = torch.empty(1, B, n_pos, Hkv, dtype=torch.uint8, device="cuda")
    dms.dms_synth_normal(seed, 0, 0, 1, B, 0, n_pos, Hkv, D, code, K.data_ptr(), st)
    dms.dms_synth_normal(seed, 1, 0, 1, B, 0, n_pos, Hkv, D, code, V.data_ptr(), st)
    t = torch.tensor([thr], dtype=torch.int32, device="cuda")
    dms.dms_synth_flags(seed, 0, 1, B, 0, n_pos, Hkv, t.data_ptr(), F.data_ptr(), st)
    return K[0], V[0], F[0]


def _host_sequence(seed, b, n_pos, Hkv, D, thr, in_kind="bf16"):
    """The same draws for one sequence, from the NumPy generator: [n_pos, Hkv, D] x 2, [n_pos, Hkv]."""
    pos = np.arange(n_pos)
    K = np.stack([synth.normal(seed, 0, 0, b, pos[:, None], h, np.arange(D)[None, :], in_kind)
                  for h in range(Hkv)], axis=1)
    V = np.stack([synth.normal(seed, 1, 0, b, pos[:, None], h, np.arange(D)[None, :], in_kind)
                  for h in range(Hkv)], axis=1)
    F = np.stack([synth.evict_flags(seed, 0, b, pos, h, thr[h]) for h in range(Hkv)], axis=1)
    return K, V, F


@pytest.mark.parametrize("kind,in_kind", [("bf16", "bf16"), ("fp8", "bf16"), ("int4", "bf16"),
                                          ("fp8", "f32"), ("int4", "f32")])
def test_both_piece_sizes_match_the_oracle(kind, in_kind):
    Hkv, Hq, D, P, w, seed = 16, 32, 128, 1000, 64, 91
    sm = torch.cuda.get_device_properties(0).multi_processor_count
    n_chunks = (P + 255) // 256
    # a batch whose 256-token CTA count crosses 16 x SMs (256-token spans),
    # and a batch of 2 (64-token spans)
    batches = [-(-16 * sm // (n_chunks * Hkv)) + 1, 2]
    thr = [synth.keep_threshold(p) for p in KEEP]
    Kd, Vd, Fd = _device_inputs(seed, batches[0], P + 1, Hkv, D, thr, in_kind)
    rng = np.random.default_rng(seed)
    host = {}
    for B in batches:
        pool = dms.Pool(1, B, Hq, Hkv, D, w, CODE[kind], B * Hkv * (P // BT + 3), P + 2)
        pool.buffer[pool.layout.blocks:].fill_(0xFF)       # stale bytes in every block
        pool.compact_prefill(0, Kd[:B, :P].contiguous(), Vd[:B, :P].contiguous(), Fd[:B, :P].contiguous())
        state = read_state(pool)
        assert state["error"] == 0
        check_block_invariants(pool, state)
        scales = None
        if kind == "fp8":   # amax over every prompt row of the batch (exact in any order)
            scales = [(ofp8.fp8_scale(np.float32(Kd[:B, :P, h].float().abs().max().item())),
                       ofp8.fp8_scale(np.float32(Vd[:B, :P, h].float().abs().max().item())))
                      for h in range(Hkv)]
            for h in range(Hkv):
                assert state["scales"][0, h, 0] == scales[h][0] and state["scales"][0, h, 1] == scales[h][1]
        seqs = sorted({0, B - 1, int(rng.integers(0, B))})
        for b in seqs:
            if b not in host:
                host[b] = _host_sequence(seed, b, P + 1, Hkv, D, thr, in_kind)
            K, V, F = host[b]
            for h in range(Hkv):
                hd = head_id(pool.cfg, 0, b, h)
                store = oracle_store(F[:P, h], np.zeros(0, np.uint8), w, P)
                n = store.n_slots
                if kind == "int4":
                    assert state["n_slots"][hd] == n and state["n_retained"][hd] == store.n_retained
                    for idx, e in enumerate(store.ring):
                        if e is not None:
                            assert state["ring"][hd, idx] == (e[0] | (e[1] << 31)), (hd, idx)
                    pos = np.array([store.pos_of_slot[s] for s in range(n)])
                    ck, sk, cv, sv = int4_rows(pool, state, hd, n)
                    qk, ek = oint4.quantize(K[pos, h])
                    qv, ev = oint4.quantize(V[pos, h])
                    assert np.array_equal(ck, qk) and np.array_equal(sk, ek), (B, b, h)
                    assert np.array_equal(cv, qv) and np.array_equal(sv, ev), (B, b, h)
                else:
                    rk = {j: K[j, h] for j in range(P)}
                    rv = {j: V[j, h] for j in range(P)}
                    check_head_store(pool, state, hd, store, rk, rv, kind,
                                     None if scales is None else scales[h])
                if kind != "bf16" and n % BT:
                    assert not _v_tail_bytes(pool, state, hd, n, kind).any(), (B, b, h)
        # one decode step over every head; outputs of the sampled sequences
        # against the oracle on the stored values
        pool.append_evict_layers(0, P, Kd[None, :B, P].contiguous(), Vd[None, :B, P].contiguous(),
                                 Fd[None, :B, P].contiguous())
        Q = synth.q_tokens(seed, 0, B, P, Hq, D, "bf16")
        out = torch.empty(1, B, Hq, D, dtype=torch.bfloat16, device="cuda")
        pool.decode_attn_layers(0, _dev(Q[None]), out)
        got = out[0].float().cpu().numpy()
        assert np.isfinite(got).all()
        del pool
        for b in seqs:
            K, V, F = host[b]
            Ks, Vs = K.astype(np.float64), V.astype(np.float64)
            if kind == "fp8":
                for h in range(Hkv):
                    Ks[:, h] = ofp8.dequantize(ofp8.quantize(K[:, h], scales[h][0]), scales[h][0])
                    Vs[:, h] = ofp8.dequantize(ofp8.quantize(V[:, h], scales[h][1]), scales[h][1])
            elif kind == "int4":
                Ks, Vs = oint4.stored(K), oint4.stored(V)
            exp = oatt.decode_attention(Q[b].astype(np.float64), Ks, Vs, F, P, w)
            assert (np.abs(got[b] - exp) < TOL[kind]).all(), (kind, B, b)


def test_refused_call_leaves_the_planner_clean():
    """A compaction the planner refuses (its layer is not empty) still resets
    the arrival tickets and the FP8 maxima: the next call, into another layer,
    takes its scales from its own rows only (the refused call's rows are 100x
    larger) and stores every head bit-exactly."""
    L, B, Hq, Hkv, D, P, w, seed = 2, 3, 4, 2, 128, 300, 32, 92
    thr = [synth.keep_threshold(0.3)] * Hkv
    pool = dms.Pool(L, B, Hq, Hkv, D, w, dms.DMS_FP8_E4M3, L * B * Hkv * (P // BT + 2), P + 1)
    K = synth.kv_tokens(seed, 0, 0, B, 0, P, Hkv, D, "bf16")
    V = synth.kv_tokens(seed, 1, 0, B, 0, P, Hkv, D, "bf16")
    F = synth.flag_tokens(seed, 0, B, 0, P, Hkv, thr)
    Fd = torch.from_numpy(np.ascontiguousarray(F)).cuda()
    pool.compact_prefill(0, _dev(K), _dev(V), Fd)
    pool.compact_prefill(0, _dev(K * 100), _dev(V * 100), Fd)          # refused: layer 0 is full
    assert pool.stats(check=False).error_flags & dms.DEVERR_LAYER_NOT_EMPTY
    K1 = synth.kv_tokens(seed, 0, 1, B, 0, P, Hkv, D, "bf16")
    V1 = synth.kv_tokens(seed, 1, 1, B, 0, P, Hkv, D, "bf16")
    F1 = synth.flag_tokens(seed, 1, B, 0, P, Hkv, thr)
    pool.compact_prefill(1, _dev(K1), _dev(V1), torch.from_numpy(np.ascontiguousarray(F1)).cuda())
    state = read_state(pool)
    for layer, (Kx, Vx, Fx) in enumerate(((K, V, F), (K1, V1, F1))):
        scales = [(ofp8.fp8_scale(np.abs(Kx[:, :, h]).max()), ofp8.fp8_scale(np.abs(Vx[:, :, h]).max()))
                  for h in range(Hkv)]
        for h in range(Hkv):
            assert state["scales"][layer, h, 0] == scales[h][0] and state["scales"][layer, h, 1] == scales[h][1]
            for b in range(B):
                store = oracle_store(Fx[b, :, h], np.zeros(0, np.uint8), w, P)
                check_head_store(pool, state, head_id(pool.cfg, layer, b, h), store,
                                 {j: Kx[b, j, h] for j in range(P)}, {j: Vx[b, j, h] for j in range(P)},
                                 "fp8", scales[h])
    check_block_invariants(pool, state)


@pytest.mark.parametrize("kind,P", [("bf16", 16384), ("bf16", 16384 + 300), ("f32", 16384 + 300)])
def test_copy_stores_either_side_of_the_one_launch_limit(kind, P):
    """Copy stores (bf16, fp32) take one launch up to 16384 prompt tokens and
    the plan + scatter launches past it: both give the oracle's store bit for
    bit."""
    B, Hq, Hkv, D, w, seed = 2, 4, 4, 64, 512, 93
    thr = [synth.keep_threshold(p) for p in (0.2, 1.0, 0.0, 0.05)]
    Kd, Vd, Fd = _device_inputs(seed, B, P, Hkv, D, thr, kind)
    code = dms.DMS_F32 if kind == "f32" else dms.DMS_BF16
    pool = dms.Pool(1, B, Hq, Hkv, D, w, code, B * Hkv * (P // BT + 3), P + 2)
    pool.buffer[pool.layout.blocks:].fill_(0xFF)
    pool.compact_prefill(0, Kd, Vd, Fd)
    state = read_state(pool)
    assert state["error"] == 0
    check_block_invariants(pool, state)
    F = Fd.cpu().numpy()
    for b in range(B):
        K, V, _ = _host_sequence(seed, b, P, Hkv, D, thr, kind)
        for h in range(Hkv):
            store = oracle_store(F[b, :, h], np.zeros(0, np.uint8), w, P)
            check_head_store(pool, state, head_id(pool.cfg, 0, b, h), store,
                             {j: K[j, h] for j in range(P)}, {j: V[j, h] for j in range(P)}, kind)
