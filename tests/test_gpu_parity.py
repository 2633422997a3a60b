"""GPU parity of the CUDA path against the CPU oracle (through the C ABI).

Bookkeeping (counts, slots, ring, stored bytes) must be bit-exact; attention
outputs must be within max-abs 1e-5 (fp32 store), 2e-2 (bf16), 6e-2 (FP8).
Small cases compare every head at every step; the workloads at full size run
in the launch configuration the benchmark times (all layers per call, one
CTA per SM) and compare every head at one decode step (the 128K stress
workload: sampled heads) and sampled heads at others.
"""
import numpy as np
import pytest
import torch

import synth
from synth import configs
from oracle import attention as oatt
from oracle import fp8 as ofp8
from oracle import reference as oref
from compact_decode_attention_b200 import dms
from compact_decode_attention_b200.workload import DeviceWorkload

from gpu_util import (check_block_invariants, check_head_store, head_id, oracle_store, read_state)

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-2, "fp8": 6e-2}
KIND_CODE = {"f32": dms.DMS_F32, "bf16": dms.DMS_BF16, "fp8": dms.DMS_FP8_E4M3}


def round_to(x, kind):
    if kind == "f32":
        return x.astype(np.float32)
    return synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(x))


# ---------------------------------------------------------------------------
# small cases with host-made inputs: every head, every step
# ---------------------------------------------------------------------------

def run_small(K, V, flags, Q, P, w, kind="f32", max_batch=None, max_blocks=None,
              max_context=None, single_layer_api=False, sm_scale=0.0):
    """K, V [B, P+S, Hkv, D] and Q [S, B, Hq, D] float32 in input precision;
    flags [B, P+S, Hkv] uint8.  Returns (pool, outputs [S, B, Hq, D])."""
    B, T, Hkv, D = K.shape
    S = T - P
    Hq = Q.shape[2]
    dt = torch.float32 if kind == "f32" else torch.bfloat16
    pool = dms.Pool(1, max_batch or B, Hq, Hkv, D, w, KIND_CODE[kind],
                    max_blocks or (B * Hkv * ((T + 63) // 64 + 1)), max_context or (T + 1))
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dt).cuda()  # noqa: E731
    if P > 0:
        pool.compact_prefill(0, dev(K[:, :P]), dev(V[:, :P]),
                             torch.from_numpy(np.ascontiguousarray(flags[:, :P])).cuda())
    outs = []
    ws = pool.workspace(1, B)
    stream = torch.cuda.current_stream().cuda_stream
    for s in range(S):
        t = P + s
        k1, v1 = dev(K[None, :, t]), dev(V[None, :, t])
        f1 = torch.from_numpy(np.ascontiguousarray(flags[None, :, t])).cuda()
        q1 = dev(Q[None, s])
        out = torch.empty(1, B, Hq, D, dtype=dt, device="cuda")
        if single_layer_api:
            dms.dms_append_evict(pool.handle, 0, B, t, k1.data_ptr(), v1.data_ptr(), KIND_CODE[kind] if kind != "fp8" else dms.DMS_BF16,
                                 f1.data_ptr(), stream)
            dms.dms_decode_attn(pool.handle, 0, B, q1.data_ptr(), dms.torch_dtype_code(dt), out.data_ptr(),
                                sm_scale, ws.data_ptr(), ws.numel(), stream)
        else:
            pool.append_evict_layers(0, t, k1, v1, f1)
            pool.decode_attn_layers(0, q1, out, sm_scale)
        outs.append(out[0].float().cpu().numpy())
    return pool, np.array(outs)


def oracle_outputs(K, V, flags, Q, P, w, sm_scale=None, kv_store=None):
    """fp64 oracle outputs [S, B, Hq, D]; kv_store maps (K, V) to stored values."""
    B = K.shape[0]
    S = Q.shape[0]
    Ks, Vs = (K, V) if kv_store is None else kv_store(K, V)
    out = np.zeros(Q.shape)
    for s in range(S):
        t = P + s
        for b in range(B):
            out[s, b] = oatt.decode_attention(Q[s, b].astype(np.float64), Ks[b, :t + 1], Vs[b, :t + 1],
                                              flags[b, :t + 1], t, w, sm_scale)
    return out


def make_inputs(seed, B, P, S, Hq, Hkv, D, kind, p_keep=0.3, flags=None):
    in_kind = "f32" if kind == "f32" else "bf16"
    K = synth.kv_tokens(seed, 0, 0, B, 0, P + S, Hkv, D, in_kind)
    V = synth.kv_tokens(seed, 1, 0, B, 0, P + S, Hkv, D, in_kind)
    Q = np.stack([synth.q_tokens(seed, 0, B, P + s, Hq, D, in_kind) for s in range(S)]) if S else \
        np.zeros((0, B, Hq, D), np.float32)
    if flags is None:
        flags = synth.flag_tokens(seed, 0, B, 0, P + S, Hkv, [synth.keep_threshold(p_keep)] * Hkv)
    return K, V, flags, Q


def check_all_heads(pool, K, V, flags, P, w, kind, scales=None):
    state = read_state(pool)
    assert state["error"] == 0
    B, T, Hkv, _ = K.shape
    for b in range(B):
        for h in range(Hkv):
            store = oracle_store(flags[b, :P, h], flags[b, P:, h], w, P)
            rk = {j: K[b, j, h] for j in range(T)}
            rv = {j: V[b, j, h] for j in range(T)}
            check_head_store(pool, state, head_id(pool.cfg, 0, b, h), store, rk, rv, kind,
                             None if scales is None else scales[h])
    check_block_invariants(pool, state)
    return state


def test_tiny_fp32_workload_every_step():
    """The single-layer fp32 workload: every head, every step, tolerance 1e-5."""
    wl = configs.TINY_FP32
    K = synth.kv_tokens(wl.seed, 0, 0, wl.batch, 0, wl.prompt + wl.decode, wl.n_kv_heads, wl.head_dim, "f32")
    V = synth.kv_tokens(wl.seed, 1, 0, wl.batch, 0, wl.prompt + wl.decode, wl.n_kv_heads, wl.head_dim, "f32")
    flags = synth.flag_tokens(wl.seed, 0, wl.batch, 0, wl.prompt + wl.decode, wl.n_kv_heads, wl.thresholds()[0])
    Q = np.stack([synth.q_tokens(wl.seed, 0, wl.batch, wl.prompt + s, wl.n_q_heads, wl.head_dim, "f32")
                  for s in range(wl.decode)])
    pool, got = run_small(K, V, flags, Q, wl.prompt, wl.window, "f32")
    exp = oracle_outputs(K, V, flags, Q, wl.prompt, wl.window)
    assert np.abs(got - exp).max() < TOL["f32"]
    check_all_heads(pool, K, V, flags, wl.prompt, wl.window, "f32")
    st = pool.stats()
    assert st.error_flags == 0 and st.retained_tokens == sum(
        oracle_store(flags[b, :wl.prompt, h], flags[b, wl.prompt:, h], wl.window, wl.prompt).n_retained
        for b in range(wl.batch) for h in range(wl.n_kv_heads))


@pytest.mark.parametrize("kind,D,g", [("bf16", 64, 4), ("bf16", 128, 4), ("bf16", 128, 8),
                                      ("f32", 128, 2), ("bf16", 64, 1), ("bf16", 128, 3)])
def test_small_ragged_all_heads(kind, D, g):
    """Several tiles and ragged tails per head, varied head dims and GQA groups."""
    B, Hkv, P, S, w = 2, 3, 700, 70, 100
    K, V, flags, Q = make_inputs(11 + D + g, B, P, S, Hkv * g, Hkv, D, kind, p_keep=0.25)
    pool, got = run_small(K, V, flags, Q, P, w, kind)
    exp = oracle_outputs(K, V, flags, Q, P, w)
    assert np.abs(got - exp).max() < TOL[kind]
    check_all_heads(pool, K, V, flags, P, w, kind)


def test_single_layer_api_and_explicit_scale():
    K, V, flags, Q = make_inputs(5, 1, 300, 20, 8, 2, 64, "bf16")
    pool, got = run_small(K, V, flags, Q, 300, 40, "bf16", single_layer_api=True, sm_scale=0.07)
    exp = oracle_outputs(K, V, flags, Q, 300, 40, sm_scale=0.07)
    assert np.abs(got - exp).max() < TOL["bf16"]


@pytest.mark.parametrize("P,w,S", [(20, 64, 60), (1, 8, 30), (0, 8, 25), (130, 1, 20)])
def test_edge_prompt_and_window(P, w, S):
    """Prompt shorter than the window, one-token and empty prompts, w = 1."""
    K, V, flags, Q = make_inputs(7 + P + w, 2, P, S, 8, 2, 64, "bf16", p_keep=0.2)
    pool, got = run_small(K, V, flags, Q, P, w, "bf16")
    exp = oracle_outputs(K, V, flags, Q, P, w)
    assert np.abs(got - exp).max() < TOL["bf16"]
    check_all_heads(pool, K, V, flags, P, w, "bf16")


@pytest.mark.parametrize("pattern", ["all", "none"])
def test_interpolation_endpoints(pattern):
    """All tokens flagged: a sliding window of w; none flagged: full attention."""
    B, P, S, Hkv, w = 1, 400, 40, 2, 64
    fl = np.ones((B, P + S, Hkv), np.uint8) if pattern == "all" else np.zeros((B, P + S, Hkv), np.uint8)
    K, V, flags, Q = make_inputs(3, B, P, S, 8, Hkv, 128, "bf16", flags=fl)
    pool, got = run_small(K, V, flags, Q, P, w, "bf16")
    exp = oracle_outputs(K, V, flags, Q, P, w)
    assert np.abs(got - exp).max() < TOL["bf16"]
    st = read_state(pool)
    expect_n = w if pattern == "all" else P + S
    assert np.all(st["n_slots"][:Hkv] == expect_n) and np.all(st["n_retained"][:Hkv] == expect_n)


def test_eviction_off_window_keeps_everything():
    """A window longer than the context (the pages' 1M reference) keeps every token."""
    B, P, S, Hkv = 1, 300, 10, 2
    K, V, flags, Q = make_inputs(4, B, P, S, 4, Hkv, 64, "bf16", p_keep=0.0)
    pool, got = run_small(K, V, flags, Q, P, 1_000_000, "bf16")
    ref = oracle_outputs(K, V, np.zeros_like(flags), Q, P, 1)   # no flags = full attention
    assert np.abs(got - ref).max() < TOL["bf16"]
    assert np.all(read_state(pool)["n_slots"][:Hkv] == P + S)


def test_batch_below_max_batch():
    K, V, flags, Q = make_inputs(9, 2, 200, 15, 8, 2, 64, "bf16")
    pool, got = run_small(K, V, flags, Q, 200, 32, "bf16", max_batch=5)
    exp = oracle_outputs(K, V, flags, Q, 200, 32)
    assert np.abs(got - exp).max() < TOL["bf16"]
    st = read_state(pool)
    assert np.all(st["n_slots"][2 * 2:] == 0)          # sequences 2..4 untouched


def test_split_heads_merge_across_many_ctas():
    """One long head next to short ones: the long head is cut over most CTAs
    and merged by log-sum-exp; the short ones stay inside one CTA."""
    B, Hkv, P, S, w = 1, 4, 20000, 3, 16
    fl = np.ones((B, P + S, Hkv), np.uint8)
    fl[:, :, 1] = 0                        # head 1 keeps everything: 313 blocks
    K, V, flags, Q = make_inputs(21, B, P, S, 16, Hkv, 128, "bf16", flags=fl)
    pool, got = run_small(K, V, flags, Q, P, w, "bf16")
    exp = oracle_outputs(K, V, flags, Q, P, w)
    assert np.abs(got - exp).max() < TOL["bf16"]


def test_many_short_heads_in_one_call():
    """2 layers x 360 sequences x 8 kv-heads = 5760 heads of ~1-2 blocks in
    one call: every CTA's range crosses dozens of heads, and the per-thread
    head scan covers ~26 heads per thread; sampled sequences of both layers
    match the oracle."""
    L, B, Hq, Hkv, D, P, w = 2, 360, 8, 8, 128, 90, 16
    pool = dms.Pool(L, B, Hq, Hkv, D, w, dms.DMS_BF16, L * B * Hkv * 3, P + 2)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).cuda()  # noqa: E731
    data = []
    for layer in range(L):
        K = synth.kv_tokens(31, 0, layer, B, 0, P + 1, Hkv, D, "bf16")
        V = synth.kv_tokens(31, 1, layer, B, 0, P + 1, Hkv, D, "bf16")
        fl = synth.flag_tokens(31, layer, B, 0, P + 1, Hkv, [synth.keep_threshold(0.4)] * Hkv)
        pool.compact_prefill(layer, dev(K[:, :P]), dev(V[:, :P]), torch.from_numpy(fl[:, :P].copy()).cuda())
        data.append((K, V, fl))
    kn = np.stack([d[0][:, P] for d in data])
    vn = np.stack([d[1][:, P] for d in data])
    fn = np.stack([d[2][:, P] for d in data])
    pool.append_evict_layers(0, P, dev(kn), dev(vn), torch.from_numpy(fn.copy()).cuda())
    Q = np.stack([synth.q_tokens(31, layer, B, P, Hq, D, "bf16") for layer in range(L)])
    out = torch.empty(L, B, Hq, D, dtype=torch.bfloat16, device="cuda")
    pool.decode_attn_layers(0, dev(Q), out)
    got = out.float().cpu().numpy()
    for layer in range(L):
        K, V, fl = data[layer]
        for b in (0, 1, 179, 358, 359):
            exp = oatt.decode_attention(Q[layer, b].astype(np.float64), K[b], V[b], fl[b], P, w)
            assert np.abs(got[layer, b] - exp).max() < TOL["bf16"], (layer, b)
    assert read_state(pool)["error"] == 0


def test_fp8_store_small():
    """FP8-E4M3 store: scales bit-exact, stored codes bit-exact, outputs within 6e-2."""
    B, Hkv, P, S, w, D = 2, 2, 500, 40, 64, 128
    K, V, flags, Q = make_inputs(13, B, P, S, 8, Hkv, D, "fp8", p_keep=0.3)
    pool, got = run_small(K, V, flags, Q, P, w, "fp8")
    scales = [(ofp8.fp8_scale(np.abs(K[:, :P, h]).max()), ofp8.fp8_scale(np.abs(V[:, :P, h]).max()))
              for h in range(Hkv)]
    st = read_state(pool)
    for h in range(Hkv):
        assert st["scales"][0, h, 0] == scales[h][0] and st["scales"][0, h, 1] == scales[h][1]

    def store(Kx, Vx):
        Ks = np.empty(Kx.shape)
        Vs = np.empty(Vx.shape)
        for h in range(Hkv):
            Ks[:, :, h] = ofp8.dequantize(ofp8.quantize(Kx[:, :, h], scales[h][0]), scales[h][0])
            Vs[:, :, h] = ofp8.dequantize(ofp8.quantize(Vx[:, :, h], scales[h][1]), scales[h][1])
        return Ks, Vs

    exp = oracle_outputs(K, V, flags, Q, P, w, kv_store=store)
    assert np.abs(got - exp).max() < TOL["fp8"]
    check_all_heads(pool, K, V, flags, P, w, "fp8", scales=scales)


# ---------------------------------------------------------------------------
# failure paths: detected on the host or reported in the device error word
# ---------------------------------------------------------------------------

def test_blocks_exhausted_is_reported_and_nothing_written():
    K, V, flags, Q = make_inputs(1, 1, 500, 0, 4, 2, 64, "bf16", p_keep=1.0)
    pool, _ = run_small(K, V, flags, Q, 500, 32, "bf16", max_blocks=3)
    st = pool.stats(check=False)
    assert st.error_flags & dms.DEVERR_BLOCKS_EXHAUSTED
    with pytest.raises(dms.DmsError) as e:
        pool.stats()
    assert e.value.status == dms.DMS_ERR_DEVICE
    assert np.all(read_state(pool)["n_slots"] == 0)


def test_position_past_max_context_is_rejected():
    """A head cannot outgrow its block table: positions at or past max_context
    are refused on the host (the device check behind it is never reached)."""
    K, V, flags, Q = make_inputs(2, 1, 64, 2, 4, 1, 64, "bf16", p_keep=1.0)
    with pytest.raises(dms.DmsError) as e:
        run_small(K, V, flags, Q, 64, 128, "bf16", max_context=64)
    assert e.value.status == dms.DMS_ERR_INVALID_ARG


def test_prefill_into_filled_layer_is_refused():
    K, V, flags, Q = make_inputs(2, 1, 100, 0, 4, 1, 64, "bf16")
    pool, _ = run_small(K, V, flags, Q, 100, 16, "bf16")
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).cuda()  # noqa: E731
    before = read_state(pool)
    pool.compact_prefill(0, dev(K), dev(V), torch.from_numpy(flags).cuda())
    after = read_state(pool)
    assert pool.stats(check=False).error_flags & dms.DEVERR_LAYER_NOT_EMPTY
    assert np.array_equal(before["n_slots"], after["n_slots"])
    pool.reset()
    assert pool.stats().error_flags == 0 and np.all(read_state(pool)["n_slots"] == 0)


def test_invalid_arguments_are_rejected_on_the_host():
    pool = dms.Pool(2, 2, 8, 2, 64, 16, dms.DMS_BF16, 100, 1000)
    k = torch.zeros(1, 2, 2, 64, dtype=torch.bfloat16, device="cuda")
    f = torch.zeros(1, 2, 2, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    with pytest.raises(dms.DmsError) as e:     # layer range past the pool
        dms.dms_append_evict_layers(pool.handle, 1, 2, 2, 0, k.data_ptr(), k.data_ptr(), dms.DMS_BF16, f.data_ptr(), s)
    assert e.value.status == dms.DMS_ERR_INVALID_ARG
    with pytest.raises(dms.DmsError):           # dtype mismatch
        dms.dms_append_evict_layers(pool.handle, 0, 1, 2, 0, k.data_ptr(), k.data_ptr(), dms.DMS_F32, f.data_ptr(), s)
    with pytest.raises(dms.DmsError):           # misaligned input
        dms.dms_append_evict_layers(pool.handle, 0, 1, 2, 0, k.data_ptr() + 2, k.data_ptr(), dms.DMS_BF16, f.data_ptr(), s)
    ws = pool.workspace(1, 2)
    with pytest.raises(dms.DmsError) as e:     # workspace too small
        dms.dms_decode_attn_layers(pool.handle, 0, 1, 2, k.data_ptr(), dms.DMS_BF16, k.data_ptr(), 0.0,
                                   ws.data_ptr(), 16, s)
    assert e.value.status == dms.DMS_ERR_CAPACITY
    buf = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(dms.DmsError) as e:     # pool buffer too small
        dms.dms_pool_create(pool.cfg, buf.data_ptr(), buf.numel(), s)
    assert e.value.status == dms.DMS_ERR_CAPACITY


# ---------------------------------------------------------------------------
# the workloads at full size
# ---------------------------------------------------------------------------

def _sample_heads(wl, n_extra=2):
    probs = wl.keep_probs()
    heads = {(0, 0, 0), (wl.n_layers - 1, wl.batch - 1, wl.n_kv_heads - 1), (wl.n_layers // 2, 0, 3)}
    lo = np.unravel_index(np.argmin(probs), probs.shape)
    hi = np.unravel_index(np.argmax(probs), probs.shape)
    heads |= {(int(lo[0]), 0, int(lo[1])), (int(hi[0]), wl.batch // 2, int(hi[1]))}
    if wl.keep == "heavy_tail":
        full = np.argwhere(probs >= 1.0)[:n_extra]
        heads |= {(int(l), wl.batch - 1, int(h)) for l, h in full}
    return sorted(heads)


def _full_size(wl, check_steps, heads=None, all_heads_step=None):
    """Prefill and decode a workload at full size in the launch configuration
    the benchmark times.  Sampled heads are compared with the oracle at
    check_steps; at all_heads_step every (layer, sequence, kv-head) is, so
    that every CTA boundary, rotated range and cross-CTA merge of the real
    partition is checked.  FP8: every (layer, kv-head) scale bit-exact."""
    import oracle_jobs
    P, S, g = wl.prompt, wl.decode, wl.group
    dw = DeviceWorkload(wl, S, pregenerate_steps=wl.batch * wl.n_layers <= 288)
    dw.prefill()
    heads = heads or _sample_heads(wl)
    scales = None
    state = read_state(dw.pool)
    assert state["error"] == 0
    if wl.kv_dtype == "fp8":
        scales = [oref.fp8_layer_scales(wl, l) for l in range(wl.n_layers)]
        for l in range(wl.n_layers):
            for h in range(wl.n_kv_heads):
                assert state["scales"][l, h, 0] == scales[l][h][0], (l, h)
                assert state["scales"][l, h, 1] == scales[l][h][1], (l, h)
        l0, h0 = heads[0][0], heads[0][2]          # the chunked per-head definition agrees
        assert oref.fp8_head_scales(wl, l0, h0) == scales[l0][h0]
    every = [(l, b, h) for l in range(wl.n_layers) for b in range(wl.batch) for h in range(wl.n_kv_heads)]
    worst = 0.0
    for s in range(S):
        if dw.step_inputs is None:
            si = dw.make_step_inputs(P + s, 1)
            dw.pool.append_evict_layers(0, P + s, si["k"][0], si["v"][0], si["evict"][0])
            dw.pool.decode_attn_layers(0, si["q"][0], dw.out)
        else:
            dw.step(s)
        if s in check_steps or s == all_heads_step:
            out = dw.out.float().cpu().numpy()
            which = every if s == all_heads_step else heads
            exps = oracle_jobs.expected_outputs(wl, which, P + s, scales)
            for (l, b, h), exp in zip(which, exps):
                err = np.abs(out[l, b, h * g:(h + 1) * g] - exp).max()
                worst = max(worst, err)
                assert err < TOL[wl.kv_dtype], (l, b, h, s, err)
    # bookkeeping and stored bytes of the sampled heads after the last step
    state = read_state(dw.pool)
    assert state["error"] == 0
    for (l, b, h) in heads:
        fl = oref.head_flags(wl, l, b, h, P + S)
        store = oracle_store(fl[:P], fl[P:], wl.window, P)
        pos = np.array(sorted(store.pos_of_slot.values()))
        rk = dict(zip(pos, oref.head_input(wl, 0, l, b, h, 0, P + S)[pos]))
        rv = dict(zip(pos, oref.head_input(wl, 1, l, b, h, 0, P + S)[pos]))
        check_head_store(dw.pool, state, head_id(dw.pool.cfg, l, b, h), store, rk, rv,
                         wl.kv_dtype, None if scales is None else scales[l][h])
    check_block_invariants(dw.pool, state)
    st = dw.pool.stats()
    assert st.error_flags == 0
    return worst


def test_llama_1b_ctx8k_full_size():
    """All 128 heads at decode step 64; sampled heads at four steps."""
    wl = configs.LLAMA1B_CTX8K
    _full_size(wl, {0, 1, wl.decode - 1}, all_heads_step=64)


def test_qwen3_8b_ctx8k_full_size():
    """All 288 heads at decode step 64; sampled heads at four steps."""
    wl = configs.QWEN8B_CTX8K
    _full_size(wl, {0, 1, wl.decode - 1}, all_heads_step=64)


def test_qwen3_8b_fp8_b8_ctx32k_full_size():
    """All 2304 heads at the last decode step; every FP8 scale."""
    wl = configs.QWEN8B_FP8_B8_CTX32K
    heads = [(0, 0, 0), (35, 7, 7), (17, 3, 4)]
    _full_size(wl, {0}, heads=heads, all_heads_step=wl.decode - 1)


@pytest.mark.slow
def test_qwen3_8b_b16_ctx128k_stress_full_size():
    wl = configs.QWEN8B_B16_CTX128K
    probs = wl.keep_probs()
    full = [tuple(x) for x in np.argwhere(probs >= 1.0)[:2]]
    heads = [(int(full[0][0]), 15, int(full[0][1])), (int(full[1][0]), 0, int(full[1][1])),
             (0, 0, 0), (35, 15, 7)]
    _full_size(wl, {0, wl.decode - 1}, heads=heads)
