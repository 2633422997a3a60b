"""Pins of the CPU oracle against things other than itself (CPU only).

Each check is chosen so that a plausible slip in the oracle (the window edge
off by one, a dropped scale, transposed operands, a wrong GQA mapping, a
wrong retire order, a wrong FP8 rounding) fails at least one of them:

* library routines: torch's fp64 scaled_dot_product_attention (with its own
  GQA expansion), torch's and ml_dtypes' float8_e4m3fn casts;
* an operational model of delayed eviction written independently of the
  oracle's inequality (tokens carry a removal step), brute-forced over every
  flag pattern of short prompts;
* closed forms: retained counts, uniform mean for zero keys, one-hot values
  reading off the weights, a single visible key returning its value, the
  slot recurrence, the page's 6.4x compression at ctx 8192;
* page figures and format landmarks stored under tests/golden/.
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch

import synth
from synth import configs
from oracle import attention, compaction, fp8, int4, mask, projection, reference, slots

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
PAGE = json.load(open(os.path.join(GOLDEN, "page_figures.json")))
E4M3 = json.load(open(os.path.join(GOLDEN, "e4m3_spec.json")))


# ---------------------------------------------------------------------------
# independent operational model of delayed eviction
# ---------------------------------------------------------------------------

def operational_cache_sets(evict, w):
    """Cache contents after each arrival: a flagged token is given a removal
    step w after its arrival and is physically dropped when that step comes."""
    cache = []          # (position, removal step or None)
    sets = []
    for t, f in enumerate(evict):
        cache = [(p, r) for (p, r) in cache if r is None or r > t]
        cache.append((t, t + w if f else None))
        sets.append(sorted(p for p, _ in cache))
    return sets


def sdpa(q, K, V, scale, mask_=None):
    """torch fp64 SDPA for one decode query: q [Hq, D], K/V [n, Hkv, D]."""
    qt = torch.from_numpy(np.asarray(q, np.float64))[None, :, None, :]
    Kt = torch.from_numpy(np.asarray(K, np.float64)).permute(1, 0, 2)[None]
    Vt = torch.from_numpy(np.asarray(V, np.float64)).permute(1, 0, 2)[None]
    am = None
    if mask_ is not None:   # [Hkv, n] -> broadcast to each query head of the group
        g = q.shape[0] // K.shape[1]
        am = torch.from_numpy(np.repeat(mask_, g, axis=0))[None, :, None, :]
    out = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, attn_mask=am, scale=scale,
                                                           enable_gqa=True)
    return out[0, :, 0, :].numpy()


def rand_case(rng, n, Hq=8, Hkv=2, D=16):
    q = rng.standard_normal((Hq, D))
    K = rng.standard_normal((n, Hkv, D))
    V = rng.standard_normal((n, Hkv, D))
    return q, K, V


# ---------------------------------------------------------------------------
# mask and attention
# ---------------------------------------------------------------------------

def test_eviction_off_window_gives_full_attention():
    rng = np.random.default_rng(0)
    w_off = PAGE["eviction_off_window"]["value"]
    t = 40
    q, K, V = rand_case(rng, t + 1)
    evict = rng.integers(0, 2, size=(t + 1, 2)).astype(np.uint8)
    got = attention.decode_attention(q, K, V, evict, t, w_off, 0.3)
    np.testing.assert_allclose(got, sdpa(q, K, V, 0.3), rtol=0, atol=1e-12)


def test_no_flags_gives_full_attention_for_any_window():
    rng = np.random.default_rng(1)
    t = 33
    q, K, V = rand_case(rng, t + 1)
    evict = np.zeros((t + 1, 2), dtype=np.uint8)
    for w in (1, 2, 7):
        got = attention.decode_attention(q, K, V, evict, t, w, 0.25)
        np.testing.assert_allclose(got, sdpa(q, K, V, 0.25), rtol=0, atol=1e-12)


def test_all_flags_give_sliding_window_of_w():
    rng = np.random.default_rng(2)
    t = 50
    q, K, V = rand_case(rng, t + 1)
    evict = np.ones((t + 1, 2), dtype=np.uint8)
    for w in (1, 3, 8):
        got = attention.decode_attention(q, K, V, evict, t, w, 0.2)
        ref = sdpa(q, K[t - w + 1:], V[t - w + 1:], 0.2)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_page_window_holds_exactly_512_tokens_when_all_flagged():
    w = PAGE["delay_window"]["value"]
    t = PAGE["ctx_len"]["value"] - 1
    evict = np.ones(t + 1, dtype=np.uint8)
    vis = mask.visible_positions(t, evict, w)
    assert len(vis) == 512 and vis[0] == t - 511 and vis[-1] == t


def test_general_flags_match_sdpa_with_operational_mask():
    """Random flags: the oracle equals torch SDPA given the cache contents of
    the operational model as a boolean mask (also pins the GQA mapping, the
    score scale and the softmax axis)."""
    rng = np.random.default_rng(3)
    n, w = 64, 5
    q, K, V = rand_case(rng, n, Hq=12, Hkv=3, D=8)
    evict = (rng.random((n, 3)) < 0.7).astype(np.uint8)
    for t in (0, 4, 5, 17, 63):
        m = np.zeros((3, t + 1), dtype=bool)
        for h in range(3):
            m[h, operational_cache_sets(evict[:t + 1, h], w)[t]] = True
        got = attention.decode_attention(q, K[:t + 1], V[:t + 1], evict[:t + 1], t, w, 0.37)
        np.testing.assert_allclose(got, sdpa(q, K[:t + 1], V[:t + 1], 0.37, m), rtol=0, atol=1e-12)


def sdpa_prefill(Q, K, V, scale, mask_):
    """torch fp64 SDPA over all prompt queries: Q [P, Hq, D], K/V [P, Hkv, D],
    mask_ [Hkv, P, P] boolean (query, key)."""
    g = Q.shape[1] // K.shape[1]
    qt = torch.from_numpy(np.asarray(Q, np.float64)).permute(1, 0, 2)[None]
    Kt = torch.from_numpy(np.asarray(K, np.float64)).permute(1, 0, 2)[None]
    Vt = torch.from_numpy(np.asarray(V, np.float64)).permute(1, 0, 2)[None]
    am = torch.from_numpy(np.repeat(mask_, g, axis=0))[None]
    out = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, attn_mask=am, scale=scale,
                                                           enable_gqa=True)
    return out[0].permute(1, 0, 2).numpy()


def test_prefill_attention_matches_sdpa_with_operational_mask():
    """Every prompt query, random flags: the oracle equals torch SDPA whose
    (query, key) mask comes from the operational model's cache contents."""
    rng = np.random.default_rng(11)
    P, w, Hq, Hkv, D = 40, 6, 6, 3, 8
    Q = rng.standard_normal((P, Hq, D))
    _, K, V = rand_case(rng, P, Hq=Hq, Hkv=Hkv, D=D)
    evict = (rng.random((P, Hkv)) < 0.6).astype(np.uint8)
    m = np.zeros((Hkv, P, P), dtype=bool)
    for h in range(Hkv):
        for i, vis in enumerate(operational_cache_sets(evict[:, h], w)):
            m[h, i, vis] = True
    got = attention.prefill_attention(Q, K, V, evict, w, 0.41)
    np.testing.assert_allclose(got, sdpa_prefill(Q, K, V, 0.41, m), rtol=0, atol=1e-12)


def test_prefill_attention_endpoints():
    """w >= P: plain causal attention (torch's is_causal); all flags and w = 1:
    each query sees only itself, so the output is its own value row."""
    rng = np.random.default_rng(12)
    P, Hq, Hkv, D = 33, 4, 2, 8
    Q = rng.standard_normal((P, Hq, D))
    _, K, V = rand_case(rng, P, Hq=Hq, Hkv=Hkv, D=D)
    flags = np.ones((P, Hkv), np.uint8)
    got = attention.prefill_attention(Q, K, V, flags, P, 0.3)
    qt = torch.from_numpy(Q).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(
        qt, torch.from_numpy(K).permute(1, 0, 2)[None], torch.from_numpy(V).permute(1, 0, 2)[None],
        is_causal=True, scale=0.3, enable_gqa=True)[0].permute(1, 0, 2).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    only_self = attention.prefill_attention(Q, K, V, flags, 1, 0.3)
    np.testing.assert_allclose(only_self, np.repeat(V, Hq // Hkv, axis=1), rtol=0, atol=1e-12)


def test_projection_one_hot_tokens_read_out_weight_rows():
    """x = e_d: k and v are row d of the projection, the logit is the
    predictor weight of row d plus the bias (pins the column split of k / v
    per head and the predictor layout)."""
    rng = np.random.default_rng(21)
    dm, Hkv, D = 24, 3, 8
    W = rng.standard_normal((dm, 2 * Hkv * D))
    we, be = rng.standard_normal((dm, Hkv)), rng.standard_normal(Hkv)
    for d in (0, 7, dm - 1):
        x = np.zeros(dm)
        x[d] = 1.0
        k, v, logit = projection.project_token(x, W, we, be, Hkv, D)
        for h in range(Hkv):
            assert np.array_equal(k[h], W[d, h * D:(h + 1) * D])
            assert np.array_equal(v[h], W[d, (Hkv + h) * D:(Hkv + h + 1) * D])
        assert np.array_equal(logit, we[d] + be)
    assert np.array_equal(projection.evict_flags(np.array([-1.0, 0.0, 1e-9]), 0.0), [0, 0, 1])


def test_bf16_rounding_matches_torch_and_rounds_fp64_once():
    """On fp32 inputs the oracle's bf16 rounding equals torch's; on fp64
    values just above a tie it rounds up where fp64 -> fp32 -> bf16 would
    round to even (a double-rounding trap)."""
    rng = np.random.default_rng(22)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(projection.bf16_round(x.astype(np.float64)), ref)
    one = 1.0
    tie = one + 2.0 ** -8                      # halfway between bf16 1.0 and 1.0 + 2^-7
    assert projection.bf16_round(np.array([tie]))[0] == 1.0          # tie to even
    above = tie + 2.0 ** -40                   # rounds to 1.0 in fp32, but is above the tie
    assert np.float32(above) == np.float32(tie)
    assert projection.bf16_round(np.array([above]))[0] == 1.0 + 2.0 ** -7


def test_int4_codes_are_the_nearest_multiples_of_the_group_scale():
    """Brute force: each code is the q in [-7, 7] whose q * scale is nearest
    to x (ties to the even q), the scale is the fp16 rounding of amax / 7 in
    fp32, and the largest magnitude of a group maps to +-7."""
    rng = np.random.default_rng(31)
    x = (rng.standard_normal((50, 128)) * np.exp(rng.uniform(-6, 4, (50, 1)))).astype(np.float32)
    x[3, 32:64] = 0.0                                   # a group of zeros
    q, s = int4.quantize(x)
    amax = np.abs(x.reshape(50, 4, 32)).max(-1)
    assert np.array_equal(s, np.float16(amax.astype(np.float32) / np.float32(7)).astype(np.float32))
    assert np.all(s[3, 1] == 0) and np.all(q[3, 32:64] == 0)
    cand = np.arange(-7, 8, dtype=np.float64)
    sx = np.repeat(s.astype(np.float64), 32, axis=-1)
    for i in range(50):
        for d in range(0, 128, 7):
            if sx[i, d] == 0:
                continue
            err = np.abs(np.float64(np.float32(x[i, d]) / np.float32(sx[i, d])) - cand)
            best = cand[err == err.min()]
            want = best[0] if len(best) == 1 else best[(best % 2) == 0][0]
            assert q[i, d] == want, (i, d)
    big = np.abs(x.reshape(50, 4, 32)).argmax(-1)
    for i in range(50):
        for g in range(4):
            if s[i, g] > 0:
                assert abs(int(q[i, g * 32 + big[i, g]])) == 7


def test_int4_error_is_within_half_a_scale_step():
    rng = np.random.default_rng(32)
    x = rng.standard_normal((200, 128)).astype(np.float32)
    q, s = int4.quantize(x)
    err = np.abs(int4.dequantize(q, s) - x.astype(np.float64))
    # half a step, plus the fp16 rounding of the scale stretched over 7 steps
    bound = np.repeat(s.astype(np.float64), 32, axis=-1) * (0.5 + 7 * 2.0 ** -11) + 1e-30
    assert np.all(err <= bound)


def test_zero_keys_give_uniform_mean_of_visible_values():
    # flags on even positions, w = 3, t = 10: the visible set is the odd
    # positions plus the last three (8, 9, 10)
    t, w = 10, 3
    evict = np.array([1 - (j % 2) for j in range(t + 1)], dtype=np.uint8)
    expect_vis = [1, 3, 5, 7, 8, 9, 10]
    rng = np.random.default_rng(4)
    V = rng.standard_normal((t + 1, 1, 6))
    K = np.zeros((t + 1, 1, 6))
    q = rng.standard_normal((2, 6))
    got = attention.decode_attention(q, K, V, evict[:, None], t, w, 1.0)
    np.testing.assert_allclose(got, np.tile(V[expect_vis, 0].mean(axis=0), (2, 1)), atol=1e-14)


def test_one_hot_values_read_off_attention_weights():
    rng = np.random.default_rng(5)
    t, w, D = 11, 4, 12            # D >= t+1 so value j is the unit vector e_j
    evict = (rng.random(t + 1) < 0.5).astype(np.uint8)
    K = rng.standard_normal((t + 1, 1, D))
    V = np.eye(D)[: t + 1][:, None, :]
    q = rng.standard_normal((1, D))
    o = attention.decode_attention(q, K, V, evict[:, None], t, w, 0.5)[0]
    vis = operational_cache_sets(evict, w)[t]
    s = 0.5 * K[vis, 0] @ q[0]
    p = np.exp(s - s.max())
    p /= p.sum()
    expect = np.zeros(D)
    expect[vis] = p
    np.testing.assert_allclose(o, expect, atol=1e-14)
    hidden = [j for j in range(t + 1) if j not in vis]
    assert np.all(o[hidden] == 0.0)


def test_single_visible_key_returns_its_value_exactly():
    rng = np.random.default_rng(6)
    t = 9
    q, K, V = rand_case(rng, t + 1, Hq=4, Hkv=1, D=8)
    evict = np.ones((t + 1, 1), dtype=np.uint8)
    got = attention.decode_attention(q, K, V, evict, t, 1, 0.9)
    assert np.array_equal(got, np.tile(V[t, 0], (4, 1)))


@pytest.mark.parametrize("w", [1, 2, 3, 4])
def test_brute_force_visible_sets_match_operational_model(w):
    for P in range(1, 11):
        for bits in itertools.product((0, 1), repeat=P):
            evict = np.array(bits, dtype=np.uint8)
            op = operational_cache_sets(evict, w)
            for t in range(P):
                assert list(mask.visible_positions(t, evict, w)) == op[t]


# ---------------------------------------------------------------------------
# compaction and slot bookkeeping
# ---------------------------------------------------------------------------

def test_prefill_retained_count_closed_form():
    rng = np.random.default_rng(7)
    for P, w, p in [(256, 32, 0.85), (1000, 512, 0.9), (300, 512, 0.5), (1, 4, 1.0), (513, 512, 1.0)]:
        evict = (rng.random(P) < p).astype(np.uint8)
        kept = compaction.prefill_kept_positions(evict, w)
        older = max(0, P - w)
        assert len(kept) == min(P, w) + int((evict[:older] == 0).sum())
        assert list(kept) == operational_cache_sets(evict, w)[P - 1]


def test_prefill_slots_are_ranks_and_ring_holds_last_window():
    rng = np.random.default_rng(8)
    P, w = 200, 16
    evict = (rng.random(P) < 0.8).astype(np.uint8)
    slot = compaction.prefill_slots(evict, w)
    pos = sorted(slot)
    assert [slot[j] for j in pos] == list(range(len(pos)))
    ring = compaction.prefill_ring(evict, w)
    for j in range(P - w, P):
        assert ring[j % w] == (slot[j], int(evict[j]))
    short = compaction.prefill_ring(evict[:5], w)
    assert [e is None for e in short] == [False] * 5 + [True] * (w - 5)


@pytest.mark.parametrize("P,w,p,steps", [(64, 8, 0.7, 80), (5, 8, 0.9, 30), (40, 1, 1.0, 10),
                                         (100, 16, 0.0, 20)])
def test_decode_slots_follow_reuse_recurrence_and_hold_visible_set(P, w, p, steps):
    """slot(t) = slot(t-w) when token t-w was flagged, else the next new slot;
    the held positions are exactly the visible set, one slot each."""
    rng = np.random.default_rng(P * 131 + w)
    evict = (rng.random(P + steps) < p).astype(np.uint8)
    store = slots.HeadStore(evict[:P], w)
    slot_of = dict(compaction.prefill_slots(evict[:P], w))
    n_slots = len(slot_of)
    op = operational_cache_sets(evict, w)
    for t in range(P, P + steps):
        expect = slot_of[t - w] if (t - w >= 0 and evict[t - w]) else n_slots
        if expect == n_slots:
            n_slots += 1
        s = store.append(t, int(evict[t]))
        slot_of[t] = s
        assert s == expect
        assert store.n_slots == n_slots == store.n_retained
        assert list(store.positions()) == op[t]
        assert sorted(store.pos_of_slot) == list(range(store.n_slots))
        assert len(store.free) == 0


def test_llama_workload_compaction_matches_page_compression():
    """The 6.4x of the pages at ctx 8192 is 1280 kept tokens per head; the
    Llama-3.2-1B workload (keep 0.10, w 512) has exactly that expectation,
    and its seeded flags land within binomial error of it."""
    wl = configs.LLAMA1B_CTX8K
    P = PAGE["ctx_len"]["value"]
    assert wl.prompt == P and wl.window == PAGE["delay_window"]["value"]
    expect = wl.window + wl.p_keep * (P - wl.window)
    assert abs(expect - P / PAGE["compression_llama_3_2_1b"]["value"]) < 1e-9
    sigma = np.sqrt((P - wl.window) * wl.p_keep * (1 - wl.p_keep))
    counts = []
    for layer in range(wl.n_layers):
        for h in range(wl.n_kv_heads):
            flags = reference.head_flags(wl, layer, 0, h, P)
            counts.append(len(compaction.prefill_kept_positions(flags, wl.window)))
    counts = np.array(counts)
    assert np.all(np.abs(counts - expect) < 6 * sigma)
    assert abs(counts.mean() - expect) < 5 * sigma / np.sqrt(len(counts))


# ---------------------------------------------------------------------------
# FP8 E4M3 codec
# ---------------------------------------------------------------------------

ALL_CODES = np.arange(256, dtype=np.uint8)


def test_e4m3_golden_landmarks():
    for code, val in E4M3["codes"].items():
        got = fp8.e4m3_decode(np.uint8(int(code, 16)))
        assert got == val and np.signbit(got) == np.signbit(val)
    for code in E4M3["nan_codes"]:
        assert np.isnan(fp8.e4m3_decode(np.uint8(int(code, 16))))
    finite = fp8.e4m3_decode(ALL_CODES)
    finite = finite[~np.isnan(finite)]
    assert finite.max() == E4M3["max_finite"]
    assert np.abs(finite[finite != 0]).min() == E4M3["min_subnormal"]


def test_e4m3_decode_matches_torch_and_ml_dtypes():
    ml_dtypes = pytest.importorskip("ml_dtypes")
    ours = fp8.e4m3_decode(ALL_CODES)
    tt = torch.from_numpy(ALL_CODES.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ml = ALL_CODES.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for ref in (tt, ml):
        assert np.array_equal(np.isnan(ours), np.isnan(ref))
        ok = ~np.isnan(ours)
        assert np.array_equal(ours[ok], ref[ok])


def test_e4m3_encode_roundtrips_every_finite_code():
    vals = fp8.e4m3_decode(ALL_CODES)
    ok = ~np.isnan(vals)
    assert np.array_equal(fp8.e4m3_encode(vals[ok]), ALL_CODES[ok])


def test_e4m3_midpoints_round_to_even_and_match_torch():
    pos = np.sort(fp8.e4m3_decode(np.arange(0x7F, dtype=np.uint8)))
    mids = (pos[:-1] + pos[1:]) / 2
    codes = fp8.e4m3_encode(mids)
    assert np.all(codes % 2 == 0)                         # even mantissa wins the tie
    assert np.all((fp8.e4m3_decode(codes) == pos[:-1]) | (fp8.e4m3_decode(codes) == pos[1:]))
    tt = torch.from_numpy(mids.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, tt)
    neg = fp8.e4m3_encode(-mids)
    assert np.array_equal(neg, codes | 0x80)


def test_e4m3_encode_matches_torch_on_dense_fp32_grid():
    x = np.linspace(-448.0, 448.0, 2_000_001, dtype=np.float32)
    x = np.concatenate([x, np.float32(2.0) ** -np.arange(0, 12, 0.125).astype(np.float32)])
    tt = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(fp8.e4m3_encode(x), tt)


def test_e4m3_saturates_instead_of_nan():
    big = np.array([448.5, 463.9, 464.0, 470.0, 1e4, 3e38], dtype=np.float32)
    assert np.all(fp8.e4m3_encode(big) == 0x7E)
    assert np.all(fp8.e4m3_encode(-big) == 0xFE)
    assert fp8.e4m3_encode(np.float32(np.nan)) == 0x7F


def test_fp8_scale_and_fp32_quotient():
    assert fp8.fp8_scale(448.0) == 1.0 and fp8.fp8_scale(0.0) == 1.0
    assert fp8.fp8_scale(1.0) == np.float32(1.0) / np.float32(448.0)
    rng = np.random.default_rng(9)
    x = rng.standard_normal(100_000).astype(np.float32)
    s = fp8.fp8_scale(np.abs(x).max())
    y = torch.from_numpy(x) / torch.tensor(s, dtype=torch.float32)
    tt = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(fp8.quantize(x, s), tt)
    assert np.abs(fp8.dequantize(fp8.quantize(x, s), s)).max() <= np.abs(x).max()


# ---------------------------------------------------------------------------
# generator sanity (its bit-exact twin on the device is tested on the GPU)
# ---------------------------------------------------------------------------

def test_splitmix64_reference_sequence():
    """First outputs of SplitMix64 from state 0 (Vigna's splitmix64.c)."""
    assert [int(synth.hash64(0, n)) for n in (1, 2, 3)] == [
        0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_generator_moments_and_flag_rate():
    x = synth.normal_f32(5, synth.STREAM_K, 3, 1, np.arange(200_000), 2, 7)
    assert abs(x.mean()) < 5 / np.sqrt(x.size) and abs(x.var() - 1) < 0.02
    assert np.abs(x).max() <= 6.0
    xb = synth.normal(5, synth.STREAM_K, 3, 1, np.arange(1000), 2, 7, "bf16")
    assert np.array_equal(xb, torch.from_numpy(x[:1000]).to(torch.bfloat16).float().numpy())
    thr = synth.keep_threshold(0.1)
    f = synth.evict_flags(5, 0, 0, np.arange(200_000), 0, thr)
    assert abs((1 - f.mean()) - 0.1) < 5 * np.sqrt(0.09 / f.size)


def test_oracle_and_product_do_not_import_each_other():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for dirpath, _, files in os.walk(os.path.join(root, "oracle")):
        for f in files:
            if f.endswith(".py"):
                src = open(os.path.join(dirpath, f)).read()
                assert "compact_decode_attention_b200" not in src, f
    pkg = os.path.join(root, "compact_decode_attention_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f


# ---------------------------------------------------------------------------
# per-head glue of oracle/reference.py, against whole tensors drawn from the
# generator and library routines (torch SDPA, torch's float8 cast)
# ---------------------------------------------------------------------------

def _glue_workload(kv_dtype="bf16", in_dtype="bf16", head_dim=16):
    """Three layers, batch 3, GQA 4 and a keep probability drawn per
    (layer, kv-head), so a slip in the layer / sequence / head indexing of
    the glue picks other draws."""
    return configs.Workload("glue_pin", 3, 3, 12, 3, head_dim, 90, 8, 20, kv_dtype, in_dtype, 17,
                            "uniform", extra={"lo": 0.05, "hi": 0.9})


def _torch_fp8_store(x, scale):
    """Stored values of an FP8 store via torch: e4m3fn(x / scale) * scale, the
    quotient in fp32, saturated to +-448 before the cast (torch's cast gives
    NaN above 464; decode tokens may exceed the prompt's amax)."""
    y = torch.from_numpy(np.asarray(x, np.float32)) / torch.tensor(scale, dtype=torch.float32)
    y = torch.clamp(y, -448.0, 448.0)
    return y.to(torch.float8_e4m3fn).to(torch.float64).numpy() * np.float64(scale)


def test_glue_inputs_are_the_workload_tensors():
    """head_flags / head_input / head_query return slices of the whole-tensor
    draws of the same workload: (layer, sequence, kv-head) in the right
    places, the query rows of kv-head h being query heads h*g .. h*g+g-1."""
    wl = _glue_workload()
    thr = wl.thresholds()
    assert len(np.unique(thr)) == thr.size          # every (layer, head) draws its own rate
    n = 50
    for layer in range(wl.n_layers):
        K = synth.kv_tokens(wl.seed, 0, layer, wl.batch, 0, n, wl.n_kv_heads, wl.head_dim, "bf16")
        V = synth.kv_tokens(wl.seed, 1, layer, wl.batch, 0, n, wl.n_kv_heads, wl.head_dim, "bf16")
        F = synth.flag_tokens(wl.seed, layer, wl.batch, 0, n, wl.n_kv_heads, thr[layer])
        Q = synth.q_tokens(wl.seed, layer, wl.batch, 37, wl.n_q_heads, wl.head_dim, "bf16")
        for b in range(wl.batch):
            for h in range(wl.n_kv_heads):
                assert np.array_equal(reference.head_flags(wl, layer, b, h, n), F[b, :, h])
                assert np.array_equal(reference.head_input(wl, 0, layer, b, h, 5, 20), K[b, 5:25, h])
                assert np.array_equal(reference.head_input(wl, 1, layer, b, h, 0, n), V[b, :, h])
                g = wl.group
                assert np.array_equal(reference.head_query(wl, layer, b, h, 37), Q[b, h * g:(h + 1) * g])


def test_glue_fp8_scales_are_amax_over_every_sequence_and_prompt_row():
    """fp8_head_scales = amax / 448 over all batch rows and all prompt
    positions of the (layer, kv-head), before eviction; the decode tokens
    after the prompt do not count.  A small chunk size makes the amax loop
    cross chunk and sequence boundaries."""
    wl = _glue_workload("fp8")
    for layer in range(wl.n_layers):
        K = synth.kv_tokens(wl.seed, 0, layer, wl.batch, 0, wl.prompt, wl.n_kv_heads, wl.head_dim, "bf16")
        V = synth.kv_tokens(wl.seed, 1, layer, wl.batch, 0, wl.prompt, wl.n_kv_heads, wl.head_dim, "bf16")
        for h in range(wl.n_kv_heads):
            sk, sv = reference.fp8_head_scales(wl, layer, h, chunk=7)
            want_k = (torch.from_numpy(K[:, :, h]).abs().max() / 448.0).item()
            want_v = (torch.from_numpy(V[:, :, h]).abs().max() / 448.0).item()
            assert sk == np.float32(want_k) and sv == np.float32(want_v), (layer, h)
            # one sequence, or the rows after the prompt, give another amax
            one = np.float32(np.abs(K[0, :, h]).max() / np.float32(448))
            assert any(np.float32(np.abs(K[b, :, h]).max() / np.float32(448)) != sk
                       for b in range(wl.batch)) or one == sk


@pytest.mark.parametrize("kv_dtype", ["bf16", "fp8", "f32"])
def test_glue_expected_output_matches_sdpa_on_workload_tensors(kv_dtype):
    """expected_output for every (layer, sequence, kv-head) at a few decode
    positions equals torch's fp64 SDPA over the whole tensors of the
    workload, masked by the operational model of delayed eviction, with the
    store's values formed by torch (bf16 / fp32 inputs as drawn; FP8 through
    torch's e4m3fn cast with scales from torch's amax)."""
    in_dtype = "f32" if kv_dtype == "f32" else "bf16"
    wl = _glue_workload(kv_dtype, in_dtype)
    g, D, w = wl.group, wl.head_dim, wl.window
    thr = wl.thresholds()
    for layer in range(wl.n_layers):
        T = wl.prompt + wl.decode
        K = synth.kv_tokens(wl.seed, 0, layer, wl.batch, 0, T, wl.n_kv_heads, D, in_dtype)
        V = synth.kv_tokens(wl.seed, 1, layer, wl.batch, 0, T, wl.n_kv_heads, D, in_dtype)
        F = synth.flag_tokens(wl.seed, layer, wl.batch, 0, T, wl.n_kv_heads, thr[layer])
        scales = {}
        Ks, Vs = K.astype(np.float64), V.astype(np.float64)
        if kv_dtype == "fp8":
            for h in range(wl.n_kv_heads):
                sk = np.float32((torch.from_numpy(K[:, :wl.prompt, h]).abs().max() / 448.0).item())
                sv = np.float32((torch.from_numpy(V[:, :wl.prompt, h]).abs().max() / 448.0).item())
                scales[h] = (sk, sv)
                Ks[:, :, h] = _torch_fp8_store(K[:, :, h], sk)
                Vs[:, :, h] = _torch_fp8_store(V[:, :, h], sv)
        for t in (wl.prompt, wl.prompt + 3, T - 1):
            Q = synth.q_tokens(wl.seed, layer, wl.batch, t, wl.n_q_heads, D, in_dtype)
            for b in range(wl.batch):
                m = np.zeros((wl.n_kv_heads, t + 1), dtype=bool)
                for h in range(wl.n_kv_heads):
                    m[h, operational_cache_sets(F[b, :t + 1, h], w)[t]] = True
                ref = sdpa(Q[b], Ks[b, :t + 1], Vs[b, :t + 1], 1.0 / np.sqrt(D), m)
                for h in range(wl.n_kv_heads):
                    got = reference.expected_output(wl, layer, b, h, t, scales=scales.get(h))
                    np.testing.assert_allclose(got, ref[h * g:(h + 1) * g], rtol=0, atol=1e-12,
                                               err_msg=f"{kv_dtype} layer {layer} seq {b} head {h} t {t}")


def test_glue_stored_rows_of_a_4bit_store_are_the_group_quantised_rows():
    """stored_rows of a 4-bit workload: each row is its own group-scaled
    4-bit rounding (brute force per element: the nearest multiple of the
    group's fp16 scale among -7..7)."""
    wl = _glue_workload("int4", head_dim=64)
    pos = np.array([0, 3, 40, 89])
    Kr, Vr = reference.stored_rows(wl, 1, 2, 1, pos)
    for stream, got in ((0, Kr), (1, Vr)):
        x = reference.head_input(wl, stream, 1, 2, 1, 0, wl.prompt)[pos]
        for i in range(len(pos)):
            for gq in range(wl.head_dim // 32):
                grp = x[i, 32 * gq:32 * gq + 32]
                s = np.float64(np.float16(np.float32(np.abs(grp).max()) / np.float32(7)))
                cand = np.arange(-7, 8) * s
                for d in range(32):
                    err = np.abs(cand - grp[d])
                    assert np.isclose(got[i, 32 * gq + d], cand[err.argmin()], rtol=0, atol=1e-12) or \
                        np.sum(err == err.min()) > 1


def test_glue_layer_scales_equal_the_per_head_scales():
    """fp8_layer_scales (one threaded pass over a layer) gives each head the
    scales fp8_head_scales takes chunk by chunk."""
    wl = _glue_workload("fp8")
    for layer in range(wl.n_layers):
        assert reference.fp8_layer_scales(wl, layer) == [
            reference.fp8_head_scales(wl, layer, h, chunk=11) for h in range(wl.n_kv_heads)]
