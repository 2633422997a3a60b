"""dms_project_append: the K/V projection of a decode token with the eviction
decision and the append fused into its epilogue (through the C ABI).

The kernel accumulates in fp32 and rounds k and v to bf16; the oracle rounds
the exact (fp64) projection.  The two can differ by one bf16 ulp where the
exact value lies within fp32 rounding of a bf16 midpoint, so stored rows are
compared within one ulp; the eviction decision is compared wherever the
logit is clear of the threshold by more than fp32 accumulation can move it
(1e-3 of sum |x w|), and the flags the kernel took are read back from the
window ring and fed to the oracle's slot simulator, which must then agree
with the store bit for bit.  Attention over the projected tokens is compared
with the fp64 oracle as everywhere (2e-2 bf16, 6e-2 FP8)."""
import numpy as np
import pytest
import torch

import synth
from oracle import attention as oatt
from oracle import fp8 as ofp8
from oracle import projection as oproj
from compact_decode_attention_b200 import dms

from gpu_util import check_block_invariants, head_id, oracle_store, read_state, stored_rows

pytestmark = pytest.mark.gpu


def _bf16_values(a):
    return oproj.bf16_round(np.asarray(a, np.float64))


def _dev(a, dt=torch.bfloat16):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dt).cuda()


@pytest.mark.parametrize("kind", ["bf16", "fp8"])
def test_projected_tokens_match_the_oracle(kind):
    L, Bmax, Hq, Hkv, D, w, dm, P, S = 1, 3, 8, 2, 128, 16, 320, 40, 20
    rng = np.random.default_rng(61)
    pool = dms.Pool(L, Bmax, Hq, Hkv, D, w, dms.DMS_BF16 if kind == "bf16" else dms.DMS_FP8_E4M3, 64, P + S + 1)
    W = _bf16_values(rng.standard_normal((dm, 2 * Hkv * D)) / np.sqrt(dm))
    we = _bf16_values(rng.standard_normal((dm, Hkv)) / np.sqrt(dm))
    be = (rng.standard_normal(Hkv) * 0.1).astype(np.float32)
    Wd, wed, bed = _dev(W), _dev(we), torch.from_numpy(be).cuda()
    slots = [2, 0]
    hist = []
    for j, slot in enumerate(slots):                   # prompts of their own
        K = synth.kv_tokens(70 + j, 0, 0, 1, 0, P, Hkv, D, "bf16")[0]
        V = synth.kv_tokens(70 + j, 1, 0, 1, 0, P, Hkv, D, "bf16")[0]
        F = synth.flag_tokens(70 + j, 0, 1, 0, P, Hkv, [synth.keep_threshold(0.4)] * Hkv)[0]
        pool.compact_prefill_seqs(0, slot, _dev(K[None]), _dev(V[None]), torch.from_numpy(F[None].copy()).cuda())
        hist.append({"K": np.zeros((P + S, Hkv, D)), "V": np.zeros((P + S, Hkv, D)),
                     "F": np.zeros((P + S, Hkv), np.uint8)})
        hist[j]["K"][:P], hist[j]["V"][:P], hist[j]["F"][:P] = K, V, F
    sc = read_state(pool)["scales"][0].astype(np.float64)      # FP8: set by the first prefill

    def stored_values(j, t):
        K, V = hist[j]["K"][:t + 1], hist[j]["V"][:t + 1]
        if kind == "bf16":
            return K, V
        Ks = np.stack([ofp8.dequantize(ofp8.quantize(K[:, h], sc[h, 0]), sc[h, 0]) for h in range(Hkv)], 1)
        Vs = np.stack([ofp8.dequantize(ofp8.quantize(V[:, h], sc[h, 1]), sc[h, 1]) for h in range(Hkv)], 1)
        return Ks, Vs

    ids = torch.tensor(slots, dtype=torch.int32, device="cuda")
    decided = 0
    for step in range(S):
        t = P + step
        X = _bf16_values(rng.standard_normal((len(slots), dm)))
        pos = torch.full((len(slots),), t, dtype=torch.int64, device="cuda")
        pool.project_append(0, ids, pos, _dev(X), Wd, wed, bed, 0.0)
        state = read_state(pool)
        for j, slot in enumerate(slots):
            k, v, lg = oproj.project_token(X[j], W, we, be, Hkv, D)
            hist[j]["K"][t], hist[j]["V"][t] = oproj.bf16_round(k), oproj.bf16_round(v)
            for h in range(Hkv):
                took = int(state["ring"][head_id(pool.cfg, 0, slot, h), t % w] >> 31)
                if abs(lg[h]) > 1e-3 * float(np.abs(X[j]) @ np.abs(we[:, h])):
                    assert took == int(lg[h] > 0.0), (step, j, h, lg[h])
                    decided += 1
                hist[j]["F"][t, h] = took
        q = rng.standard_normal((1, len(slots), Hq, D))
        out = torch.empty(1, len(slots), Hq, D, dtype=torch.bfloat16, device="cuda")
        pool.decode_attn_seqs(0, ids, _dev(q), out)
        got = out.float().cpu().numpy()
        for j in range(len(slots)):
            Ks, Vs = stored_values(j, t)
            exp = oatt.decode_attention(_bf16_values(q[0, j]), Ks, Vs, hist[j]["F"][:t + 1], t, w)
            assert np.abs(got[0, j] - exp).max() < (2e-2 if kind == "bf16" else 6e-2), (step, j)
    assert decided > 0.9 * S * len(slots) * Hkv
    # bookkeeping bit-exact given the flags; bf16 rows within one ulp of the exact projection
    state = read_state(pool)
    assert state["error"] == 0
    for j, slot in enumerate(slots):
        for h in range(Hkv):
            hd = head_id(pool.cfg, 0, slot, h)
            F = hist[j]["F"][:, h]
            store = oracle_store(F[:P], F[P:], w, P)
            assert state["n_slots"][hd] == store.n_slots and state["n_retained"][hd] == store.n_retained
            for idx, e in enumerate(store.ring):
                if e is not None:
                    assert state["ring"][hd, idx] == (e[0] | (e[1] << 31))
            if kind == "bf16":
                gk, gv = stored_rows(pool, state, hd, store.n_slots, "bf16")
                pos_of = np.array([store.pos_of_slot[s] for s in range(store.n_slots)])
                for got_b, ref in ((gk, hist[j]["K"][pos_of, h]), (gv, hist[j]["V"][pos_of, h])):
                    vals = synth.bf16_bits_to_f32(got_b.view(np.uint16)).astype(np.float64)
                    assert np.all(np.abs(vals - ref) <= np.abs(ref) * 2.0 ** -7 + 1e-30)
    check_block_invariants(pool, state)


def test_unsupported_shapes_are_refused():
    pool = dms.Pool(1, 1, 8, 2, 64, 16, dms.DMS_BF16, 16, 256)
    x = torch.zeros(1, 64, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(64, 2 * 2 * 64, dtype=torch.bfloat16, device="cuda")
    we = torch.zeros(64, 2, dtype=torch.bfloat16, device="cuda")
    pos = torch.zeros(1, dtype=torch.int64, device="cuda")
    with pytest.raises(dms.DmsError) as e:
        pool.project_append(0, None, pos, x, w, we)
    assert e.value.status == dms.DMS_ERR_UNSUPPORTED
