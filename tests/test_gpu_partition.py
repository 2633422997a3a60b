"""Decode attention over ragged, mixed batches: how the kernel cuts the
flat block list into CTA ranges (heads cut between CTAs, a CTA's range
starting with its last head, heads of one block and of many, sequence slots
with nothing stored) must not change any output.

Each case draws per (layer, kv-head) keep probabilities from window-only
(0), keep-all (1) and in between, gives every sequence its own prompt
length, decodes a few steps with each sequence at its own position, and
compares every output row with the fp64 oracle (2e-2, bf16).  A slot that
was never filled holds no key: its output rows are zero by definition."""
import numpy as np
import pytest
import torch

import synth
from oracle import attention as oatt
from compact_decode_attention_b200 import dms

from gpu_util import read_state

pytestmark = pytest.mark.gpu

TOL = 2e-2


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).cuda()


@pytest.mark.parametrize("seed,L,D", [(0, 1, 128), (1, 3, 128), (2, 2, 64), (3, 4, 128)])
def test_ragged_mixed_batches_match_the_oracle(seed, L, D):
    rng = np.random.default_rng(1000 + seed)
    Hkv, g, w, S = 4, 2, 64, 3
    Hq = Hkv * g
    n_seq = int(rng.integers(3, 7))
    empty = int(rng.integers(0, n_seq))              # one slot stays empty
    prompts = [int(x) for x in rng.integers(1, 2600, size=n_seq)]
    prompts[empty] = 0
    choice = rng.integers(0, 3, size=(L, Hkv))        # 0: window only, 1: keep all, 2: in between
    p_keep = np.where(choice == 0, 0.0, np.where(choice == 1, 1.0, rng.uniform(0.05, 0.6, (L, Hkv))))
    thr = [[synth.keep_threshold(p) for p in p_keep[layer]] for layer in range(L)]
    T = max(prompts) + S + 1
    blocks = L * n_seq * Hkv * (T // 64 + 2)
    pool = dms.Pool(L, n_seq, Hq, Hkv, D, w, dms.DMS_BF16, blocks, T)
    hist = {}
    for layer in range(L):
        for b in range(n_seq):
            P = prompts[b]
            n_pos = P + S
            K = synth.kv_tokens(seed + 13 * b, 0, layer, 1, 0, n_pos, Hkv, D, "bf16")[0]
            V = synth.kv_tokens(seed + 13 * b, 1, layer, 1, 0, n_pos, Hkv, D, "bf16")[0]
            F = synth.flag_tokens(seed + 7 * b, layer, 1, 0, n_pos, Hkv, thr[layer])[0]
            hist[layer, b] = (K, V, F)
            if P > 0:
                pool.compact_prefill_seqs(layer, b, _dev(K[None, :P]), _dev(V[None, :P]),
                                          torch.from_numpy(np.ascontiguousarray(F[None, :P])).cuda())
    live = [b for b in range(n_seq) if prompts[b] > 0]
    order = list(rng.permutation(live))               # call rows in an order of their own
    ids = torch.tensor(order, dtype=torch.int32, device="cuda")
    for s in range(S):
        pos = torch.tensor([prompts[b] + s for b in order], dtype=torch.int64, device="cuda")
        k = np.stack([np.stack([hist[layer, b][0][prompts[b] + s] for b in order]) for layer in range(L)])
        v = np.stack([np.stack([hist[layer, b][1][prompts[b] + s] for b in order]) for layer in range(L)])
        f = np.stack([np.stack([hist[layer, b][2][prompts[b] + s] for b in order]) for layer in range(L)])
        pool.append_evict_seqs(0, ids, pos, _dev(k), _dev(v), torch.from_numpy(np.ascontiguousarray(f)).cuda())
        q = np.stack([synth.q_tokens(seed + s, layer, len(order), 0, Hq, D, "bf16") for layer in range(L)])
        out = torch.empty(L, len(order), Hq, D, dtype=torch.bfloat16, device="cuda")
        pool.decode_attn_seqs(0, ids, _dev(q), out)
        got = out.float().cpu().numpy()
        for layer in range(L):
            for r, b in enumerate(order):
                K, V, F = hist[layer, b]
                t = prompts[b] + s
                exp = oatt.decode_attention(q[layer, r].astype(np.float64), K[:t + 1], V[:t + 1],
                                            F[:t + 1], t, w)
                assert np.abs(got[layer, r] - exp).max() < TOL, (seed, s, layer, b)
    # the empty slot: no key, output zero
    eid = torch.tensor([empty], dtype=torch.int32, device="cuda")
    q = np.stack([synth.q_tokens(seed + 99, layer, 1, 0, Hq, D, "bf16") for layer in range(L)])
    out = torch.full((L, 1, Hq, D), 7.0, dtype=torch.bfloat16, device="cuda")
    pool.decode_attn_seqs(0, eid, _dev(q), out)
    assert float(out.float().abs().max()) == 0.0
    assert read_state(pool)["error"] == 0
