"""The device's FP8-E4M3 encoder, through the store, on a dense grid of fp32
inputs (through the C ABI).

FastDMS quantises what eviction keeps ("FastDMS: vLLM BF16/FP8보다 빠른 6.4x
KV cache 압축" (molayo1419.me), paragraph after the speed table); the codes a
store holds must equal the oracle's software encoder (round to nearest even,
saturating to +-448) bit for bit.  A first prefill of sequence 0 sets each
head's scales from its own rows (amax / 448); a second prefill, of sequence
1, and decode appends of both reuse them.  Sequence 1 and the appends carry
the grid: a dense sweep of [-500, 500] (past +-448, so saturation is
exercised), every midpoint between neighbouring E4M3 values and the fp32
values just either side of it, the subnormal range, and signed zeros -- all
as fp32 inputs, the path that bf16 workloads never take.  With scale 1 the
quotient x / scale is x itself; with a scale that is not a power of two the
fp32 division is part of what must agree."""
import numpy as np
import pytest
import torch

from oracle import fp8 as ofp8
from compact_decode_attention_b200 import dms

from gpu_util import check_block_invariants, head_id, read_state, stored_rows

pytestmark = pytest.mark.gpu

B, HQ, HKV, D, P, S = 2, 8, 8, 128, 1024, 4


def _grid(n: int, scale: np.float32) -> np.ndarray:
    """n fp32 values whose quotients by `scale` cover the E4M3 grid densely."""
    pos = np.sort(ofp8.e4m3_decode(np.arange(0x7F, dtype=np.uint8)))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)           # exact in fp32
    up = np.nextafter(mids, np.float32(np.inf))
    down = np.nextafter(mids, np.float32(-np.inf))
    sub = np.linspace(0, 2.0 ** -6, 4097, dtype=np.float32)
    sat = np.linspace(440.0, 500.0, 4001, dtype=np.float32)
    special = np.array([0.0, -0.0, 448.0, 464.0, np.nextafter(np.float32(464), np.float32(0)),
                        2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -11], dtype=np.float32)
    core = np.concatenate([mids, up, down, sub, sat, special])
    core = np.concatenate([core, -core])
    dense = np.linspace(-500.0, 500.0, n - len(core), dtype=np.float32)
    q = np.concatenate([core, dense])
    rng = np.random.default_rng(5)
    q = q[rng.permutation(len(q))]
    # inputs whose fp32 quotient by `scale` lands on (or next to) the grid
    return (q.astype(np.float64) * np.float64(scale)).astype(np.float32)


@pytest.mark.parametrize("amax", [448.0, 0.7316])
def test_fp8_store_encodes_a_dense_grid_like_the_oracle(amax):
    amax = np.float32(amax)
    scale = ofp8.fp8_scale(amax)
    rng = np.random.default_rng(int(amax * 1000))
    pool = dms.Pool(1, B, HQ, HKV, D, 4 * (P + S), dms.DMS_FP8_E4M3, B * HKV * ((P + S) // 64 + 2),
                    P + S + 1)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()  # noqa: E731
    keep_all = torch.zeros(1, P, HKV, dtype=torch.uint8, device="cuda")
    # sequence 0: values within +-amax, each head's largest magnitude exactly amax
    x0 = (rng.uniform(-1, 1, size=(2, 1, P, HKV, D)) * amax).astype(np.float32)
    x0[:, 0, 7, :, 5] = amax
    x0[:, 0, 9, :, 6] = -amax
    pool.compact_prefill_seqs(0, 0, dev(x0[0]), dev(x0[1]), keep_all)
    state = read_state(pool)
    assert np.all(state["scales"][0, :, 0] == scale) and np.all(state["scales"][0, :, 1] == scale)
    # sequence 1 and the decode steps: the grid
    n = P * HKV * D
    g = _grid(2 * (n + S * B * HKV * D), scale)
    x1 = g[:2 * n].reshape(2, 1, P, HKV, D)
    xs = g[2 * n:].reshape(2, S, B, HKV, D)
    pool.compact_prefill_seqs(0, 1, dev(x1[0]), dev(x1[1]), keep_all)
    for s in range(S):
        pool.append_evict_layers(0, P + s, dev(xs[0, s][None]), dev(xs[1, s][None]),
                                 torch.zeros(1, B, HKV, dtype=torch.uint8, device="cuda"))
    state = read_state(pool)
    assert state["error"] == 0
    check_block_invariants(pool, state)
    for b in range(B):
        rows_k = np.concatenate([x0[0, 0] if b == 0 else x1[0, 0], xs[0, :, b]], axis=0)  # [P+S, Hkv, D]
        rows_v = np.concatenate([x0[1, 0] if b == 0 else x1[1, 0], xs[1, :, b]], axis=0)
        for h in range(HKV):
            hd = head_id(pool.cfg, 0, b, h)
            assert state["n_slots"][hd] == P + S                     # nothing evicted: slot j = position j
            got_k, got_v = stored_rows(pool, state, hd, P + S, "fp8")
            want_k = ofp8.quantize(rows_k[:, h], scale).reshape(P + S, D)
            want_v = ofp8.quantize(rows_v[:, h], scale).reshape(P + S, D)
            bad = np.argwhere(got_k != want_k)
            assert len(bad) == 0, (b, h, bad[:3], rows_k[:, h][tuple(bad[0])], got_k[tuple(bad[0])])
            bad = np.argwhere(got_v != want_v)
            assert len(bad) == 0, (b, h, bad[:3], rows_v[:, h][tuple(bad[0])], got_v[tuple(bad[0])])
    # saturation was exercised: some grid quotients lie past 448
    assert (np.abs(g.astype(np.float64) / np.float64(scale)) > 464).any()
