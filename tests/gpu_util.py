"""Test helpers: read the pool's bookkeeping back from the device and
undo the documented stored-row layouts (include/dms.h), then compare with
the oracle.  Nothing here computes attention or eviction."""
from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import fp8 as ofp8
from oracle import slots as oslots

BT = 64


def read_state(pool) -> dict:
    """Copy every bookkeeping region of the pool to host numpy arrays."""
    lay, cfg = pool.layout, pool.cfg
    nh = lay.n_heads

    def reg(name, dtype, count):
        return pool.region(name, dtype, count).cpu().numpy()

    hdr = reg("header", torch.int32, 8)
    return {
        "n_slots": reg("n_slots", torch.int32, nh),
        "n_retained": reg("n_retained", torch.int32, nh),
        "free_top": reg("free_top", torch.int32, nh),
        "ring": reg("ring", torch.int32, nh * cfg.window).view(np.uint32).reshape(nh, cfg.window),
        "ring_row": reg("ring_row", torch.int32, nh * cfg.window).reshape(nh, cfg.window),
        "last_block": reg("last_block", torch.int32, nh),
        "bt": reg("block_table", torch.int32, nh * lay.max_blocks_per_head).reshape(nh, -1),
        "scales": reg("scales", torch.float32, cfg.n_layers * cfg.n_kv_heads * 2).reshape(
            cfg.n_layers, cfg.n_kv_heads, 2),
        "next_block": int(hdr[0]), "block_stack_top": int(hdr[1]), "error": int(hdr[2]) & 0xFFFFFFFF,
    }


def head_id(cfg, layer, b, h):
    return (layer * cfg.max_batch + b) * cfg.n_kv_heads + h


def _unpermute_rows(raw: np.ndarray, rows: np.ndarray, kind: str, D: int, which: str) -> np.ndarray:
    """raw [n, tile-or-row bytes] stored bytes -> logical [n, D * esize] bytes."""
    n = raw.shape[0]
    if kind in ("f32", "bf16"):
        nch = raw.shape[1] // 16
        ch = np.arange(nch)[None, :] ^ (rows[:, None] & 7)          # physical chunk of logical c
        idx = (ch[:, :, None] * 16 + np.arange(16)[None, None, :]).reshape(n, -1)
        return np.take_along_axis(raw, idx, axis=1)
    # FP8, D = 128
    d = np.arange(D)
    if which == "K":
        pos = (((d & 7) >> 1) << 5) | ((d >> 4) << 2) | (((d >> 3) & 1) << 1) | (d & 1)
        byte = (((pos[None, :] >> 4) ^ (rows[:, None] & 7)) << 4) | (pos[None, :] & 15)
        return np.take_along_axis(raw, byte, axis=1)
    # V: transposed tile [D][64]; raw holds the whole tile of each row's block
    r = rows[:, None]
    off = d[None, :] * 64 + ((((r & 7) >> 1) << 4) | ((r >> 4) << 2) | (((r >> 3) & 1) << 1) | (r & 1))
    return np.take_along_axis(raw, off, axis=1)


def stored_rows(pool, state, hd: int, n: int, kind: str):
    """Logical bytes of the K and V rows held in slots 0..n-1 of head hd."""
    lay, cfg = pool.layout, pool.cfg
    D = cfg.head_dim
    esz = {"f32": 4, "bf16": 2, "fp8": 1}[kind]
    row_b = D * esz
    tile_b = BT * row_b
    slots = np.arange(n)
    blk = state["bt"][hd, slots // BT].astype(np.int64)
    rows = slots % BT
    base = torch.tensor(lay.blocks + blk * lay.block_bytes, device=pool.buffer.device)
    rows_t = torch.tensor(rows, device=pool.buffer.device)
    buf = pool.buffer
    k_off = base[:, None] + rows_t[:, None] * row_b + torch.arange(row_b, device=buf.device)[None, :]
    k_raw = buf[k_off].cpu().numpy()
    if kind == "fp8":
        v_off = base[:, None] + tile_b + torch.arange(tile_b, device=buf.device)[None, :]
    else:
        v_off = k_off + tile_b
    v_raw = buf[v_off].cpu().numpy()
    return (_unpermute_rows(k_raw, rows, kind, D, "K"), _unpermute_rows(v_raw, rows, kind, D, "V"))


def int4_rows(pool, state, hd: int, n: int):
    """Codes and scales held in slots 0..n-1 of head hd of a 4-bit store:
    (codes_k, scales_k, codes_v, scales_v), codes int8 [n, D] (nibble - 8),
    scales float32 [n, D / 32], undoing the DMS_INT4 layout of include/dms.h."""
    lay = pool.layout
    D = pool.cfg.head_dim
    tile = BT * (D // 2 + D // 16)
    nib = BT * D // 2
    slots = np.arange(n)
    blk = state["bt"][hd, slots // BT].astype(np.int64)
    rows = slots % BT
    raw = {}
    for b in np.unique(blk):
        o = int(lay.blocks + b * lay.block_bytes)
        raw[int(b)] = pool.buffer[o:o + 2 * tile].cpu().numpy()
    d = np.arange(D)
    kword = ((d & 7) >> 1) * 16 + (d >> 5) * 4                 # + row * 64
    kshift = 8 * ((d >> 4) & 1) + 4 * ((d >> 3) & 1) + 16 * (d & 1)
    ck = np.zeros((n, D), np.int8)
    cv = np.zeros((n, D), np.int8)
    sk = np.zeros((n, D // 32), np.float32)
    sv = np.zeros((n, D // 32), np.float32)
    for i in range(n):
        kt = raw[int(blk[i])][:tile]
        vt = raw[int(blk[i])][tile:]
        r = int(rows[i])
        kw = kt[:nib].view(np.uint32)[(r * 64 + kword) // 4]
        ck[i] = ((kw >> kshift.astype(np.uint32)) & 0xF).astype(np.int16) - 8
        vword = d * 32 + ((r & 7) >> 1) * 8 + (r >> 5) * 4
        vshift = 8 * ((r >> 4) & 1) + 4 * ((r >> 3) & 1) + 16 * (r & 1)
        vw = vt[:nib].view(np.uint32)[vword // 4]
        cv[i] = ((vw >> np.uint32(vshift)) & 0xF).astype(np.int16) - 8
        sk[i] = kt[nib:].view(np.float16).reshape(BT, D // 32)[r].astype(np.float32)
        sv[i] = vt[nib:].view(np.float16).reshape(D // 32, BT)[:, r].astype(np.float32)
    return ck, sk, cv, sv


def expected_row_bytes(values_f32: np.ndarray, kind: str, scale=None) -> np.ndarray:
    """Bytes the store should hold for rows given in input precision (float32 array)."""
    if kind == "f32":
        return np.ascontiguousarray(values_f32.astype(np.float32)).view(np.uint8).reshape(len(values_f32), -1)
    if kind == "bf16":
        bits = synth.f32_to_bf16_bits(values_f32)
        return np.ascontiguousarray(bits).view(np.uint8).reshape(len(values_f32), -1)
    return ofp8.quantize(values_f32, scale).reshape(len(values_f32), -1)


def oracle_store(prompt_flags: np.ndarray, decode_flags: np.ndarray, w: int, P: int):
    """Oracle head store after prefill and the given decode steps."""
    st = oslots.HeadStore(prompt_flags, w)
    for s, f in enumerate(decode_flags):
        st.append(P + s, int(f))
    return st


def check_head_store(pool, state, hd, store, rows_k_f32, rows_v_f32, kind, scales=None):
    """Bit-exact comparison of one head's counters, ring and stored rows with the oracle.

    rows_*_f32: dict position -> float32 row in input precision."""
    cfg = pool.cfg
    assert state["n_slots"][hd] == store.n_slots, (hd, state["n_slots"][hd], store.n_slots)
    assert state["n_retained"][hd] == store.n_retained
    assert state["free_top"][hd] == len(store.free)
    for idx, e in enumerate(store.ring):
        if e is not None:
            assert state["ring"][hd, idx] == (e[0] | (e[1] << 31)), (hd, idx)
            slot = e[0]
            assert state["ring_row"][hd, idx] == state["bt"][hd, slot // BT] * BT + slot % BT, (hd, idx)
    if store.n_slots > 0 and store.n_slots % BT:
        assert state["last_block"][hd] == state["bt"][hd, (store.n_slots - 1) // BT]
    n = store.n_slots
    got_k, got_v = stored_rows(pool, state, hd, n, kind)
    pos = [store.pos_of_slot[s] for s in range(n)]
    exp_k = expected_row_bytes(np.stack([rows_k_f32[p] for p in pos]), kind,
                               None if scales is None else scales[0])
    exp_v = expected_row_bytes(np.stack([rows_v_f32[p] for p in pos]), kind,
                               None if scales is None else scales[1])
    assert np.array_equal(got_k, exp_k), f"K rows differ for head {hd}"
    assert np.array_equal(got_v, exp_v), f"V rows differ for head {hd}"


def check_block_invariants(pool, state):
    """Physical blocks: in range, owned by exactly one (head, block index)."""
    ns = state["n_slots"]
    owned = []
    for hd in np.nonzero(ns)[0]:
        nb = (ns[hd] + BT - 1) // BT
        owned.append(state["bt"][hd, :nb])
    if not owned:
        return
    allb = np.concatenate(owned)
    assert allb.min() >= 0 and allb.max() < state["next_block"]
    assert len(np.unique(allb)) == len(allb), "a block is owned twice"
