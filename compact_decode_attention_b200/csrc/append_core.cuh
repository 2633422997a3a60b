// One decode step of one head of the compact store, shared by the append
// kernel and the fused projection epilogue.
//
// DMS delayed eviction: at step t the token leaving the window is t - w,
// found at ring index t mod w; when it was flagged its slot is pushed on the
// head's free stack and the new token takes the top of that stack, else the
// token takes slot n_slots, opening a new block when that slot starts one
// ("NVIDIA veröffentlicht Qwen3-8B-DMS-8x ..." (mindverse), section
// "Dynamic Memory Sparsification (DMS): Eine innovative Lösung"; slot reuse:
// "FastDMS: vLLM BF16/FP8보다 빠른 6.4x KV cache 압축" (molayo1419.me),
// opening paragraphs).
#pragma once

#include "dms_internal.cuh"

namespace dms {

// Pop a block from the global free-block stack (blocks released by finished
// sequences); -1 when it is empty.  Only pops run during an append, so a
// successful compare-and-swap owns the entry below the old top.
__device__ __forceinline__ int pop_free_block(const PoolView& v) {
  int top = *reinterpret_cast<volatile int*>(&v.hdr->block_stack_top);
  while (top > 0) {
    const int prev = atomicCAS(&v.hdr->block_stack_top, top, top - 1);
    if (prev == top) return v.block_stack[top - 1];
    top = prev;
  }
  return -1;
}

struct AppendSlot {
  int slot;    // logical slot of token t, -1 when nothing may be written
  int prow;    // physical row (block * BT + row)
  int opened;  // the slot opened a new block
};

// Bookkeeping of token t (flag `flag`) for head hd = (layer l, sequence b,
// kv-head h); one thread.  All its loads are independent of each other.
__device__ __forceinline__ AppendSlot append_bookkeeping(const PoolView& v, int l, int b, int h,
                                                         int hd, int t, uint32_t flag) {
  AppendSlot r{-1, -1, 0};
  const int64_t ri = int64_t(hd) * v.w + t % v.w;
  int ns = v.n_slots[hd], nr = v.n_retained[hd], ft = v.free_top[hd];
  const int lb = v.last_block[hd];
  const uint32_t e = v.ring[ri];
  const int er = v.ring_row[ri];
  if (t >= v.w && (e >> 31)) {
    // token t - w retires; its slot is pushed on the LIFO free stack and
    // popped right back by the new token, so the pair is done in registers
    // and the row comes from the row ring
    if (ft < v.free_cap) {
      r.slot = int(e & 0x7fffffffu);
      r.prow = er;
      nr -= 1;
    } else {
      report_error(v.hdr, DMS_DEVERR_FREE_STACK_FULL, l, b, h);
    }
  } else if (ft > 0) {      // a slot freed earlier and not reused yet
    ft -= 1;
    r.slot = v.free_stack[int64_t(hd) * v.free_cap + ft];
    r.prow = v.bt[int64_t(hd) * v.mbh + r.slot / v.BT] * v.BT + r.slot % v.BT;
  } else if (ns / v.BT < v.mbh) {
    r.slot = ns;
    ns += 1;
    if (r.slot % v.BT == 0) {  // a new block: a released one, else a fresh one
      int id = pop_free_block(v);
      if (id < 0) id = atomicAdd(&v.hdr->next_block, 1);
      if (id < v.max_blocks) {
        v.bt[int64_t(hd) * v.mbh + r.slot / v.BT] = id;
        v.last_block[hd] = id;
        r.prow = id * v.BT;
        r.opened = 1;
      } else {
        report_error(v.hdr, DMS_DEVERR_BLOCKS_EXHAUSTED, l, b, h);
        r.slot = -1;
      }
    } else {
      r.prow = lb * v.BT + r.slot % v.BT;
    }
  } else {
    report_error(v.hdr, DMS_DEVERR_HEAD_TABLE_FULL, l, b, h);
  }
  if (r.slot >= 0 && !DMS_CHECK(r.prow >= 0 && r.prow < v.max_blocks * v.BT, v.hdr, 101, hd, r.prow))
    r.slot = -1;
  if (r.slot >= 0) {
    v.n_slots[hd] = ns;
    v.n_retained[hd] = nr + 1;
    v.free_top[hd] = ft;
    v.ring[ri] = uint32_t(r.slot) | (flag << 31);
    v.ring_row[ri] = r.prow;
  }
  return r;
}

// ---- 4-bit rows (DMS_INT4, head_dim 128) ----
// Scale of a group of 32: fp16(amax / 7) (fp32 quotient, nearest even,
// 65504 at most); code = clamp(rint(x / scale), -7, 7), kept as the nibble
// code + 8; scale 0 gives code 0.
__device__ __forceinline__ float int4_group_scale(float amax) {
  const float s = __half2float(__float2half_rn(__fdiv_rn(amax, 7.f)));
  return s > 65504.f ? 65504.f : s;
}
__device__ __forceinline__ uint32_t int4_nibble(float x, float scale) {
  if (!(scale > 0.f)) return 8u;
  const float r = fminf(fmaxf(rintf(__fdiv_rn(x, scale)), -7.f), 7.f);
  return uint32_t(int(r) + 8);
}

// One token's K and V rows into a 4-bit store (one warp): lane l holds
// elements 4l .. 4l+3 of each row (values in input precision).  K words and
// scales are written whole; V nibbles share 32-bit words with 7 other tokens
// of the block, so they are cleared and set with atomics -- or, with
// s_vwords (a zeroed shared-memory image of the block's 1024 V nibble words),
// OR-ed into that image for the caller to write out.
// store_row_int4_at writes row `row` of the block image at blk (global
// memory, or a shared-memory stage: the atomics work on either).
__device__ __forceinline__ void store_row_int4_at(uint8_t* blk, int row, int64_t tile_bytes,
                                                  const float (&k4)[4], const float (&v4)[4],
                                                  int lane, uint32_t* s_vwords = nullptr) {
  uint8_t* vt = blk + tile_bytes;
  // group of lane l: elements 4l.. lie in group l / 8; amax over its 8 lanes
  float ka = fmaxf(fmaxf(fabsf(k4[0]), fabsf(k4[1])), fmaxf(fabsf(k4[2]), fabsf(k4[3])));
  float va = fmaxf(fmaxf(fabsf(v4[0]), fabsf(v4[1])), fmaxf(fabsf(v4[2]), fabsf(v4[3])));
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    ka = fmaxf(ka, __shfl_xor_sync(0xffffffffu, ka, o));
    va = fmaxf(va, __shfl_xor_sync(0xffffffffu, va, o));
  }
  const float ks = int4_group_scale(ka), vs = int4_group_scale(va);
  uint32_t c16 = 0;                  // the lane's four K nibbles, element 4l + i at bits 4i
#pragma unroll
  for (int i = 0; i < 4; ++i) c16 |= int4_nibble(k4[i], ks) << (4 * i);
  // K word (owner q, word kw) for lanes 0..15: element d = 32kw + 16j + 8hi + 2q + lo
  // comes from lane 8kw + 4j + 2hi + q/2, nibble 2(q&1) + lo
  uint32_t word = 0;
  const int q = (lane >> 2) & 3, kw = lane & 3;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
#pragma unroll
    for (int hi = 0; hi < 2; ++hi) {
      const int src = lane < 16 ? 8 * kw + 4 * j + 2 * hi + (q >> 1) : lane;
      const uint32_t pair = (__shfl_sync(0xffffffffu, c16, src) >> (8 * (q & 1))) & 0xFFu;
      word |= (pair & 0xFu) << (8 * j + 4 * hi);
      word |= (pair >> 4) << (8 * j + 4 * hi + 16);
    }
  }
  if (lane < 16) *reinterpret_cast<uint32_t*>(blk + row * 64 + q * 16 + kw * 4) = word;
  if ((lane & 7) == 0) {
    *reinterpret_cast<__half*>(blk + int4k_scale(row, lane >> 3)) = __float2half_rn(ks);
    *reinterpret_cast<__half*>(vt + int4v_scale(row, lane >> 3)) = __float2half_rn(vs);
  }
  const int sh = int4v_shift(row);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (s_vwords) {
      atomicOr(s_vwords + (int4v_word(4 * lane + i, row) >> 2), int4_nibble(v4[i], vs) << sh);
    } else {
      uint32_t* w = reinterpret_cast<uint32_t*>(vt + int4v_word(4 * lane + i, row));
      atomicAnd(w, ~(0xFu << sh));
      atomicOr(w, int4_nibble(v4[i], vs) << sh);
    }
  }
}

__device__ __forceinline__ void store_row_int4(const PoolView& v, int prow, const float (&k4)[4],
                                               const float (&v4)[4], int lane,
                                               uint32_t* s_vwords = nullptr) {
  store_row_int4_at(v.blocks + int64_t(prow / v.BT) * v.block_bytes, prow % v.BT, v.tile_bytes, k4,
                    v4, lane, s_vwords);
}

// Store one token's K and V rows, given as float values already rounded to
// the store's input precision, into physical row prow (one warp).  bf16 and
// fp32 stores copy the values; an FP8 store quantises them with the layer's
// scales (E4M3 of x / scale, nearest even, saturating), a 4-bit store with
// per-group scales; both clear the block's transposed V tile first when the
// token opened its block.
__device__ __forceinline__ void store_row_from_float(const PoolView& v, int l, int h, int prow,
                                                     int opened, const float* krow,
                                                     const float* vrow, int lane) {
  const int row = prow % v.BT;
  uint8_t* blk = v.blocks + int64_t(prow / v.BT) * v.block_bytes;
  if (v.kv_dtype == DMS_INT4) {
    if (opened) {   // tokens past the last one of a new block decode to 0
      uint4* tile = reinterpret_cast<uint4*>(blk + v.tile_bytes);
      for (int c = lane; c < int(v.tile_bytes / 16); c += 32) tile[c] = make_uint4(0, 0, 0, 0);
      __syncwarp();
    }
    float k4[4], v4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      k4[i] = krow[4 * lane + i];
      v4[i] = vrow[4 * lane + i];
    }
    store_row_int4(v, prow, k4, v4, lane);
    return;
  }
  if (v.kv_dtype == DMS_FP8_E4M3) {
    if (opened) {
      uint4* tile = reinterpret_cast<uint4*>(blk + v.tile_bytes);
      for (int c = lane; c < int(v.tile_bytes / 16); c += 32) tile[c] = make_uint4(0, 0, 0, 0);
      __syncwarp();
    }
    const float sK = v.scales[(int64_t(l) * v.Hkv + h) * 2 + 0];
    const float sV = v.scales[(int64_t(l) * v.Hkv + h) * 2 + 1];
    for (int d = lane; d < v.D; d += 32) {
      blk[fp8k_byte(row, d)] = f32_to_e4m3(__fdiv_rn(krow[d], sK));
      blk[v.tile_bytes + fp8v_byte(row, d)] = f32_to_e4m3(__fdiv_rn(vrow[d], sV));
    }
    return;
  }
  const int esz = v.kv_dtype == DMS_F32 ? 4 : 2;
  for (int d = lane; d < v.D; d += 32) {
    const int c = d * esz / 16, within = (d * esz) % 16;
    const int64_t off = int64_t(row) * v.row_bytes + swz_chunk(c, row) * 16 + within;
    if (esz == 4) {
      *reinterpret_cast<float*>(blk + off) = krow[d];
      *reinterpret_cast<float*>(blk + v.tile_bytes + off) = vrow[d];
    } else {
      *reinterpret_cast<__nv_bfloat16*>(blk + off) = __float2bfloat16_rn(krow[d]);
      *reinterpret_cast<__nv_bfloat16*>(blk + v.tile_bytes + off) = __float2bfloat16_rn(vrow[d]);
    }
  }
}

template <typename T>
__device__ __forceinline__ float in_to_f32(T x);
template <>
__device__ __forceinline__ float in_to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float in_to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

// One decode step of one head, one warp: token t (flag `flag`, valid in
// lane 0) of head hd = (layer l, sequence b, kv-head h) with input rows
// krow, vrow (D elements each, 16-byte aligned).  Lane 0 does the
// bookkeeping; all lanes load the new rows first (they do not depend on the
// bookkeeping) and store them once the destination is known.
// STORE: 0 = copy (bf16 / fp32 store, input in the store's dtype), 1 = FP8,
// 2 = 4-bit.
template <typename InT, int STORE>
__device__ __forceinline__ void append_head_warp(const PoolView& v, int l, int b, int h, int hd, int t,
                                                 const InT* krow, const InT* vrow, uint32_t flag,
                                                 int lane) {
  // ---- new rows into registers (bf16/fp32: 16-byte chunks, K then V) ----
  const int nch = int(v.row_bytes >> 4);       // chunks per row: 8, 16 or 32
  constexpr int kMaxPerLane = 2;               // 2 * 32 chunks per lane pair covers fp32 D=128
  uint4 chunk[kMaxPerLane];
  if constexpr (STORE == 0) {
#pragma unroll
    for (int r = 0; r < kMaxPerLane; ++r) {
      const int c = lane + 32 * r;
      if (c < 2 * nch) {
        const uint8_t* src = reinterpret_cast<const uint8_t*>(c < nch ? krow : vrow) + (c % nch) * 16;
        chunk[r] = *reinterpret_cast<const uint4*>(src);
      }
    }
  }

  // ---- bookkeeping (lane 0; all its loads are independent) ----
  int slot = -1, prow = -1, opened = 0;
  if (lane == 0) {
    const AppendSlot r = append_bookkeeping(v, l, b, h, hd, t, flag);
    slot = r.slot;
    prow = r.prow;
    opened = r.opened;
  }
  slot = __shfl_sync(0xffffffffu, slot, 0);
  prow = __shfl_sync(0xffffffffu, prow, 0);
  opened = __shfl_sync(0xffffffffu, opened, 0);
  if (slot < 0) return;
  const int row = prow % v.BT;
  uint8_t* blk = v.blocks + int64_t(prow / v.BT) * v.block_bytes;

  // ---- store the row ----
  if constexpr (STORE == 2) {
    if (opened) {   // tokens past the last one of a new block decode to 0
      uint4* tile = reinterpret_cast<uint4*>(blk + v.tile_bytes);
      for (int c = lane; c < int(v.tile_bytes / 16); c += 32) tile[c] = make_uint4(0, 0, 0, 0);
      __syncwarp();
    }
    float k4[4], v4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      k4[e] = in_to_f32(krow[4 * lane + e]);
      v4[e] = in_to_f32(vrow[4 * lane + e]);
    }
    store_row_int4(v, prow, k4, v4, lane);
  } else if constexpr (STORE == 0) {
#pragma unroll
    for (int r = 0; r < kMaxPerLane; ++r) {
      const int c = lane + 32 * r;
      if (c < 2 * nch) {
        uint8_t* dst = blk + (c < nch ? 0 : v.tile_bytes) + int64_t(row) * v.row_bytes +
                       swz_chunk(c % nch, row) * 16;
        *reinterpret_cast<uint4*>(dst) = chunk[r];
      }
    }
  } else {
    // a block opened by this step gets its transposed V tile cleared first,
    // so token columns not yet written decode to 0 (the attention kernel
    // reads whole V tiles)
    if (opened) {
      uint4* tile = reinterpret_cast<uint4*>(blk + v.tile_bytes);
      for (int c = lane; c < int(v.tile_bytes / 16); c += 32) tile[c] = make_uint4(0, 0, 0, 0);
      __syncwarp();
    }
    const float sK = v.scales[(int64_t(l) * v.Hkv + h) * 2 + 0];
    const float sV = v.scales[(int64_t(l) * v.Hkv + h) * 2 + 1];
    if (lane < 8) {            // K: lane lc fills 16-byte chunk lc of the permuted row
      const int lc = lane;
      uint8_t codes[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int p = lc * 16 + e;
        const int d = ((p >> 2) & 7) * 16 + ((p >> 1) & 1) * 8 + (p >> 5) * 2 + (p & 1);
        codes[e] = f32_to_e4m3(__fdiv_rn(in_to_f32(krow[d]), sK));
      }
      *reinterpret_cast<uint4*>(blk + row * 128 + ((lc ^ (row & 7)) << 4)) =
          *reinterpret_cast<const uint4*>(codes);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {  // V: 4 elements per lane into the transposed tile
      const int d = lane * 4 + e;
      blk[v.tile_bytes + fp8v_byte(row, d)] = f32_to_e4m3(__fdiv_rn(in_to_f32(vrow[d]), sV));
    }
  }
}

}  // namespace dms
