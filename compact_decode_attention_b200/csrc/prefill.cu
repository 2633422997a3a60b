// dms_compact_prefill: stream compaction of one layer's prompt K/V into the
// compact store.
//
// At the end of a prompt of P tokens the last query sits at t = P - 1; the
// store keeps exactly the positions that query can see under DMS delayed
// eviction -- every token younger than the window w, and every older token
// that carries no evict flag ("NVIDIA veröffentlicht Qwen3-8B-DMS-8x ..."
// (mindverse), section "Dynamic Memory Sparsification (DMS): Eine innovative
// Lösung").  Evicted tokens are never written, so their memory is never
// taken (FastDMS page, opening paragraphs: compact store that reclaims
// evicted slots).  For an FP8 store the per-head scale is taken before
// eviction and the kept rows are quantised (FastDMS page, FP8 paragraph:
// eviction is decided before FP8 quantisation).
//
// Copy stores (bf16, fp32) take one launch instead, a cluster per
// (sequence, kv-head) (csrc/prefill_cluster.cu), for prompts up to 16384
// tokens.  FP8 and 4-bit stores, and longer prompts, take two kernels, in
// stream order:
//   plan     one CTA per (256-token chunk, sequence): per-head kept counts by
//            warp ballot + popcount (and, for an FP8 store, the per-head |x|
//            maximum of every prompt row).  The last CTA of a sequence to
//            finish turns its heads' chunk counts into exclusive prefix sums;
//            the last of those plans the layer: block allocation in
//            (sequence, head) order, block tables, counters, FP8 scales.
//            Arrival is counted with tickets, so no CTA ever waits.
//   scatter  one CTA per (64- or 256-token piece, kv-head, sequence),
//            launched as a programmatic dependent: it ranks its kept tokens
//            from the flags while the planner runs, then waits for the plan
//            and copies (or quantises) each kept row into its slot and fills
//            the window ring.  For FP8 and 4-bit stores the CTA holding the
//            last prompt token also clears the V rows past the head's last
//            slot in its last block (the attention reads whole V tiles).
#include "append_core.cuh"

namespace dms {

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

// Two adjacent input elements (p 4- or 8-byte aligned) as floats.
__device__ __forceinline__ void load_pair(const __nv_bfloat16* p, float& a, float& b) {
  const __nv_bfloat162 x = __ldg(reinterpret_cast<const __nv_bfloat162*>(p));
  a = __low2float(x);
  b = __high2float(x);
}
__device__ __forceinline__ void load_pair(const float* p, float& a, float& b) {
  const float2 x = __ldg(reinterpret_cast<const float2*>(p));
  a = x.x;
  b = x.y;
}

__device__ __forceinline__ bool keep_token(int j, int P, int w, uint8_t flag) {
  // visible to the last prompt query t = P - 1
  return j < P && (flag == 0 || (P - 1 - j) < w);
}

// ---------------------------------------------------------------------------
// Layer plan, run by the last CTA of the plan kernel (256 threads) once every
// sequence's chunk counts are scanned and pair_n holds each pair's kept count.
__device__ void plan_layer(const PoolView& v, int layer, int seq0, int batch) {
  __shared__ int s_fail;
  __shared__ int s_warp[8];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int pairs = batch * v.Hkv;
  const int stack = v.hdr->block_stack_top;
  const int next = v.hdr->next_block;
  if (tid == 0) s_fail = 0;
  __syncthreads();
  // the target heads must be empty and each head's blocks must fit its
  // table; blocks per pair -> exclusive prefix over pairs in (sequence, head)
  // order
  int running = 0;
  for (int p0 = 0; p0 < pairs; p0 += blockDim.x) {
    const int p = p0 + tid;
    int nb = 0;
    if (p < pairs) {
      const int hd = v.head(layer, seq0 + p / v.Hkv, p % v.Hkv);
      const int ns = v.n_slots[hd], nr = v.n_retained[hd], n = __ldcg(v.pair_n + p);
      nb = (n + v.BT - 1) / v.BT;
      if (ns != 0 || nr != 0) {
        atomicExch(&s_fail, 1);
        report_error(v.hdr, DMS_DEVERR_LAYER_NOT_EMPTY, layer, seq0 + p / v.Hkv, p % v.Hkv);
      }
      if (nb > v.mbh) {
        atomicExch(&s_fail, 1);
        report_error(v.hdr, DMS_DEVERR_HEAD_TABLE_FULL, layer, seq0 + p / v.Hkv, p % v.Hkv);
      }
    }
    int incl = nb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    int before = 0, all = 0;
    for (int q = 0; q < int(blockDim.x >> 5); ++q) {
      before += q < warp ? s_warp[q] : 0;
      all += s_warp[q];
    }
    if (p < pairs) v.pair_base[p] = running + before + incl - nb;
    running += all;
    __syncthreads();
  }
  const int total = running;
  if (tid == 0 && int64_t(total) > int64_t(stack) + (v.max_blocks - next)) {
    s_fail = 1;
    report_error(v.hdr, DMS_DEVERR_BLOCKS_EXHAUSTED, layer, -1, -1);
  }
  __syncthreads();   // pair_base visible to the whole CTA, s_fail final
  const bool ok = s_fail == 0;
  if (ok) {
    // block tables: allocation index a -> free stack top first, then bump
    for (int p = warp; p < pairs; p += blockDim.x >> 5) {
      const int hd = v.head(layer, seq0 + p / v.Hkv, p % v.Hkv);
      const int n = __ldcg(v.pair_n + p), base = __ldcg(v.pair_base + p);
      const int nb = (n + v.BT - 1) / v.BT;
      for (int k = lane; k < nb; k += 32) {
        const int a = base + k;
        v.bt[int64_t(hd) * v.mbh + k] = a < stack ? v.block_stack[stack - 1 - a] : next + (a - stack);
      }
      if (lane == 0) {
        v.n_slots[hd] = n;
        v.n_retained[hd] = n;
        v.free_top[hd] = 0;
        const int a = base + nb - 1;
        v.last_block[hd] = nb == 0 ? -1 : a < stack ? v.block_stack[stack - 1 - a] : next + (a - stack);
      }
    }
  }
  if (v.kv_dtype == DMS_FP8_E4M3) {
    // the first prefill into a layer sets its scales (0 = not set yet); later
    // prefills of other sequences reuse them, saturating like decode tokens.
    // The maxima are cleared for the next call either way.
    for (int i = tid; i < 2 * v.Hkv; i += blockDim.x) {
      const float a = __uint_as_float(__ldcg(v.amax + i));
      v.amax[i] = 0;
      if (!ok) continue;
      const float s = a > 0.f ? __fdiv_rn(a, 448.0f) : 1.0f;
      const int which = i / v.Hkv, h = i % v.Hkv;
      float* dst = v.scales + (int64_t(layer) * v.Hkv + h) * 2 + which;
      if (*dst == 0.f) *dst = s;
    }
  }
  if (tid == 0) {
    if (ok) {
      v.hdr->block_stack_top = stack > total ? stack - total : 0;
      v.hdr->next_block = next + (total > stack ? total - stack : 0);
    }
    v.hdr->prefill_go = ok ? 1 : 0;
  }
}

// ---------------------------------------------------------------------------
// One CTA of 256 threads per (256-token chunk, sequence).  AMAX: also fold
// every prompt row of the chunk into the per-head |x| maxima (FP8 store).
template <typename InT, bool AMAX>
__global__ void __launch_bounds__(256) prefill_plan_kernel(PoolView v, int layer, int seq0, int batch,
                                                           int P, const uint8_t* __restrict__ evict,
                                                           const InT* __restrict__ k,
                                                           const InT* __restrict__ vv) {
  extern __shared__ uint32_t s_amax[];   // [2][Hkv], AMAX only
  __shared__ int s_cnt[32][8];           // [head of a group of 32][warp]
  __shared__ int s_last;
  const int b = blockIdx.y, chunk = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = chunk * kPrefillChunk + tid;
  const int n_chunks = gridDim.x;
  if (chunk == 0 && b == 0) {   // warm L2 with what the planner reads cold
    for (int p = tid; p < batch * v.Hkv; p += blockDim.x) {
      const int hd = v.head(layer, seq0 + p / v.Hkv, p % v.Hkv);
      prefetch_l2(v.n_slots + hd);
      prefetch_l2(v.n_retained + hd);
    }
    if (tid == 0) prefetch_l2(v.hdr);
  }
  for (int h0 = 0; h0 < v.Hkv; h0 += 32) {
    const int nh = min(32, v.Hkv - h0);
    const uint8_t* fl = evict + (int64_t(b) * P + j) * v.Hkv + h0;
    uint8_t f[32];   // every flag load of the group in flight before the first ballot
#pragma unroll
    for (int hh = 0; hh < 32; ++hh) f[hh] = hh < nh && j < P ? __ldg(fl + hh) : 0;
#pragma unroll
    for (int hh = 0; hh < 32; ++hh) {
      if (hh < nh) {
        const unsigned m = __ballot_sync(0xffffffffu, keep_token(j, P, v.w, f[hh]));
        if (lane == 0) s_cnt[hh][warp] = __popc(m);
      }
    }
    __syncthreads();
    if (tid < nh) {
      int c = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) c += s_cnt[tid][q];
      v.chunk_counts[(int64_t(b) * v.Hkv + h0 + tid) * v.n_chunks_max + chunk] = c;
    }
    __syncthreads();
  }
  if constexpr (AMAX) {
    for (int i = tid; i < 2 * v.Hkv; i += blockDim.x) s_amax[i] = 0;
    __syncthreads();
    constexpr int VEC = 16 / sizeof(InT);
    constexpr int U = 4;                  // K and V vectors in flight per thread, each
    const int j0 = chunk * kPrefillChunk;
    const int nj = min(kPrefillChunk, P - j0);
    const int64_t row0 = (int64_t(b) * P + j0) * v.Hkv;  // first row of the chunk
    const int vec_per_row = v.D / VEC;
    const int nvec = nj * v.Hkv * vec_per_row;
    const uint4* srck = reinterpret_cast<const uint4*>(k + row0 * v.D);
    const uint4* srcv = reinterpret_cast<const uint4*>(vv + row0 * v.D);
    const int stride = blockDim.x;
    // vector i belongs to head (i / vec_per_row) mod Hkv: every vector of a
    // thread has the same head when the stride spans whole tokens
    const bool fixed = stride % (vec_per_row * v.Hkv) == 0;
    int cur = fixed ? (tid / vec_per_row) % v.Hkv : -1;
    float ak = 0.f, av = 0.f;
    const auto vmax = [](const uint4& raw) {
      const InT* x = reinterpret_cast<const InT*>(&raw);
      float m = 0.f;
#pragma unroll
      for (int e = 0; e < VEC; ++e) m = fmaxf(m, fabsf(to_f32(x[e])));
      return m;
    };
    for (int i0 = tid; i0 < nvec; i0 += U * stride) {
      uint4 rk[U], rv[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = i0 + u * stride;
        rk[u] = i < nvec ? __ldg(srck + i) : make_uint4(0, 0, 0, 0);   // zeros leave a maximum as it is
        rv[u] = i < nvec ? __ldg(srcv + i) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (!fixed) {
          const int hh = ((i0 + u * stride) / vec_per_row) % v.Hkv;
          if (hh != cur) {
            if (cur >= 0) {
              atomicMax(&s_amax[cur], __float_as_uint(ak));
              atomicMax(&s_amax[v.Hkv + cur], __float_as_uint(av));
            }
            cur = hh;
            ak = av = 0.f;
          }
        }
        ak = fmaxf(ak, vmax(rk[u]));
        av = fmaxf(av, vmax(rv[u]));
      }
    }
    if (cur >= 0) {
      atomicMax(&s_amax[cur], __float_as_uint(ak));
      atomicMax(&s_amax[v.Hkv + cur], __float_as_uint(av));
    }
    __syncthreads();
    for (int i = tid; i < 2 * v.Hkv; i += blockDim.x) atomicMax(&v.amax[i], s_amax[i]);
  }
  // arrival: the last CTA of this sequence scans its heads' chunk counts
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&v.prefill_tickets[b], 1) == n_chunks - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int h = warp; h < v.Hkv; h += blockDim.x >> 5) {
    int32_t* cc = v.chunk_counts + (int64_t(b) * v.Hkv + h) * v.n_chunks_max;
    int carry = 0;
    for (int c0 = 0; c0 < n_chunks; c0 += 32 * 8) {
      int x[8], own = 0;   // lane owns chunks c0 + 8 * lane .. + 7
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int c = c0 + 8 * lane + u;
        x[u] = c < n_chunks ? __ldcg(cc + c) : 0;
        own += x[u];
      }
      int incl = own;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int run = carry + incl - own;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int c = c0 + 8 * lane + u;
        if (c < n_chunks) cc[c] = run;
        run += x[u];
      }
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) v.pair_n[b * v.Hkv + h] = carry;
  }
  if (tid == 0) v.prefill_tickets[b] = 0;
  if (batch > 1) {
    // arrival: the last sequence to finish plans the layer
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&v.prefill_tickets[v.Bmax], 1) == batch - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (tid == 0) v.prefill_tickets[v.Bmax] = 0;
  } else {
    __threadfence();   // pair_n of the one sequence, written above, is read through L2
    __syncthreads();
  }
  pdl_launch_dependents();   // the scatter grid may be scheduled while the plan is made
  plan_layer(v, layer, seq0, batch);
}

// ---------------------------------------------------------------------------
// One CTA of 256 threads per (SPAN-token span, kv-head, sequence): a 64-token
// piece of a 256-token chunk (the pieces before it in the chunk give its
// offset) or a whole chunk.  STORE: 0 = copy (bf16 / fp32 store), 1 = FP8,
// 2 = 4-bit.
template <typename InT, int STORE, int SPAN>
__global__ void __launch_bounds__(256) prefill_scatter_kernel(PoolView v, int layer, int seq0, int P,
                                                              const InT* __restrict__ k,
                                                              const InT* __restrict__ vv,
                                                              const uint8_t* __restrict__ evict) {
  static_assert(kPrefillChunk % SPAN == 0 && SPAN % 32 == 0, "a span is whole warps of one chunk");
  constexpr int kPieces = kPrefillChunk / SPAN, kSpanWarps = SPAN / 32;
  constexpr int kBatchItems = 4;          // 16-byte copies in flight per thread
  __shared__ int s_kept[SPAN];            // chunk-local token index of each kept rank
  __shared__ int s_wcnt[8];
  // 4-bit store: V nibble words of the blocks the span's slots touch
  __shared__ uint32_t s_vw[STORE == 2 ? SPAN / 64 + 1 : 1][STORE == 2 ? kInt4Nibbles / 4 : 1];
  const int chunk = blockIdx.x / kPieces, piece = blockIdx.x % kPieces;
  const int h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = chunk * kPrefillChunk + threadIdx.x;
  const int64_t in_row_elems = v.D;
  // ranks from the flags (inputs only: this overlaps the planner)
  const uint8_t f = j < P ? __ldg(evict + (int64_t(b) * P + j) * v.Hkv + h) : 0;
  const bool keep = keep_token(j, P, v.w, f);
  const unsigned m = __ballot_sync(0xffffffffu, keep);
  if (lane == 0) s_wcnt[warp] = __popc(m);
  __syncthreads();
  const int w0 = piece * kSpanWarps;      // the span's first warp
  const bool mine = warp >= w0 && warp < w0 + kSpanWarps;
  int piece_base = 0, before = 0, nkept = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int c = s_wcnt[q];
    if (q < w0) {
      piece_base += c;
    } else if (q < w0 + kSpanWarps) {
      nkept += c;
      before += q < warp ? c : 0;
    }
  }
  const int rank = before + __popc(m & ((1u << lane) - 1u));
  if (mine && keep) s_kept[rank] = threadIdx.x;
  __syncthreads();                        // s_kept complete
  const auto src_row = [&](const InT* x, int kk) {
    return x + ((int64_t(b) * P + chunk * kPrefillChunk + s_kept[kk]) * v.Hkv + h) * in_row_elems;
  };
  // The inputs are ready before the plan: each thread loads its first source
  // data now, while the planner runs, and stores it once the slots are known.
  // copy: 16-byte chunks, kBatchItems of K and of V per thread in flight
  const int nch = int(v.row_bytes >> 4);
  const int n_items = STORE == 0 ? nkept * nch : STORE == 1 ? nkept * 8 : nkept;
  uint4 xk[kBatchItems], xv[kBatchItems];
  const auto load_copy = [&](int i0) {
#pragma unroll
    for (int u = 0; u < kBatchItems; ++u) {
      const int i = i0 + u * blockDim.x + threadIdx.x;
      if (i < n_items) {
        const int kk = i / nch, c = i % nch;
        xk[u] = __ldg(reinterpret_cast<const uint4*>(src_row(k, kk)) + c);
        xv[u] = __ldg(reinterpret_cast<const uint4*>(src_row(vv, kk)) + c);
      }
    }
  };
  // FP8 (D = 128): item i = 16 elements (chunk lc = i & 7) of kept row i >> 3.
  // K: stored byte e of chunk lc is element d = 64 (lc & 1) + 2 (lc >> 1)
  // + 16 (e >> 2) + 8 ((e >> 1) & 1) + (e & 1) (the fp8k_pos split): four
  // pairs of adjacent elements per 16-element block, loaded as pairs.
  // V: elements 16 lc .. 16 lc + 15, one 16-byte load per 16 bytes.
  constexpr int kVecs = 16 * int(sizeof(InT)) / 16;
  float kx[16];
  uint4 vraw[kVecs];
  const auto load_fp8 = [&](int i) {
    const int kk = i >> 3, lc = i & 7;
    const InT* srck = src_row(k, kk);
    const int dk0 = (lc & 1) * 64 + (lc >> 1) * 2;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
#pragma unroll
      for (int hi = 0; hi < 2; ++hi) load_pair(srck + dk0 + 16 * g + 8 * hi, kx[4 * g + 2 * hi], kx[4 * g + 2 * hi + 1]);
    }
#pragma unroll
    for (int u = 0; u < kVecs; ++u) vraw[u] = __ldg(reinterpret_cast<const uint4*>(src_row(vv, kk) + 16 * lc) + u);
  };
  // 4-bit: one warp per kept row, lane l holds elements 4l .. 4l+3
  float k4[4], v4[4];
  const auto load_int4 = [&](int kk) {
    const InT* srck = src_row(k, kk);
    const InT* srcv = src_row(vv, kk);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      k4[e] = to_f32(srck[4 * lane + e]);
      v4[e] = to_f32(srcv[4 * lane + e]);
    }
  };
  if constexpr (STORE == 0) load_copy(0);
  if constexpr (STORE == 1) {
    if (int(threadIdx.x) < n_items) load_fp8(threadIdx.x);
  }
  if constexpr (STORE == 2) {
    if (warp < n_items) load_int4(warp);
  }
  pdl_wait_prerequisites();               // the plan is complete and visible
  const int go = v.hdr->prefill_go;
  const int base = v.chunk_counts[(int64_t(b) * v.Hkv + h) * v.n_chunks_max + chunk] + piece_base;
  if (!go) return;
  const int hd = v.head(layer, seq0 + b, h);
  const int32_t* table = v.bt + int64_t(hd) * v.mbh;
  // prompt position of each kept slot (quantised stores: the prompt
  // attention gathers its old kept keys from the bf16 prompt by position)
  if (STORE != 0 && v.pos_of_slot && mine && keep)
    v.pos_of_slot[(int64_t(b) * v.Hkv + h) * (int64_t(v.mbh) * v.BT) + base + rank] = j;
  if (mine && keep && j >= P - v.w) {
    const int slot = base + rank;
    const int64_t ri = int64_t(hd) * v.w + (j % v.w);
    v.ring[ri] = uint32_t(slot) | (uint32_t(f != 0) << 31);
    v.ring_row[ri] = table[slot / v.BT] * v.BT + slot % v.BT;
  }
  if constexpr (STORE == 2) {
    // V nibbles: the span's slots [base, base + nkept) touch at most
    // SPAN / 64 + 1 blocks; their nibble words are built in shared memory
    // and written once each -- whole when every token of the word is this
    // CTA's, else with an AND / OR of this CTA's nibbles (neighbouring spans
    // own the other tokens).  In the head's last block the rows past the last
    // slot count as this CTA's (zero nibbles) when it holds the last token.
    constexpr int kWords = kInt4Nibbles / 4;           // V nibble words of a block (D = 128)
    const int kb0 = base / v.BT;
    const int nbt = nkept > 0 ? (base + nkept - 1) / v.BT - kb0 + 1 : 0;
    for (int i = threadIdx.x; i < nbt * kWords; i += blockDim.x) s_vw[i / kWords][i % kWords] = 0;
    __syncthreads();
    for (int kk = warp; kk < nkept; kk += blockDim.x / 32) {
      if (kk != warp) load_int4(kk);
      const int slot = base + kk;
      const int blk = table[slot / v.BT];
      if (!DMS_CHECK(blk >= 0 && blk < v.max_blocks, v.hdr, 202, hd, slot)) continue;
      store_row_int4(v, blk * v.BT + slot % v.BT, k4, v4, lane, s_vw[slot / v.BT - kb0]);
    }
    __syncthreads();
    const bool holds_last = int(blockIdx.x) == (P - 1) / SPAN;
    for (int i = threadIdx.x; i < nbt * kWords; i += blockDim.x) {
      const int kb = kb0 + i / kWords, d = (i % kWords) >> 3, wi = i & 7;
      const int lo = max(base, kb * v.BT) - kb * v.BT;
      const int hi = holds_last && kb == (base + nkept - 1) / v.BT ? v.BT - 1
                                                                  : min(base + nkept, (kb + 1) * v.BT) - 1 - kb * v.BT;
      uint32_t mask = 0;   // word wi of element row d: tokens 32 (wi & 1) + 16 e2 + 8 e1 + 2 (wi >> 1) + e0
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int t = (wi & 1) * 32 + ((e >> 2) & 1) * 16 + ((e >> 1) & 1) * 8 + (wi >> 1) * 2 + (e & 1);
        if (t >= lo && t <= hi) mask |= 0xFu << int4v_shift(t);
      }
      const int blk = table[kb];
      if (mask == 0 || !DMS_CHECK(blk >= 0 && blk < v.max_blocks, v.hdr, 204, hd, kb)) continue;
      uint32_t* w = reinterpret_cast<uint32_t*>(v.blocks + int64_t(blk) * v.block_bytes + v.tile_bytes +
                                                int4v_word(d, (wi & 1) * 32 + (wi >> 1) * 2));
      const uint32_t x = s_vw[i / kWords][i % kWords];
      if (mask == 0xFFFFFFFFu) {
        *w = x;
      } else {
        atomicAnd(w, ~mask);
        if (x) atomicOr(w, x);
      }
    }
  } else if constexpr (STORE == 0) {
    // bitwise row copy, 16-byte chunks swizzled by row
    for (int i0 = 0; i0 < n_items; i0 += kBatchItems * blockDim.x) {
      if (i0) load_copy(i0);
#pragma unroll
      for (int u = 0; u < kBatchItems; ++u) {
        const int i = i0 + u * blockDim.x + threadIdx.x;
        if (i >= n_items) break;
        const int kk = i / nch, c = i % nch;
        const int slot = base + kk;
        const int row = slot % v.BT;
        const int blk = table[slot / v.BT];
        if (DMS_CHECK(slot < v.mbh * v.BT && blk >= 0 && blk < v.max_blocks, v.hdr, 201, hd, slot)) {
          uint8_t* dst = v.blocks + int64_t(blk) * v.block_bytes + int64_t(row) * v.row_bytes + swz_chunk(c, row) * 16;
          *reinterpret_cast<uint4*>(dst) = xk[u];
          *reinterpret_cast<uint4*>(dst + v.tile_bytes) = xv[u];
        }
      }
    }
  } else {
    const float sK = v.scales[(int64_t(layer) * v.Hkv + h) * 2 + 0];
    const float sV = v.scales[(int64_t(layer) * v.Hkv + h) * 2 + 1];
    for (int i = threadIdx.x; i < n_items; i += blockDim.x) {
      if (i != int(threadIdx.x)) load_fp8(i);
      const int kk = i >> 3, lc = i & 7;
      const int slot = base + kk;
      const int row = slot % v.BT;
      uint8_t* blk = v.blocks + int64_t(table[slot / v.BT]) * v.block_bytes;
      const InT* vx = reinterpret_cast<const InT*>(vraw);
      uint8_t codes[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) codes[e] = f32_to_e4m3(__fdiv_rn(kx[e], sK));
      *reinterpret_cast<uint4*>(blk + row * 128 + ((lc ^ (row & 7)) << 4)) =
          *reinterpret_cast<const uint4*>(codes);
      // V tile transposed: one byte per element
#pragma unroll
      for (int e = 0; e < 16; ++e)
        blk[v.tile_bytes + fp8v_byte(row, 16 * lc + e)] = f32_to_e4m3(__fdiv_rn(to_f32(vx[e]), sV));
    }
  }
  if constexpr (STORE != 0) {
    // The piece holding the last prompt token holds the head's last slot n - 1
    // (the window keeps that token): zero the V rows past it in its block, so
    // those token columns decode to 0.  No other CTA writes those rows.
    const int n = base + nkept;
    const int r0 = n % v.BT;
    if (int(blockIdx.x) == (P - 1) / SPAN && r0 != 0) {
      const int blk_id = table[(n - 1) / v.BT];
      if (DMS_CHECK(blk_id >= 0 && blk_id < v.max_blocks, v.hdr, 203, hd, n)) {
        uint8_t* vt = v.blocks + int64_t(blk_id) * v.block_bytes + v.tile_bytes;
        if constexpr (STORE == 1) {
          for (int i = threadIdx.x; i < (v.BT - r0) * v.D; i += blockDim.x)
            vt[fp8v_byte(r0 + i / v.D, i % v.D)] = 0;
        } else {   // 4-bit: the nibbles of those rows were written as zeros above
          for (int i = threadIdx.x; i < (v.BT - r0) * (v.D / 32); i += blockDim.x)
            *reinterpret_cast<__half*>(vt + int4v_scale(r0 + i / (v.D / 32), i % (v.D / 32))) = __float2half_rn(0.f);
        }
      }
    }
  }
}

}  // namespace dms

using namespace dms;

namespace dms {
// The plan kernel (counts, prefix sums, block tables, counters, FP8 scales);
// shared with the fused prefill attention, which scatters the kept rows itself.
template <typename InT, bool AMAX>
static dms_status launch_plan(dms_pool* pool, int layer, int seq0, int batch, int prompt_len,
                              const uint8_t* evict, const void* k, const void* v, cudaStream_t stream) {
  const PoolView& pv = pool->view;
  const int n_chunks = (prompt_len + kPrefillChunk - 1) / kPrefillChunk;
  const size_t smem = AMAX ? sizeof(uint32_t) * 2 * pv.Hkv : 0;
  prefill_plan_kernel<InT, AMAX><<<dim3(n_chunks, batch), 256, smem, stream>>>(
      pv, layer, seq0, batch, prompt_len, evict, static_cast<const InT*>(k), static_cast<const InT*>(v));
  return cuda_status(cudaGetLastError(), "prefill_plan_kernel");
}

dms_status prefill_plan_launch(dms_pool* pool, int layer, int seq0, int batch, int prompt_len,
                               const uint8_t* evict, cudaStream_t stream) {
  return launch_plan<__nv_bfloat16, false>(pool, layer, seq0, batch, prompt_len, evict, nullptr, nullptr,
                                           stream);
}

template <typename InT, int STORE>
static dms_status launch_scatter(const dms_pool* pool, int layer, int seq0, int batch, int prompt_len,
                                 const void* k, const void* v, const uint8_t* evict, cudaStream_t stream) {
  const PoolView& pv = pool->view;
  const int n_chunks = (prompt_len + kPrefillChunk - 1) / kPrefillChunk;
  const int64_t ctas = int64_t(n_chunks) * pv.Hkv * batch;   // with 256-token spans
  // Short prompts: 64-token spans, so that the dense chunks (the window,
  // keep-all heads) spread over four CTAs each; from 16 x SMs CTAs on (four
  // rounds at four resident per SM) the dense ones balance out.  Spans of
  // several chunks measured slower: a CTA's copy rounds are serial.
  const bool small = ctas < int64_t(16) * pool->sm_count;
  const auto kk = static_cast<const InT*>(k);
  const auto vv = static_cast<const InT*>(v);
  cudaError_t e;
  if (small)
    e = launch_pdl(prefill_scatter_kernel<InT, STORE, 64>, dim3(n_chunks * 4, pv.Hkv, batch), dim3(256), 0,
                   stream, pv, layer, seq0, prompt_len, kk, vv, evict);
  else
    e = launch_pdl(prefill_scatter_kernel<InT, STORE, 256>, dim3(n_chunks, pv.Hkv, batch), dim3(256), 0,
                   stream, pv, layer, seq0, prompt_len, kk, vv, evict);
  return cuda_status(e, "prefill_scatter_kernel");
}
}  // namespace dms

extern "C" dms_status dms_compact_prefill(dms_pool* pool, int layer, int batch, int prompt_len,
                                          const void* k, const void* v, dms_dtype in_dtype,
                                          const uint8_t* evict, cudaStream_t stream) {
  return dms_compact_prefill_seqs(pool, layer, 0, batch, prompt_len, k, v, in_dtype, evict, stream);
}

extern "C" dms_status dms_compact_prefill_seqs(dms_pool* pool, int layer, int seq0, int batch,
                                               int prompt_len, const void* k, const void* v,
                                               dms_dtype in_dtype, const uint8_t* evict,
                                               cudaStream_t stream) {
  if (!pool) {
    set_last_error("null pool");
    return DMS_ERR_INVALID_ARG;
  }
  const PoolView& pv = pool->view;
  if (layer < 0 || layer >= pv.L || seq0 < 0 || batch < 1 || seq0 + batch > pv.Bmax ||
      prompt_len < 0 || prompt_len > pool->cfg.max_context) {
    set_last_error("bad layer/sequences/prompt_len (%d, %d+%d, %d)", layer, seq0, batch, prompt_len);
    return DMS_ERR_INVALID_ARG;
  }
  if (prompt_len == 0) return DMS_OK;
  if (!k || !v || !evict) {
    set_last_error("null input pointer");
    return DMS_ERR_INVALID_ARG;
  }
  const bool fp8 = pv.kv_dtype == DMS_FP8_E4M3, int4 = pv.kv_dtype == DMS_INT4;
  if (!(in_dtype == DMS_F32 || in_dtype == DMS_BF16) || (!fp8 && !int4 && int(in_dtype) != pv.kv_dtype)) {
    set_last_error("in_dtype %d does not match kv_dtype %d", int(in_dtype), pv.kv_dtype);
    return DMS_ERR_INVALID_ARG;
  }
  if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15) {
    set_last_error("k and v must be 16-byte aligned");
    return DMS_ERR_INVALID_ARG;
  }
  if (batch > 65535) {
    set_last_error("batch %d exceeds the 65535 sequences of one prefill launch", batch);
    return DMS_ERR_UNSUPPORTED;
  }
  const bool bf16 = in_dtype == DMS_BF16;
  if (!fp8 && !int4 && prompt_len <= prefill_cluster_max_prompt())   // copy stores: one launch
    return prefill_cluster_launch(pool, layer, seq0, batch, prompt_len, k, v, in_dtype, evict, stream);
  dms_status st;
  if (fp8)
    st = bf16 ? launch_plan<__nv_bfloat16, true>(pool, layer, seq0, batch, prompt_len, evict, k, v, stream)
              : launch_plan<float, true>(pool, layer, seq0, batch, prompt_len, evict, k, v, stream);
  else
    st = prefill_plan_launch(pool, layer, seq0, batch, prompt_len, evict, stream);
  if (st != DMS_OK) return st;
  if (bf16)
    return fp8 ? launch_scatter<__nv_bfloat16, 1>(pool, layer, seq0, batch, prompt_len, k, v, evict, stream)
         : int4 ? launch_scatter<__nv_bfloat16, 2>(pool, layer, seq0, batch, prompt_len, k, v, evict, stream)
                : launch_scatter<__nv_bfloat16, 0>(pool, layer, seq0, batch, prompt_len, k, v, evict, stream);
  return fp8 ? launch_scatter<float, 1>(pool, layer, seq0, batch, prompt_len, k, v, evict, stream)
       : int4 ? launch_scatter<float, 2>(pool, layer, seq0, batch, prompt_len, k, v, evict, stream)
              : launch_scatter<float, 0>(pool, layer, seq0, batch, prompt_len, k, v, evict, stream);
}
