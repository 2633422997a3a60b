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
// Kernels, in stream order:
//   amax     (FP8 only) per-(kv-head) |x| maximum over every prompt row
//   count    per (sequence, 256-token chunk, head): warp ballot + popcount
//   plan     one CTA: per-head chunk prefix sums, block allocation in
//            (sequence, head) order, block tables, counters, FP8 scales
//   scatter  per (sequence, kv-head, chunk): ranks by ballot/popcount +
//            the chunk base give each kept row its slot; copy (or quantise)
//            the row into its block, fill the window ring.
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

__device__ __forceinline__ bool keep_token(int j, int P, int w, uint8_t flag) {
  // visible to the last prompt query t = P - 1
  return j < P && (flag == 0 || (P - 1 - j) < w);
}

// ---------------------------------------------------------------------------
template <typename InT>
__global__ void __launch_bounds__(256) prefill_amax_kernel(PoolView v, int P, const InT* k,
                                                           const InT* vv) {
  extern __shared__ uint32_t s_amax[];  // [2][Hkv]
  const int b = blockIdx.y;
  const int j0 = blockIdx.x * kPrefillChunk;
  const int nj = min(kPrefillChunk, P - j0);
  for (int i = threadIdx.x; i < 2 * v.Hkv; i += blockDim.x) s_amax[i] = 0;
  __syncthreads();
  constexpr int VEC = 16 / sizeof(InT);
  const int64_t row0 = (int64_t(b) * P + j0) * v.Hkv;  // first row of the chunk
  const int64_t nvec = int64_t(nj) * v.Hkv * v.D / VEC;
  for (int which = 0; which < 2; ++which) {
    const uint4* src = reinterpret_cast<const uint4*>((which ? vv : k) + row0 * v.D);
    for (int64_t i = threadIdx.x; i < nvec; i += blockDim.x) {
      uint4 raw = src[i];
      const InT* x = reinterpret_cast<const InT*>(&raw);
      float m = 0.f;
#pragma unroll
      for (int e = 0; e < VEC; ++e) m = fmaxf(m, fabsf(to_f32(x[e])));
      const int h = int((i * VEC / v.D) % v.Hkv);
      atomicMax(&s_amax[which * v.Hkv + h], __float_as_uint(m));
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 2 * v.Hkv; i += blockDim.x) atomicMax(&v.amax[i], s_amax[i]);
}

// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) prefill_count_kernel(PoolView v, int P, const uint8_t* evict) {
  __shared__ int s_cnt[8];
  const int b = blockIdx.y, chunk = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = chunk * kPrefillChunk + threadIdx.x;
  for (int h = 0; h < v.Hkv; ++h) {
    const uint8_t f = j < P ? evict[(int64_t(b) * P + j) * v.Hkv + h] : 0;
    const unsigned m = __ballot_sync(0xffffffffu, keep_token(j, P, v.w, f));
    if (lane == 0) s_cnt[warp] = __popc(m);
    __syncthreads();
    if (threadIdx.x == 0) {
      int c = 0;
      for (int k = 0; k < 8; ++k) c += s_cnt[k];
      v.chunk_counts[(int64_t(b) * v.Hkv + h) * v.n_chunks_max + chunk] = c;
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// One CTA of 1024 threads.  s_n holds the kept count of each (b, h) pair.
__global__ void __launch_bounds__(1024) prefill_plan_kernel(PoolView v, int layer, int seq0, int batch,
                                                            int P) {
  extern __shared__ int s_n[];   // [batch * Hkv] kept counts, then block prefix
  __shared__ int s_fail;
  __shared__ int s_warp[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  const int pairs = batch * v.Hkv;
  const int n_chunks = (P + kPrefillChunk - 1) / kPrefillChunk;
  if (tid == 0) {
    s_fail = 0;
    v.hdr->prefill_go = 0;
  }
  __syncthreads();
  // the target sequences of the layer must be empty
  for (int p = tid; p < pairs; p += blockDim.x) {
    const int hd = v.head(layer, seq0 + p / v.Hkv, p % v.Hkv);
    if (v.n_slots[hd] != 0 || v.n_retained[hd] != 0) {
      atomicExch(&s_fail, 1);
      report_error(v.hdr, DMS_DEVERR_LAYER_NOT_EMPTY, layer, seq0 + p / v.Hkv, p % v.Hkv);
    }
  }
  __syncthreads();
  if (s_fail) return;
  // per pair: exclusive scan of chunk counts (in place) and total
  for (int p = warp; p < pairs; p += nwarps) {
    int32_t* cc = v.chunk_counts + int64_t(p) * v.n_chunks_max;
    int carry = 0;
    for (int c0 = 0; c0 < n_chunks; c0 += 32) {
      const int c = c0 + lane;
      const int x = c < n_chunks ? cc[c] : 0;
      int incl = x;
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (c < n_chunks) cc[c] = carry + incl - x;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_n[p] = carry;
  }
  __syncthreads();
  // blocks per pair, exclusive prefix over pairs in (b, h) order
  int* s_base = s_n + pairs;
  {
    int running = 0;
    for (int p0 = 0; p0 < pairs; p0 += blockDim.x) {
      const int p = p0 + tid;
      const int nb = p < pairs ? (s_n[p] + v.BT - 1) / v.BT : 0;
      if (p < pairs && nb > v.mbh) {
        atomicExch(&s_fail, 1);
        report_error(v.hdr, DMS_DEVERR_HEAD_TABLE_FULL, layer, seq0 + p / v.Hkv, p % v.Hkv);
      }
      int incl = nb;
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane == 31) s_warp[warp] = incl;
      __syncthreads();
      if (warp == 0) {
        int t = lane < nwarps ? s_warp[lane] : 0;
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, t, o);
          if (lane >= o) t += y;
        }
        s_warp[lane] = t;  // inclusive warp totals
      }
      __syncthreads();
      const int before = (warp ? s_warp[warp - 1] : 0);
      if (p < pairs) s_base[p] = running + before + incl - nb;
      running += s_warp[nwarps - 1];
      __syncthreads();
    }
    if (tid == 0) s_base[pairs] = running;
  }
  __syncthreads();
  const int total = s_base[pairs];
  const int stack = v.hdr->block_stack_top;
  const int64_t avail = int64_t(stack) + (v.max_blocks - v.hdr->next_block);
  if (tid == 0 && total > avail) {
    s_fail = 1;
    report_error(v.hdr, DMS_DEVERR_BLOCKS_EXHAUSTED, layer, -1, -1);
  }
  __syncthreads();
  if (s_fail) return;
  const int next = v.hdr->next_block;
  // block tables: allocation index a -> free stack top first, then bump
  for (int p = warp; p < pairs; p += nwarps) {
    const int hd = v.head(layer, seq0 + p / v.Hkv, p % v.Hkv);
    const int nb = (s_n[p] + v.BT - 1) / v.BT;
    for (int k = lane; k < nb; k += 32) {
      const int a = s_base[p] + k;
      const int id = a < stack ? v.block_stack[stack - 1 - a] : next + (a - stack);
      v.bt[int64_t(hd) * v.mbh + k] = id;
    }
    if (lane == 0) {
      v.n_slots[hd] = s_n[p];
      v.n_retained[hd] = s_n[p];
      v.free_top[hd] = 0;
      if (nb > 0) {
        const int a = s_base[p] + nb - 1;
        v.last_block[hd] = a < stack ? v.block_stack[stack - 1 - a] : next + (a - stack);
      } else {
        v.last_block[hd] = -1;
      }
    }
  }
  if (v.kv_dtype == DMS_FP8_E4M3) {
    // the first prefill into a layer sets its scales (0 = not set yet); later
    // prefills of other sequences reuse them, saturating like decode tokens
    for (int i = tid; i < 2 * v.Hkv; i += blockDim.x) {
      const float a = __uint_as_float(v.amax[i]);
      const float s = a > 0.f ? __fdiv_rn(a, 448.0f) : 1.0f;
      const int which = i / v.Hkv, h = i % v.Hkv;
      float* dst = v.scales + (int64_t(layer) * v.Hkv + h) * 2 + which;
      if (*dst == 0.f) *dst = s;
    }
  }
  __syncthreads();
  if (tid == 0) {
    v.hdr->block_stack_top = stack > total ? stack - total : 0;
    v.hdr->next_block = next + (total > stack ? total - stack : 0);
    v.hdr->prefill_go = 1;
  }
}

// ---------------------------------------------------------------------------
// FP8 only: clear the transposed V tile of each head's last, partly filled
// block, so that token columns past n_slots decode to 0 (the attention kernel
// reads whole V tiles).  One CTA per (sequence, kv-head).
__global__ void __launch_bounds__(256) prefill_fp8_clear_tail_kernel(PoolView v, int layer, int seq0) {
  if (!v.hdr->prefill_go) return;
  const int b = blockIdx.x / v.Hkv, h = blockIdx.x % v.Hkv;
  const int hd = v.head(layer, seq0 + b, h);
  const int n = v.n_slots[hd];
  if (n % v.BT == 0) return;
  uint8_t* blk = v.blocks + int64_t(v.bt[int64_t(hd) * v.mbh + n / v.BT]) * v.block_bytes;
  uint4* tile = reinterpret_cast<uint4*>(blk + v.tile_bytes);
  for (int i = threadIdx.x; i < int(v.tile_bytes / 16); i += blockDim.x) tile[i] = make_uint4(0, 0, 0, 0);
}

// ---------------------------------------------------------------------------
// One CTA per (256-token chunk, kv-head, sequence).  STORE: 0 = copy
// (bf16 / fp32 store), 1 = FP8, 2 = 4-bit.
template <typename InT, int STORE>
__global__ void __launch_bounds__(256) prefill_scatter_kernel(PoolView v, int layer, int seq0, int P,
                                                              const InT* __restrict__ k,
                                                              const InT* __restrict__ vv,
                                                              const uint8_t* __restrict__ evict) {
  constexpr int kBatchItems = 4;          // 16-byte copies in flight per thread
  __shared__ int s_kept[kPrefillChunk];   // chunk-local token index of each kept rank
  __shared__ int s_wcnt[8];
  if (!v.hdr->prefill_go) return;
  const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = chunk * kPrefillChunk + threadIdx.x;
  const int64_t in_row_elems = v.D;
  const int hd = v.head(layer, seq0 + b, h);
  const uint8_t f = j < P ? evict[(int64_t(b) * P + j) * v.Hkv + h] : 0;
  const bool keep = keep_token(j, P, v.w, f);
  const unsigned m = __ballot_sync(0xffffffffu, keep);
  if (lane == 0) s_wcnt[warp] = __popc(m);
  __syncthreads();
  int before = 0, nkept = 0;
  for (int q = 0; q < 8; ++q) {
    before += q < warp ? s_wcnt[q] : 0;
    nkept += s_wcnt[q];
  }
  const int rank = before + __popc(m & ((1u << lane) - 1u));
  const int base = v.chunk_counts[(int64_t(b) * v.Hkv + h) * v.n_chunks_max + chunk];
  const int32_t* table = v.bt + int64_t(hd) * v.mbh;
  if (keep) {
    s_kept[rank] = threadIdx.x;
    if (j >= P - v.w) {
      const int slot = base + rank;
      const int64_t ri = int64_t(hd) * v.w + (j % v.w);
      v.ring[ri] = uint32_t(slot) | (uint32_t(f != 0) << 31);
      v.ring_row[ri] = table[slot / v.BT] * v.BT + slot % v.BT;
    }
  }
  __syncthreads();
  if constexpr (STORE == 2) {
    // 4-bit: one warp quantises one kept row (lane l: elements 4l .. 4l+3)
    for (int kk = warp; kk < nkept; kk += blockDim.x / 32) {
      const int jj = chunk * kPrefillChunk + s_kept[kk];
      const int slot = base + kk;
      const int blk = table[slot / v.BT];
      if (!DMS_CHECK(blk >= 0 && blk < v.max_blocks, v.hdr, 202, hd, slot)) continue;
      const InT* srck = k + ((int64_t(b) * P + jj) * v.Hkv + h) * in_row_elems;
      const InT* srcv = vv + ((int64_t(b) * P + jj) * v.Hkv + h) * in_row_elems;
      float k4[4], v4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        k4[e] = to_f32(srck[4 * lane + e]);
        v4[e] = to_f32(srcv[4 * lane + e]);
      }
      store_row_int4(v, blk * v.BT + slot % v.BT, k4, v4, lane);
    }
  } else if constexpr (STORE == 0) {
    // bitwise row copy in 16-byte chunks, swizzled by row; each thread loads
    // kBatchItems K and V chunks before storing any
    const int nch = int(v.row_bytes >> 4);
    const int total = nkept * nch;
    for (int i0 = 0; i0 < total; i0 += kBatchItems * blockDim.x) {
      uint4 xk[kBatchItems], xv[kBatchItems];
      uint8_t* dst[kBatchItems];
#pragma unroll
      for (int u = 0; u < kBatchItems; ++u) {
        const int i = i0 + u * blockDim.x + threadIdx.x;
        dst[u] = nullptr;
        if (i < total) {
          const int kk = i / nch, c = i % nch;
          const int jj = chunk * kPrefillChunk + s_kept[kk];
          const int slot = base + kk;
          const int row = slot % v.BT;
          if (DMS_CHECK(slot < v.mbh * v.BT && table[slot / v.BT] >= 0 &&
                            table[slot / v.BT] < v.max_blocks, v.hdr, 201, hd, slot)) {
            dst[u] = v.blocks + int64_t(table[slot / v.BT]) * v.block_bytes +
                     int64_t(row) * v.row_bytes + swz_chunk(c, row) * 16;
            const int64_t src_off = ((int64_t(b) * P + jj) * v.Hkv + h) * v.row_bytes + c * 16;
            xk[u] = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(k) + src_off));
            xv[u] = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(vv) + src_off));
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kBatchItems; ++u) {
        if (dst[u]) {
          *reinterpret_cast<uint4*>(dst[u]) = xk[u];
          *reinterpret_cast<uint4*>(dst[u] + v.tile_bytes) = xv[u];
        }
      }
    }
  } else {
    // FP8 (D = 128): each thread quantises 16 elements of one kept row
    const float sK = v.scales[(int64_t(layer) * v.Hkv + h) * 2 + 0];
    const float sV = v.scales[(int64_t(layer) * v.Hkv + h) * 2 + 1];
    for (int i = threadIdx.x; i < nkept * 8; i += blockDim.x) {
      const int kk = i >> 3, lc = i & 7;
      const int jj = chunk * kPrefillChunk + s_kept[kk];
      const int slot = base + kk;
      const int row = slot % v.BT;
      uint8_t* blk = v.blocks + int64_t(table[slot / v.BT]) * v.block_bytes;
      const InT* srck = k + ((int64_t(b) * P + jj) * v.Hkv + h) * in_row_elems;
      const InT* srcv = vv + ((int64_t(b) * P + jj) * v.Hkv + h) * in_row_elems;
      uint8_t codes[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int pos = lc * 16 + e;
        const int d = ((pos >> 2) & 7) * 16 + ((pos >> 1) & 1) * 8 + (pos >> 5) * 2 + (pos & 1);
        codes[e] = f32_to_e4m3(__fdiv_rn(to_f32(srck[d]), sK));
      }
      *reinterpret_cast<uint4*>(blk + row * 128 + ((lc ^ (row & 7)) << 4)) =
          *reinterpret_cast<const uint4*>(codes);
      // V: elements d = lc*16 .. lc*16+15 of this token, transposed tile
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int d = lc * 16 + e;
        blk[v.tile_bytes + fp8v_byte(row, d)] = f32_to_e4m3(__fdiv_rn(to_f32(srcv[d]), sV));
      }
    }
  }
}

}  // namespace dms

using namespace dms;

namespace dms {
// Count kept tokens per 256-token chunk, then plan (prefix counts, block
// tables, counters, FP8 scales); shared with the fused prefill attention.
dms_status prefill_plan_launch(dms_pool* pool, int layer, int seq0, int batch, int prompt_len,
                               const uint8_t* evict, cudaStream_t stream) {
  const PoolView& pv = pool->view;
  const int n_chunks = (prompt_len + kPrefillChunk - 1) / kPrefillChunk;
  prefill_count_kernel<<<dim3(n_chunks, batch), 256, 0, stream>>>(pv, prompt_len, evict);
  dms_status st = cuda_status(cudaGetLastError(), "prefill_count_kernel");
  if (st != DMS_OK) return st;
  const size_t plan_smem = sizeof(int) * (2 * size_t(batch) * pv.Hkv + 1);
  if (plan_smem > 48 * 1024) {
    set_last_error("batch * n_kv_heads too large for the prefill planner");
    return DMS_ERR_UNSUPPORTED;
  }
  prefill_plan_kernel<<<1, 1024, plan_smem, stream>>>(pv, layer, seq0, batch, prompt_len);
  return cuda_status(cudaGetLastError(), "prefill_plan_kernel");
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
  const int n_chunks = (prompt_len + kPrefillChunk - 1) / kPrefillChunk;
  const dim3 grid(n_chunks, batch);
  dms_status st;
  if (fp8) {
    st = cuda_status(cudaMemsetAsync(pv.amax, 0, sizeof(uint32_t) * 2 * pv.Hkv, stream), "amax clear");
    if (st != DMS_OK) return st;
    const size_t sm = sizeof(uint32_t) * 2 * pv.Hkv;
    if (in_dtype == DMS_BF16)
      prefill_amax_kernel<__nv_bfloat16><<<grid, 256, sm, stream>>>(
          pv, prompt_len, static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v));
    else
      prefill_amax_kernel<float><<<grid, 256, sm, stream>>>(
          pv, prompt_len, static_cast<const float*>(k), static_cast<const float*>(v));
    st = cuda_status(cudaGetLastError(), "prefill_amax_kernel");
    if (st != DMS_OK) return st;
  }
  st = prefill_plan_launch(pool, layer, seq0, batch, prompt_len, evict, stream);
  if (st != DMS_OK) return st;
  if (fp8 || int4) {   // the V tile of each head's partly filled last block
    prefill_fp8_clear_tail_kernel<<<batch * pv.Hkv, 256, 0, stream>>>(pv, layer, seq0);
    st = cuda_status(cudaGetLastError(), "prefill_fp8_clear_tail_kernel");
    if (st != DMS_OK) return st;
  }
  const dim3 sgrid(n_chunks, pv.Hkv, batch);
  if (in_dtype == DMS_BF16) {
    auto kk = static_cast<const __nv_bfloat16*>(k);
    auto vv = static_cast<const __nv_bfloat16*>(v);
    if (fp8)
      prefill_scatter_kernel<__nv_bfloat16, 1><<<sgrid, 256, 0, stream>>>(pv, layer, seq0, prompt_len, kk, vv, evict);
    else if (int4)
      prefill_scatter_kernel<__nv_bfloat16, 2><<<sgrid, 256, 0, stream>>>(pv, layer, seq0, prompt_len, kk, vv, evict);
    else
      prefill_scatter_kernel<__nv_bfloat16, 0><<<sgrid, 256, 0, stream>>>(pv, layer, seq0, prompt_len, kk, vv, evict);
  } else {
    auto kk = static_cast<const float*>(k);
    auto vv = static_cast<const float*>(v);
    if (fp8)
      prefill_scatter_kernel<float, 1><<<sgrid, 256, 0, stream>>>(pv, layer, seq0, prompt_len, kk, vv, evict);
    else if (int4)
      prefill_scatter_kernel<float, 2><<<sgrid, 256, 0, stream>>>(pv, layer, seq0, prompt_len, kk, vv, evict);
    else
      prefill_scatter_kernel<float, 0><<<sgrid, 256, 0, stream>>>(pv, layer, seq0, prompt_len, kk, vv, evict);
  }
  return cuda_status(cudaGetLastError(), "prefill_scatter_kernel");
}
