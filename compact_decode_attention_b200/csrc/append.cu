// dms_append_evict: one decode step of the compact store.
//
// DMS delayed eviction: a token flagged for eviction stays visible for w
// steps and is then removed ("NVIDIA veröffentlicht Qwen3-8B-DMS-8x ..."
// (mindverse), section "Dynamic Memory Sparsification (DMS): Eine
// innovative Lösung"; "Nvidia DMS ..." (stiva.ai), section "Ключевое
// изобретение: delayed eviction").  At step t the token leaving the window
// is t - w, found at ring index t mod w; when it was flagged its slot is
// pushed on the head's free stack, and the new token takes the top of that
// stack -- FastDMS's compact store reclaiming physically evicted slots
// ("FastDMS: vLLM BF16/FP8보다 빠른 6.4x KV cache 압축" (molayo1419.me),
// opening paragraphs).  Otherwise the token takes slot n_slots, opening a
// new block when that slot starts one.
//
// One CTA does the bookkeeping of every head of the call so that new blocks
// are handed out by a prefix sum in (layer, sequence, head) order: the
// physical block ids are a deterministic function of the inputs.  The same
// CTA then writes the rows (16-byte chunks spread over all threads).
#include "dms_internal.cuh"

namespace dms {

template <typename T>
__device__ __forceinline__ float in_to_f32(T x);
template <>
__device__ __forceinline__ float in_to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float in_to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

constexpr int kAppendThreads = 512;
constexpr int kAppendRegChunks = 20;   // 16-byte input chunks a thread can hold

template <typename InT, bool FP8>
__global__ void __launch_bounds__(kAppendThreads)
    append_evict_kernel(PoolView v, int l0, int nl, int batch, int64_t pos, const InT* k,
                        const InT* vv, const uint8_t* evict) {
  extern __shared__ int s_dyn[];
  // Rows of the new tokens: chunk c of head hh is K chunk c (c < nch) or V
  // chunk c - nch.  When they fit in registers they are loaded first, so the
  // loads overlap the bookkeeping below instead of following it.
  const int nch = int(v.row_bytes >> 4);
  const int H_ = nl * batch * v.Hkv;
  const int total_chunks = H_ * 2 * nch;
  const bool preload = !FP8 && total_chunks <= int(blockDim.x) * kAppendRegChunks;
  uint4 reg[kAppendRegChunks];
  if (preload) {
#pragma unroll
    for (int r = 0; r < kAppendRegChunks; ++r) {
      const int c = threadIdx.x + r * blockDim.x;
      if (c < total_chunks) {
        const int hh = c / (2 * nch), cc = c % (2 * nch);
        const uint8_t* src = reinterpret_cast<const uint8_t*>(cc < nch ? k : vv) +
                             int64_t(hh) * v.row_bytes + (cc % nch) * 16;
        reg[r] = *reinterpret_cast<const uint4*>(src);
      }
    }
  }
  const int H = nl * batch * v.Hkv;
  int* s_slot = s_dyn;          // [H] slot of the new token (-1: failed)
  int* s_blk = s_dyn + H;       // [H] physical block of that slot
  int* s_need = s_dyn + 2 * H;  // [H] 1 when the slot opens a new block
  __shared__ int s_warp[32];
  __shared__ int s_total, s_fail_blocks;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  const int t = int(pos);
  const int ring_idx = t % v.w;

  // ---- 1. retire the token leaving the window, pick the slot -------------
  for (int i = tid; i < H; i += blockDim.x) {
    const int h = i % v.Hkv, b = (i / v.Hkv) % batch, l = l0 + i / (v.Hkv * batch);
    const int hd = v.head(l, b, h);
    int ns = v.n_slots[hd], nr = v.n_retained[hd], ft = v.free_top[hd];
    int* stack = v.free_stack + int64_t(hd) * v.free_cap;
    if (t >= v.w) {
      const uint32_t e = v.ring[int64_t(hd) * v.w + ring_idx];
      if (e >> 31) {
        if (ft < v.free_cap) {
          stack[ft++] = int(e & 0x7fffffffu);
          nr -= 1;
        } else {
          report_error(v.hdr, DMS_DEVERR_FREE_STACK_FULL, l, b, h);
        }
      }
    }
    int slot, need = 0;
    if (ft > 0) {
      slot = stack[--ft];
    } else {
      slot = ns;
      need = (slot % v.BT) == 0;
      if (slot / v.BT >= v.mbh) {
        report_error(v.hdr, DMS_DEVERR_HEAD_TABLE_FULL, l, b, h);
        slot = -1;
        need = 0;
      } else {
        ns += 1;
      }
    }
    s_slot[i] = slot;
    s_need[i] = need;
    // counters are committed in step 3 once the block (if any) is secured
    if (slot >= 0 && !DMS_CHECK(hd >= 0 && hd < v.n_heads && slot < v.mbh * v.BT, v.hdr, 101, hd, slot))
      slot = -1;
    s_blk[i] = slot < 0 ? -1 : (need ? -2 : v.bt[int64_t(hd) * v.mbh + slot / v.BT]);
    if (slot >= 0 && !need && !DMS_CHECK(s_blk[i] >= 0 && s_blk[i] < v.max_blocks, v.hdr, 102, hd, s_blk[i]))
      slot = -1, s_slot[i] = -1;
    if (slot >= 0) {
      v.free_top[hd] = ft;
      // n_slots / n_retained written below
      s_dyn[3 * H + i] = ns;
      s_dyn[4 * H + i] = nr + 1;
    }
  }
  __syncthreads();

  // ---- 2. exclusive prefix of new blocks in (layer, seq, head) order ------
  {
    int running = 0;
    for (int i0 = 0; i0 < H; i0 += blockDim.x) {
      const int i = i0 + tid;
      const int x = i < H ? s_need[i] : 0;
      int incl = x;
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane == 31) s_warp[warp] = incl;
      __syncthreads();
      if (warp == 0) {
        int tt = lane < nwarps ? s_warp[lane] : 0;
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, tt, o);
          if (lane >= o) tt += y;
        }
        s_warp[lane] = tt;
      }
      __syncthreads();
      if (i < H) s_need[i] = x ? running + (warp ? s_warp[warp - 1] : 0) + incl - x + 1 : 0;
      running += s_warp[nwarps - 1];
      __syncthreads();
    }
    if (tid == 0) {
      s_total = running;
      const int stack = v.hdr->block_stack_top;
      const int64_t avail = int64_t(stack) + (v.max_blocks - v.hdr->next_block);
      s_fail_blocks = running > avail;
      if (s_fail_blocks) report_error(v.hdr, DMS_DEVERR_BLOCKS_EXHAUSTED, l0, -1, -1);
    }
    __syncthreads();
  }

  // ---- 3. commit: new blocks, counters, ring -------------------------------
  const int stack_top = v.hdr->block_stack_top;
  const int next = v.hdr->next_block;
  for (int i = tid; i < H; i += blockDim.x) {
    const int h = i % v.Hkv, b = (i / v.Hkv) % batch, l = l0 + i / (v.Hkv * batch);
    const int hd = v.head(l, b, h);
    int slot = s_slot[i];
    if (slot < 0) continue;
    if (s_need[i]) {
      if (s_fail_blocks) {
        s_slot[i] = -1;
        continue;
      }
      const int a = s_need[i] - 1;
      const int id = a < stack_top ? v.block_stack[stack_top - 1 - a] : next + (a - stack_top);
      if (!DMS_CHECK(id >= 0 && id < v.max_blocks, v.hdr, 103, hd, id)) {
        s_slot[i] = -1;
        continue;
      }
      v.bt[int64_t(hd) * v.mbh + slot / v.BT] = id;
      s_blk[i] = id;
    }
    v.n_slots[hd] = s_dyn[3 * H + i];
    v.n_retained[hd] = s_dyn[4 * H + i];
    const uint8_t f = evict[i];  // [nl, batch, Hkv] flattened like i
    v.ring[int64_t(hd) * v.w + ring_idx] = uint32_t(slot) | (uint32_t(f != 0) << 31);
  }
  __syncthreads();
  if (tid == 0 && !s_fail_blocks) {
    const int total = s_total;
    v.hdr->block_stack_top = stack_top > total ? stack_top - total : 0;
    v.hdr->next_block = next + (total > stack_top ? total - stack_top : 0);
  }

  // ---- 4. write the rows ---------------------------------------------------
  if (preload) {
#pragma unroll
    for (int r = 0; r < kAppendRegChunks; ++r) {
      const int c = threadIdx.x + r * blockDim.x;
      if (c < total_chunks) {
        const int hh = c / (2 * nch), cc = c % (2 * nch);
        const int slot = s_slot[hh];
        if (slot < 0) continue;
        const int row = slot % v.BT;
        uint8_t* dst = v.blocks + int64_t(s_blk[hh]) * v.block_bytes + (cc < nch ? 0 : v.tile_bytes) +
                       int64_t(row) * v.row_bytes + swz_chunk(cc % nch, row) * 16;
        *reinterpret_cast<uint4*>(dst) = reg[r];
      }
    }
  } else if constexpr (!FP8) {
    for (int i = tid; i < H * nch; i += blockDim.x) {
      const int hh = i / nch, c = i % nch;
      const int slot = s_slot[hh];
      if (slot < 0) continue;
      const int row = slot % v.BT;
      uint8_t* blk = v.blocks + int64_t(s_blk[hh]) * v.block_bytes;
      const int64_t src = int64_t(hh) * v.row_bytes + c * 16;
      const int64_t dst = int64_t(row) * v.row_bytes + swz_chunk(c, row) * 16;
      *reinterpret_cast<uint4*>(blk + dst) =
          *reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(k) + src);
      *reinterpret_cast<uint4*>(blk + v.tile_bytes + dst) =
          *reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(vv) + src);
    }
  } else {
    // a new block's transposed V tile is cleared first so that token columns
    // not yet written decode to 0 (the attention kernel reads whole V tiles)
    for (int i = tid; i < H * 512; i += blockDim.x) {
      const int hh = i >> 9;
      if (s_slot[hh] < 0 || s_need[hh] == 0) continue;  // only blocks opened by this step
      uint8_t* blk = v.blocks + int64_t(s_blk[hh]) * v.block_bytes;
      reinterpret_cast<uint4*>(blk + v.tile_bytes)[i & 511] = make_uint4(0, 0, 0, 0);
    }
    __syncthreads();
    for (int i = tid; i < H * 8; i += blockDim.x) {
      const int hh = i >> 3, lc = i & 7;
      const int slot = s_slot[hh];
      if (slot < 0) continue;
      const int h = hh % v.Hkv, l = l0 + hh / (v.Hkv * batch);
      const float sK = v.scales[(int64_t(l) * v.Hkv + h) * 2 + 0];
      const float sV = v.scales[(int64_t(l) * v.Hkv + h) * 2 + 1];
      const int row = slot % v.BT;
      uint8_t* blk = v.blocks + int64_t(s_blk[hh]) * v.block_bytes;
      const InT* srck = k + int64_t(hh) * v.D;
      const InT* srcv = vv + int64_t(hh) * v.D;
      uint8_t codes[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int p = lc * 16 + e;
        const int d = ((p >> 2) & 7) * 16 + ((p >> 1) & 1) * 8 + (p >> 5) * 2 + (p & 1);
        codes[e] = f32_to_e4m3(__fdiv_rn(in_to_f32(srck[d]), sK));
      }
      *reinterpret_cast<uint4*>(blk + row * 128 + ((lc ^ (row & 7)) << 4)) =
          *reinterpret_cast<const uint4*>(codes);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int d = lc * 16 + e;
        blk[v.tile_bytes + fp8v_byte(row, d)] = f32_to_e4m3(__fdiv_rn(in_to_f32(srcv[d]), sV));
      }
    }
  }
}

}  // namespace dms

using namespace dms;

extern "C" dms_status dms_append_evict_layers(dms_pool* pool, int layer0, int n_layers, int batch,
                                              int64_t pos, const void* k, const void* v,
                                              dms_dtype in_dtype, const uint8_t* evict,
                                              cudaStream_t stream) {
  if (!pool) {
    set_last_error("null pool");
    return DMS_ERR_INVALID_ARG;
  }
  const PoolView& pv = pool->view;
  if (layer0 < 0 || n_layers < 1 || layer0 + n_layers > pv.L || batch < 1 || batch > pv.Bmax ||
      pos < 0 || pos >= pool->cfg.max_context || pos >= (int64_t(1) << 31)) {
    set_last_error("bad layer range / batch / position (%d+%d, %d, %lld)", layer0, n_layers, batch,
                   (long long)pos);
    return DMS_ERR_INVALID_ARG;
  }
  if (!k || !v || !evict) {
    set_last_error("null input pointer");
    return DMS_ERR_INVALID_ARG;
  }
  const bool fp8 = pv.kv_dtype == DMS_FP8_E4M3;
  if (!(in_dtype == DMS_F32 || in_dtype == DMS_BF16) || (!fp8 && int(in_dtype) != pv.kv_dtype)) {
    set_last_error("in_dtype %d does not match kv_dtype %d", int(in_dtype), pv.kv_dtype);
    return DMS_ERR_INVALID_ARG;
  }
  if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15) {
    set_last_error("k and v must be 16-byte aligned");
    return DMS_ERR_INVALID_ARG;
  }
  const int H = n_layers * batch * pv.Hkv;
  const size_t smem = sizeof(int) * 5 * size_t(H);
  if (smem > 200 * 1024) {
    set_last_error("too many heads (%d) for one append call; split the layer range", H);
    return DMS_ERR_UNSUPPORTED;
  }
  const int threads = kAppendThreads;
  dms_status st = DMS_OK;
#define DMS_LAUNCH_APPEND(T, F)                                                                    \
  do {                                                                                             \
    auto fn = append_evict_kernel<T, F>;                                                           \
    if (smem > 48 * 1024) {                                                                        \
      st = cuda_status(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,       \
                                            int(smem)), "append smem attribute");                  \
      if (st != DMS_OK) return st;                                                                 \
    }                                                                                              \
    fn<<<1, threads, smem, stream>>>(pv, layer0, n_layers, batch, pos, static_cast<const T*>(k),   \
                                     static_cast<const T*>(v), evict);                            \
  } while (0)
  if (in_dtype == DMS_BF16) {
    if (fp8) DMS_LAUNCH_APPEND(__nv_bfloat16, true);
    else DMS_LAUNCH_APPEND(__nv_bfloat16, false);
  } else {
    if (fp8) DMS_LAUNCH_APPEND(float, true);
    else DMS_LAUNCH_APPEND(float, false);
  }
#undef DMS_LAUNCH_APPEND
  return cuda_status(cudaGetLastError(), "append_evict_kernel");
}

extern "C" dms_status dms_append_evict(dms_pool* pool, int layer, int batch, int64_t pos,
                                       const void* k, const void* v, dms_dtype in_dtype,
                                       const uint8_t* evict, cudaStream_t stream) {
  return dms_append_evict_layers(pool, layer, 1, batch, pos, k, v, in_dtype, evict, stream);
}
