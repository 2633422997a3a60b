// Prefill compaction of a copy store (bf16 or fp32 rows) in one launch: one
// thread-block cluster per (sequence, kv-head).
//
// DMS delayed eviction at the end of the prompt (t = P - 1): a head keeps
// every token younger than the window and every older token without an
// evict flag ("NVIDIA veröffentlicht Qwen3-8B-DMS-8x ..." (mindverse),
// section "Dynamic Memory Sparsification (DMS): Eine innovative Lösung"),
// stored compactly in position order (FastDMS page, opening paragraphs).
// The two-launch path (csrc/prefill.cu) plans a whole layer in one CTA and
// then scatters; at a few heads per layer that is a chain of about six
// dependent memory round trips over two launches.  Here the C CTAs of a
// head's cluster each take a span of the prompt:
//   1. count the span's kept tokens (warp ballot + popcount) and list their
//      positions by rank;
//   2. push the count into every CTA's shared memory; after a cluster
//      barrier each CTA has every count and the head's total, takes an even
//      share of the head's kept rows (a span inside the window keeps every
//      token, others few), reads their positions from the owning CTAs'
//      lists and loads its first source chunks into registers;
//   3. CTA 0 checks that the head is empty, takes the head's blocks (the
//      global free-block stack first, then the bump pointer), writes the
//      block table and the counters, and pushes the allocation to every CTA;
//   4. after a second cluster barrier (no CTA reads another's list after
//      it) each CTA copies its rows into their slots (16-byte chunks,
//      swizzled by row) and fills the window ring for its rows inside the
//      window.
// Blocks are taken per head, so which physical blocks a head gets depends on
// the order heads reach step 3 (the logical state does not).  A head that
// is not empty is left as it is (DMS_DEVERR_LAYER_NOT_EMPTY), as is a head
// whose blocks do not fit (DMS_DEVERR_HEAD_TABLE_FULL, _BLOCKS_EXHAUSTED).
//
// Cluster barriers: every thread arrives with the same instruction at the
// same point and waits once per phase; the first phase is arrived at on
// entry and waited on before the first write into another CTA's shared
// memory (every CTA of the cluster is then running).
#include "append_core.cuh"

namespace dms {

constexpr int kPcThreads = 256;
constexpr int kPcMaxC = 16;
constexpr int kPcMaxIters = 64;   // spans of up to 63 x 256 tokens per CTA (the last row of s_wc is scratch)

__device__ __forceinline__ void pc_arrive() {
  asm volatile("barrier.cluster.arrive.release;" ::: "memory");
}
__device__ __forceinline__ void pc_wait() {
  asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ uint32_t pc_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t pc_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void pc_st_remote(const void* local, uint32_t rank, int x) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(local)), "r"(rank));
  asm volatile("st.shared::cluster.s32 [%0], %1;" ::"r"(a), "r"(x) : "memory");
}

__device__ __forceinline__ int pc_ld_remote(const void* local, uint32_t rank) {
  uint32_t a;
  int x;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(local)), "r"(rank));
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(x) : "r"(a) : "memory");
  return x;
}

__device__ __forceinline__ bool pc_keep(int j, int P, int w, uint8_t flag) {
  return j < P && (flag == 0 || (P - 1 - j) < w);
}

// span = tokens per CTA (a multiple of 256); gridDim.x = batch * Hkv * C
template <typename InT>
__global__ void __launch_bounds__(kPcThreads) prefill_cluster_kernel(PoolView v, int layer, int seq0, int P,
                                                                    int span, const InT* __restrict__ k,
                                                                    const InT* __restrict__ vv,
                                                                    const uint8_t* __restrict__ evict) {
  __shared__ int s_wc[kPcMaxIters][8];   // kept tokens per (256-token iteration, warp)
  __shared__ int s_cnt[kPcMaxC];         // kept tokens of each CTA of the cluster (pushed)
  __shared__ int s_alloc[4];             // (blocks from the free stack, stack top before, bump base, failed)
  extern __shared__ int s_kept[];        // positions of the span's kept tokens, by rank (span ints)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int C = int(pc_size()), j = int(pc_rank());
  const int pair = blockIdx.x / C, b = pair / v.Hkv, h = pair % v.Hkv;
  const int hd = v.head(layer, seq0 + b, h);
  const int p0 = j * span, p1 = min(P, p0 + span);
  const int iters = p1 > p0 ? (p1 - p0 + kPcThreads - 1) / kPcThreads : 0;
  const int64_t row_elems = v.D;
  const uint32_t row_bytes = uint32_t(v.row_bytes);
  auto src_row = [&](const InT* x, int pos) { return x + ((int64_t(b) * P + pos) * v.Hkv + h) * row_elems; };

  if (C > 1) pc_arrive();   // phase 1: this CTA runs
  pdl_launch_dependents();
  pdl_wait_prerequisites();

  // CTA 0: the state its allocation reads, loaded now (warp 1, off the
  // flags' path); the free-stack top is a first guess for the
  // compare-and-swap below
  int pre_ns = 0, pre_nr = 0, pre_top = 0;
  if (j == 0 && warp == 1 && lane == 0) {
    pre_ns = v.n_slots[hd];
    pre_nr = v.n_retained[hd];
    pre_top = *reinterpret_cast<volatile int*>(&v.hdr->block_stack_top);
    s_alloc[0] = pre_ns;
    s_alloc[1] = pre_nr;
    s_alloc[2] = pre_top;
  }
  // ---- 1. kept tokens of the span, per 256-token iteration and warp ----
  int mine = 0;
  for (int it = 0; it < iters; ++it) {
    const int pos = p0 + it * kPcThreads + tid;
    const uint8_t f = pos < p1 ? __ldg(evict + (int64_t(b) * P + pos) * v.Hkv + h) : 0;
    const bool keep = pos < p1 && pc_keep(pos, P, v.w, f);
    const unsigned m = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) s_wc[it][warp] = __popc(m);
  }
  __syncthreads();
  if (tid < 32) {   // this CTA's count, and the exclusive prefix of every (iteration, warp)
    int run = 0;
    for (int it = 0; it < iters; ++it) {
      const int c = lane < 8 ? s_wc[it][lane] : 0;
      int incl = c;
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane < 8) s_wc[it][lane] = run + incl - c;
      run += __shfl_sync(0xffffffffu, incl, 7);
    }
    mine = run;
    if (lane == 0) s_wc[kPcMaxIters - 1][0] = run;   // (read back below, by every thread)
  }
  __syncthreads();
  const int nkept = s_wc[kPcMaxIters - 1][0];
  // the span's kept positions by rank (flags again, from L2)
  for (int it = 0; it < iters; ++it) {
    const int pos = p0 + it * kPcThreads + tid;
    const uint8_t f = pos < p1 ? __ldg(evict + (int64_t(b) * P + pos) * v.Hkv + h) : 0;
    const bool keep = pos < p1 && pc_keep(pos, P, v.w, f);
    const unsigned m = __ballot_sync(0xffffffffu, keep);
    if (keep) s_kept[s_wc[it][warp] + __popc(m & ((1u << lane) - 1u))] = pos;
  }
  __syncthreads();
  (void)nkept;
  // ---- 2. counts to every CTA; prefix and total ----
  if (C > 1) {
    pc_wait();   // phase 1: every CTA of the cluster runs
    if (tid < C) pc_st_remote(&s_cnt[j], tid, mine);   // lanes of warp 0 (C <= 16) all hold the count
    pc_arrive();   // phase 2: this CTA's count is pushed
    pc_wait();
  } else if (tid == 0) {
    s_cnt[0] = mine;
  }
  __syncthreads();
  int total = 0, before = 0;
  for (int r = 0; r < C; ++r) {
    before += r < j ? s_cnt[r] : 0;
    total += s_cnt[r];
  }
  // kept tokens before each 256-token chunk of the span (the prefill
  // scratch the two-launch planner fills too; prompt attention reads it)
  if (tid < iters)
    v.chunk_counts[(int64_t(b) * v.Hkv + h) * v.n_chunks_max + p0 / kPcThreads + tid] = before + s_wc[tid][0];
  // The head's kept rows are spread evenly over the cluster's CTAs (a span
  // inside the window keeps every token, the others few): CTA j copies rows
  // [r0, r1).  Their positions are read from the owning CTAs' lists (valid
  // until the barrier after the allocation), and the first source chunks
  // are loaded while CTA 0 allocates: item i = 16-byte chunk i % nch of row
  // r0 + i / nch.
  const int r0 = int(int64_t(total) * j / C), r1 = int(int64_t(total) * (j + 1) / C);
  int* s_rows = s_kept + span;   // positions of rows r0 .. r1-1
  for (int r = r0 + tid; r < r1; r += kPcThreads) {
    int q = 0, qb = 0;
    while (r >= qb + s_cnt[q]) qb += s_cnt[q++];   // the CTA whose list holds row r
    s_rows[r - r0] = C > 1 ? pc_ld_remote(&s_kept[r - qb], q) : s_kept[r - qb];
  }
  __syncthreads();
  const int nch = int(row_bytes >> 4);
  const int items = (r1 - r0) * nch;
  constexpr int kU = 8;
  uint4 xk[kU], xv[kU];
  const auto load_items = [&](int i0) {
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u * kPcThreads + tid;
      if (i < items) {
        const int rpos = s_rows[i / nch], c = i % nch;
        xk[u] = __ldg(reinterpret_cast<const uint4*>(src_row(k, rpos)) + c);
        xv[u] = __ldg(reinterpret_cast<const uint4*>(src_row(vv, rpos)) + c);
      }
    }
  };
  load_items(0);
  // ---- 3. CTA 0: the head must be empty; its blocks; table and counters ----
  if (j == 0 && warp == 0) {
    const int nb = (total + v.BT - 1) / v.BT;
    int take = 0, top0 = 0, bump = 0, fail = 0;
    if (lane == 0) {
      if (s_alloc[0] != 0 || s_alloc[1] != 0) {   // preloaded by warp 1 (before the barriers)
        report_error(v.hdr, DMS_DEVERR_LAYER_NOT_EMPTY, layer, seq0 + b, h);
        fail = 1;
      } else if (nb > v.mbh) {
        report_error(v.hdr, DMS_DEVERR_HEAD_TABLE_FULL, layer, seq0 + b, h);
        fail = 1;
      } else {
        // blocks released by finished sequences first (only pops run here:
        // a successful compare-and-swap owns the entries below the old top)
        int top = s_alloc[2];
        while (top > 0) {
          const int t = min(nb, top);
          const int prev = atomicCAS(&v.hdr->block_stack_top, top, top - t);
          if (prev == top) {
            take = t;
            top0 = top;
            break;
          }
          top = prev;
        }
        if (nb > take) {
          bump = atomicAdd(&v.hdr->next_block, nb - take);
          if (int64_t(bump) + (nb - take) > v.max_blocks) {
            report_error(v.hdr, DMS_DEVERR_BLOCKS_EXHAUSTED, layer, seq0 + b, h);
            fail = 1;
          }
        }
      }
    }
    take = __shfl_sync(0xffffffffu, take, 0);
    top0 = __shfl_sync(0xffffffffu, top0, 0);
    bump = __shfl_sync(0xffffffffu, bump, 0);
    fail = __shfl_sync(0xffffffffu, fail, 0);
    if (!fail) {
      for (int kb = lane; kb < nb; kb += 32)
        v.bt[int64_t(hd) * v.mbh + kb] = kb < take ? v.block_stack[top0 - 1 - kb] : bump + (kb - take);
      if (lane == 0) {
        const int kl = nb - 1;
        v.last_block[hd] = kl < take ? v.block_stack[top0 - 1 - kl] : bump + (kl - take);
        v.n_slots[hd] = total;
        v.n_retained[hd] = total;
        v.free_top[hd] = 0;
      }
    }
    if (C > 1) {
      if (lane < C) {
        pc_st_remote(&s_alloc[0], lane, take);
        pc_st_remote(&s_alloc[1], lane, top0);
        pc_st_remote(&s_alloc[2], lane, bump);
        pc_st_remote(&s_alloc[3], lane, fail);
      }
    } else if (lane == 0) {
      s_alloc[0] = take;
      s_alloc[1] = top0;
      s_alloc[2] = bump;
      s_alloc[3] = fail;
    }
  }
  if (C > 1) {
    pc_arrive();   // phase 3: the allocation is pushed (and its table written)
    pc_wait();
  }
  __syncthreads();
  if (s_alloc[3]) return;
  const int take = s_alloc[0], top0 = s_alloc[1], bump = s_alloc[2];
  auto block_of = [&](int kb) { return kb < take ? v.block_stack[top0 - 1 - kb] : bump + (kb - take); };

  // ---- 4. rows r0 .. r1-1 into their slots (row r is slot r), window ring ----
  for (int r = r0 + tid; r < r1; r += kPcThreads) {
    const int pos = s_rows[r - r0];
    if (pos >= P - v.w) {   // every token of the window is kept
      const int slot = r;
      const uint8_t f = __ldg(evict + (int64_t(b) * P + pos) * v.Hkv + h);
      const int64_t ri = int64_t(hd) * v.w + (pos % v.w);
      v.ring[ri] = uint32_t(slot) | (uint32_t(f != 0) << 31);
      v.ring_row[ri] = block_of(slot / v.BT) * v.BT + slot % v.BT;
    }
  }
  for (int i0 = 0; i0 < items; i0 += kU * kPcThreads) {
    if (i0) load_items(i0);
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u * kPcThreads + tid;
      if (i < items) {
        const int slot = r0 + i / nch, c = i % nch;
        const int row = slot % v.BT;
        const int blk = block_of(slot / v.BT);
        if (!DMS_CHECK(blk >= 0 && blk < v.max_blocks, v.hdr, 501, hd, slot)) continue;
        uint8_t* dst = v.blocks + int64_t(blk) * v.block_bytes + int64_t(row) * v.row_bytes + swz_chunk(c, row) * 16;
        *reinterpret_cast<uint4*>(dst) = xk[u];
        *reinterpret_cast<uint4*>(dst + v.tile_bytes) = xv[u];
      }
    }
  }
}

// Longest prompt the one-launch compaction takes.  The kernel could take 16
// CTAs x 63 x 256 tokens, but one cluster per head is a latency design: a
// long prompt's head (131072 tokens, possibly all kept) over 16 CTAs took
// 1.27 ms a layer on the Qwen3-8B batch-16 workload against 0.6 ms in the
// two launches, whose scatter spreads every head over many CTAs.
int prefill_cluster_max_prompt() { return 16384; }
static_assert(16384 <= kPcMaxC * (kPcMaxIters - 1) * kPcThreads, "spans of at most 63 iterations");

// One launch for a copy store: clusters of C CTAs per (sequence, kv-head).
dms_status prefill_cluster_launch(dms_pool* pool, int layer, int seq0, int batch, int prompt_len,
                                  const void* k, const void* v, dms_dtype in_dtype, const uint8_t* evict,
                                  cudaStream_t stream) {
  const PoolView& pv = pool->view;
  // CTAs per head: up to 16, each with at least 256 tokens, at most 64 x 256
  int C = 1;
  while (C < kPcMaxC && int64_t(prompt_len) > int64_t(C) * 2 * kPcThreads) C *= 2;
  int span = (prompt_len + C - 1) / C;
  span = (span + kPcThreads - 1) / kPcThreads * kPcThreads;
  if (span > (kPcMaxIters - 1) * kPcThreads) {
    set_last_error("prompt of %d tokens exceeds the one-launch compaction (%d)", prompt_len,
                   kPcMaxC * kPcMaxIters * kPcThreads);
    return DMS_ERR_UNSUPPORTED;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(batch * pv.Hkv * C));
  cfg.blockDim = dim3(kPcThreads);
  cfg.dynamicSmemBytes = 2 * size_t(span) * sizeof(int);   // the span's kept positions, this CTA's rows
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = C;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  // clusters of 16 CTAs are past the portable size of 8; long spans list
  // more kept positions than the default 48 KB of shared memory hold
  static FuncAttrCache size_attr[2], smem_attr[2];
  const void* kernel = in_dtype == DMS_BF16 ? reinterpret_cast<const void*>(prefill_cluster_kernel<__nv_bfloat16>)
                                            : reinterpret_cast<const void*>(prefill_cluster_kernel<float>);
  const int ki = in_dtype == DMS_BF16 ? 0 : 1;
  dms_status st = ensure_func_attr(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1, size_attr[ki],
                                   "prefill cluster size");
  if (st == DMS_OK)
    st = ensure_func_attr(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                          2 * (kPcMaxIters - 1) * kPcThreads * int(sizeof(int)), smem_attr[ki], "prefill cluster smem");
  if (st != DMS_OK) return st;
  cudaError_t e;
  if (in_dtype == DMS_BF16)
    e = cudaLaunchKernelEx(&cfg, prefill_cluster_kernel<__nv_bfloat16>, pv, layer, seq0, prompt_len, span,
                           static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), evict);
  else
    e = cudaLaunchKernelEx(&cfg, prefill_cluster_kernel<float>, pv, layer, seq0, prompt_len, span,
                           static_cast<const float*>(k), static_cast<const float*>(v), evict);
  return cuda_status(e, "prefill_cluster_kernel");
}

}  // namespace dms
