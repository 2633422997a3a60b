// dms_release_seqs: end sequences and give their memory back to the pool.
//
// FastDMS keeps per-layer, per-head variable token counts in a pool instead
// of fixed pages and reports real allocator memory ("FastDMS: vLLM BF16/FP8
// 보다 빠른 6.4x KV cache 압축" (molayo1419.me), table "What's the catch?",
// row "PagedAttention / KV memory pool", and the paragraph before the memory
// table).  When a sequence finishes, every block its heads hold goes back on
// the global free-block stack, whole, so the next prefill or decode step of
// any sequence can take it; the heads' counters return to the empty state.
#include "dms_internal.cuh"

namespace dms {

constexpr int kReleaseWarps = 8;  // heads per CTA, one warp each

// One warp per (layer, listed sequence, kv-head).
__global__ void __launch_bounds__(32 * kReleaseWarps)
    release_kernel(PoolView v, int n_seqs, const int32_t* seq_ids) {
  const int lane = threadIdx.x & 31;
  const int i = blockIdx.x * kReleaseWarps + (threadIdx.x >> 5);
  if (i >= v.L * n_seqs * v.Hkv) return;
  const int h = i % v.Hkv, si = (i / v.Hkv) % n_seqs, l = i / (v.Hkv * n_seqs);
  const int b = seq_ids[si];
  if (b < 0 || b >= v.Bmax) {
    if (lane == 0) report_error(v.hdr, DMS_DEVERR_BAD_SEQUENCE, l, si, h);
    return;
  }
  const int hd = v.head(l, b, h);
  const int nb = (v.n_slots[hd] + v.BT - 1) / v.BT;
  int base = 0;
  if (lane == 0 && nb > 0) base = atomicAdd(&v.hdr->block_stack_top, nb);
  base = __shfl_sync(0xffffffffu, base, 0);
  for (int k = lane; k < nb; k += 32) {
    if (DMS_CHECK(base + k < v.max_blocks, v.hdr, 401, hd, base + k))
      v.block_stack[base + k] = v.bt[int64_t(hd) * v.mbh + k];
  }
  if (lane == 0) {
    v.n_slots[hd] = 0;
    v.n_retained[hd] = 0;
    v.free_top[hd] = 0;
    v.last_block[hd] = -1;
  }
}

}  // namespace dms

using namespace dms;

extern "C" dms_status dms_release_seqs(dms_pool* pool, int n_seqs, const int32_t* seq_ids,
                                       cudaStream_t stream) {
  if (!pool || !seq_ids || (reinterpret_cast<uintptr_t>(seq_ids) & 3)) {
    set_last_error("null pool, or seq_ids not a 4-byte aligned device array");
    return DMS_ERR_INVALID_ARG;
  }
  const PoolView& v = pool->view;
  if (n_seqs < 1 || n_seqs > v.Bmax) {
    set_last_error("n_seqs %d outside 1..max_batch (%d)", n_seqs, v.Bmax);
    return DMS_ERR_INVALID_ARG;
  }
  const int heads = v.L * n_seqs * v.Hkv;
  release_kernel<<<(heads + kReleaseWarps - 1) / kReleaseWarps, 32 * kReleaseWarps, 0, stream>>>(
      v, n_seqs, seq_ids);
  return cuda_status(cudaGetLastError(), "release_kernel");
}
