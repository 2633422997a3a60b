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
// One warp per head (append_head_warp in append_core.cuh): the per-head
// state it needs (counters, last block, the ring entry and the physical row
// of the token leaving the window) is read with independent loads, so the
// kernel waits on memory about once before its stores, and the rows are
// written by as many SMs as there are heads / 8.
// A new block comes from an atomic bump of the block counter: the logical
// state (slots, counts, rings, stored bytes) is a deterministic function of
// the inputs; which physical block a head gets during decode is not (prefill
// hands blocks out by a prefix sum and is deterministic).
#include "append_core.cuh"

namespace dms {

constexpr int kAppendHeadsPerCta = 8;            // one warp per head
constexpr int kAppendThreads = 32 * kAppendHeadsPerCta;

// One warp per (layer, sequence, kv-head) runs append_head_warp.
// seq_ids (nullable): pool sequence of batch row b, else b.  pos_arr
// (nullable): position of batch row b, else `pos` for every row.
// STORE: 0 = copy (bf16 / fp32 store), 1 = FP8, 2 = 4-bit
template <typename InT, int STORE>
__global__ void __launch_bounds__(kAppendThreads)
    append_evict_kernel(PoolView v, int l0, int nl, int batch, int64_t pos, const InT* k,
                        const InT* vv, const uint8_t* evict, const int32_t* seq_ids,
                        const int64_t* pos_arr, const StepSync sync) {
  // the new rows and the pool state may have been written by the kernel
  // before this one; once they are visible, let the next kernel (decode
  // attention) be scheduled
  pdl_wait_prerequisites();
  pdl_launch_dependents();
  if (sync.ready) {  // the step's inputs are copied in by another stream
    if (threadIdx.x == 0 && !wait_counter_geq(sync.ready, sync.ready_value, v.wait_ns))
      report_error(v.hdr, DMS_DEVERR_TIMEOUT, l0, -1, -1);
    __syncthreads();
  }
  const int H = nl * batch * v.Hkv;
  const int lane = threadIdx.x & 31;
  const int i = blockIdx.x * kAppendHeadsPerCta + (threadIdx.x >> 5);
  if (i >= H) return;
  const int h = i % v.Hkv, bi = (i / v.Hkv) % batch, l = l0 + i / (v.Hkv * batch);
  const int b = seq_ids ? seq_ids[bi] : bi;
  const int64_t tpos = pos_arr ? pos_arr[bi] : pos;
  if (b < 0 || b >= v.Bmax || tpos < 0 || tpos >= (int64_t(1) << 31)) {
    if (lane == 0) report_error(v.hdr, DMS_DEVERR_BAD_SEQUENCE, l, bi, h);
    return;
  }
  const uint32_t flag = lane == 0 ? uint32_t(evict[i] != 0) : 0u;  // [nl, batch, Hkv] flattened like i
  append_head_warp<InT, STORE>(v, l, b, h, v.head(l, b, h), int(tpos), k + int64_t(i) * v.D,
                               vv + int64_t(i) * v.D, flag, lane);
}

}  // namespace dms

using namespace dms;

// Checks shared by the entry points, then one launch over n_layers x batch
// heads.  seq_ids / pos_arr are device arrays or null.
static dms_status launch_append(dms_pool* pool, int layer0, int n_layers, int batch, int64_t pos,
                                const void* k, const void* v, dms_dtype in_dtype,
                                const uint8_t* evict, const int32_t* seq_ids,
                                const int64_t* pos_arr, cudaStream_t stream,
                                const StepSync& sync = StepSync{}) {
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
  const bool fp8 = pv.kv_dtype == DMS_FP8_E4M3, int4 = pv.kv_dtype == DMS_INT4;
  if (!(in_dtype == DMS_F32 || in_dtype == DMS_BF16) || (!fp8 && !int4 && int(in_dtype) != pv.kv_dtype)) {
    set_last_error("in_dtype %d does not match kv_dtype %d", int(in_dtype), pv.kv_dtype);
    return DMS_ERR_INVALID_ARG;
  }
  if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15) {
    set_last_error("k and v must be 16-byte aligned");
    return DMS_ERR_INVALID_ARG;
  }
  const int H = n_layers * batch * pv.Hkv;
  const dim3 grid((H + kAppendHeadsPerCta - 1) / kAppendHeadsPerCta);
  dms_status st = DMS_OK;
#define DMS_LAUNCH_APPEND(T, F)                                                                   \
  st = cuda_status(launch_pdl(append_evict_kernel<T, F>, grid, dim3(kAppendThreads), 0, stream,  \
                              pv, layer0, n_layers, batch, pos, static_cast<const T*>(k),         \
                              static_cast<const T*>(v), evict, seq_ids, pos_arr, sync),           \
                   "append_evict_kernel")
  const int mode = fp8 ? 1 : int4 ? 2 : 0;
  if (in_dtype == DMS_BF16) {
    if (mode == 1) DMS_LAUNCH_APPEND(__nv_bfloat16, 1);
    else if (mode == 2) DMS_LAUNCH_APPEND(__nv_bfloat16, 2);
    else DMS_LAUNCH_APPEND(__nv_bfloat16, 0);
  } else {
    if (mode == 1) DMS_LAUNCH_APPEND(float, 1);
    else if (mode == 2) DMS_LAUNCH_APPEND(float, 2);
    else DMS_LAUNCH_APPEND(float, 0);
  }
#undef DMS_LAUNCH_APPEND
  return st;
}

extern "C" dms_status dms_append_evict_layers(dms_pool* pool, int layer0, int n_layers, int batch,
                                              int64_t pos, const void* k, const void* v,
                                              dms_dtype in_dtype, const uint8_t* evict,
                                              cudaStream_t stream) {
  return launch_append(pool, layer0, n_layers, batch, pos, k, v, in_dtype, evict, nullptr, nullptr,
                       stream);
}

// The stepper's append launch: arguments as for dms_append_evict_layers,
// plus the step counters.
dms_status dms::append_layers_synced(dms_pool* pool, int layer0, int n_layers, int batch, int64_t pos,
                                     const void* k, const void* v, dms_dtype in_dtype,
                                     const uint8_t* evict, cudaStream_t stream, const StepSync& sync) {
  return launch_append(pool, layer0, n_layers, batch, pos, k, v, in_dtype, evict, nullptr, nullptr,
                       stream, sync);
}

extern "C" dms_status dms_append_evict_seqs(dms_pool* pool, int layer0, int n_layers, int n_seqs,
                                            const int32_t* seq_ids, const int64_t* pos,
                                            const void* k, const void* v, dms_dtype in_dtype,
                                            const uint8_t* evict, cudaStream_t stream) {
  if (!seq_ids || !pos || (reinterpret_cast<uintptr_t>(pos) & 7) ||
      (reinterpret_cast<uintptr_t>(seq_ids) & 3)) {
    set_last_error("seq_ids and pos must be non-null, 4- and 8-byte aligned device arrays");
    return DMS_ERR_INVALID_ARG;
  }
  return launch_append(pool, layer0, n_layers, n_seqs, 0, k, v, in_dtype, evict, seq_ids, pos,
                       stream);
}

extern "C" dms_status dms_append_evict(dms_pool* pool, int layer, int batch, int64_t pos,
                                       const void* k, const void* v, dms_dtype in_dtype,
                                       const uint8_t* evict, cudaStream_t stream) {
  return dms_append_evict_layers(pool, layer, 1, batch, pos, k, v, in_dtype, evict, stream);
}
