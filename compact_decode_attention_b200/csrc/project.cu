// dms_project_append: the model's K/V projection of a decode token with
// the DMS eviction decision and the append into the compact store fused
// into its epilogue.
//
// Per kv-head h and sequence s: k = x_s W_kv[:, h-th D columns],
// v = x_s W_kv[:, (Hkv + h)-th D columns], logit = x_s w_evict[:, h] +
// b_evict[h]; the token is flagged for (delayed) eviction when the logit
// exceeds the threshold ("NVIDIA veröffentlicht Qwen3-8B-DMS-8x ..."
// (mindverse), section "Dynamic Memory Sparsification (DMS): Eine innovative
// Lösung": a learned predictor decides per head which tokens to evict; its
// weights are an input here).  k and v are rounded to bf16 and appended as
// dms_append_evict_seqs would append them.
//
// Decode is a matrix-vector product per sequence, bound by reading the
// weights: a grid of (d_model chunk of 128 rows, kv-head) CTAs reads each
// weight once, coalesced (a warp reads 512 bytes of one row: the head's K and
// V columns), and writes fp32 partial sums; the last CTA of a head (atomic
// ticket) adds the partials in chunk order (deterministic), rounds, decides
// the flag and runs the append of every sequence of the launch.
#include "append_core.cuh"

namespace dms {

constexpr int kProjRows = 128;     // weight rows per CTA
constexpr int kProjMaxSeqs = 8;    // sequences per launch (the host loops)
constexpr int kProjThreads = 256;  // 8 warps

// dynamic shared memory: x chunk [S][128] f32, cross-warp partials [8][S][256] f32,
// logit partials [8][S] f32, finished rows [S][2][D] f32
__host__ __device__ constexpr size_t proj_smem(int D) {
  return size_t(kProjMaxSeqs) * kProjRows * 4 + size_t(8) * kProjMaxSeqs * 256 * 4 +
         size_t(8) * kProjMaxSeqs * 4 + size_t(kProjMaxSeqs) * 2 * D * 4 + 64;
}

// Partial of CTA (chunk kc, head h): part[((h * KC + kc) * S + s) * (2D + 1) + c]
template <int D>
__global__ void __launch_bounds__(kProjThreads)
    project_append_kernel(PoolView v, int layer, int S, const int32_t* seq_ids, const int64_t* pos,
                          const __nv_bfloat16* x, int dm, const __nv_bfloat16* w_kv,
                          const __nv_bfloat16* w_ev, const float* b_ev, float thr, float* part,
                          int KC) {
  static_assert(2 * D == 256, "one warp covers the head's K and V columns with 16-byte loads");
  extern __shared__ float psm[];
  float* xs = psm;                                        // [S][128]
  float* red = xs + kProjMaxSeqs * kProjRows;             // [8][S][256]
  float* lred = red + 8 * kProjMaxSeqs * 256;             // [8][S]
  float* rows = lred + 8 * kProjMaxSeqs;                  // [S][2][D]
  int* s_last = reinterpret_cast<int*>(rows + kProjMaxSeqs * 2 * D);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kc = blockIdx.x, h = blockIdx.y;
  const int Hkv = v.Hkv, NC = 2 * D + 1;
  const int d0 = kc * kProjRows, nd = min(kProjRows, dm - d0);
  const int64_t ldw = int64_t(2) * Hkv * D;

  for (int i = tid; i < S * kProjRows; i += kProjThreads) {
    const int s = i / kProjRows, d = i % kProjRows;
    xs[i] = d < nd ? __bfloat162float(x[int64_t(s) * dm + d0 + d]) : 0.f;
  }
  __syncthreads();

  // ---- K and V columns: lane covers 8 columns (lanes 0-15 K, 16-31 V) ----
  float acc[kProjMaxSeqs][8];
#pragma unroll
  for (int s = 0; s < kProjMaxSeqs; ++s)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[s][e] = 0.f;
  const int col = lane < 16 ? h * D + 8 * lane : (Hkv + h) * D + 8 * (lane - 16);
  for (int d = warp; d < nd; d += 8) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(w_kv + (int64_t(d0 + d)) * ldw + col));
    const __nv_bfloat16* wv = reinterpret_cast<const __nv_bfloat16*>(&raw);
    float wf[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) wf[e] = __bfloat162float(wv[e]);
#pragma unroll
    for (int s = 0; s < kProjMaxSeqs; ++s) {
      if (s < S) {
        const float xv = xs[s * kProjRows + d];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[s][e] = fmaf(xv, wf[e], acc[s][e]);
      }
    }
  }
  // ---- eviction logit: thread t covers rows t, t + 256, ... of the chunk ----
  float lacc[kProjMaxSeqs];
#pragma unroll
  for (int s = 0; s < kProjMaxSeqs; ++s) lacc[s] = 0.f;
  for (int d = tid; d < nd; d += kProjThreads) {
    const float we = __bfloat162float(w_ev[int64_t(d0 + d) * Hkv + h]);
#pragma unroll
    for (int s = 0; s < kProjMaxSeqs; ++s)
      if (s < S) lacc[s] = fmaf(xs[s * kProjRows + d], we, lacc[s]);
  }
#pragma unroll
  for (int s = 0; s < kProjMaxSeqs; ++s) {
    float t = lacc[s];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (lane == 0 && s < S) lred[warp * kProjMaxSeqs + s] = t;
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (s < S) red[(warp * kProjMaxSeqs + s) * 256 + 8 * lane + e] = acc[s][e];
  }
  __syncthreads();
  // ---- this CTA's partial (warps added in order) ----
  for (int i = tid; i < S * 256; i += kProjThreads) {
    const int s = i / 256, c = i % 256;
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += red[(w * kProjMaxSeqs + s) * 256 + c];
    part[((int64_t(h) * KC + kc) * S + s) * NC + c] = t;
  }
  if (tid < S) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += lred[w * kProjMaxSeqs + tid];
    part[((int64_t(h) * KC + kc) * S + tid) * NC + 2 * D] = t;
  }
  __threadfence();
  __syncthreads();
  int* ticket = v.tickets + v.head(layer, 0, h);
  if (tid == 0) *s_last = atomicAdd(ticket, 1) == KC - 1;
  __syncthreads();
  if (!*s_last) return;
  __threadfence();

  // ---- last CTA of head h: sum the partials, round, decide, append ----
  for (int i = tid; i < S * 2 * D; i += kProjThreads) {
    const int s = i / (2 * D), c = i % (2 * D);
    float t = 0.f;
    for (int k = 0; k < KC; ++k) t += __ldcg(&part[((int64_t(h) * KC + k) * S + s) * NC + c]);
    rows[i] = __bfloat162float(__float2bfloat16_rn(t));   // the store's input precision
  }
  __syncthreads();
  if (tid == 0) *ticket = 0;
  for (int s = warp; s < S; s += 8) {
    float lg = 0.f;
    if (lane == 0)
      for (int k = 0; k < KC; ++k) lg += __ldcg(&part[((int64_t(h) * KC + k) * S + s) * NC + 2 * D]);
    lg = __shfl_sync(0xffffffffu, lg, 0) + (b_ev ? b_ev[h] : 0.f);
    const int b = seq_ids ? seq_ids[s] : s;
    const int64_t tpos = pos[s];
    if (b < 0 || b >= v.Bmax || tpos < 0 || tpos >= (int64_t(1) << 31)) {
      if (lane == 0) report_error(v.hdr, DMS_DEVERR_BAD_SEQUENCE, layer, s, h);
      continue;
    }
    const int hd = v.head(layer, b, h);
    int slot = -1, prow = -1, opened = 0;
    if (lane == 0) {
      const AppendSlot r = append_bookkeeping(v, layer, b, h, hd, int(tpos), lg > thr ? 1u : 0u);
      slot = r.slot;
      prow = r.prow;
      opened = r.opened;
    }
    slot = __shfl_sync(0xffffffffu, slot, 0);
    prow = __shfl_sync(0xffffffffu, prow, 0);
    opened = __shfl_sync(0xffffffffu, opened, 0);
    if (slot < 0) continue;
    store_row_from_float(v, layer, h, prow, opened, rows + s * 2 * D, rows + s * 2 * D + D, lane);
  }
}

}  // namespace dms

using namespace dms;

extern "C" dms_status dms_project_workspace_bytes(const dms_pool* pool, int n_seqs, int d_model,
                                                  size_t* bytes) {
  if (!pool || !bytes || n_seqs < 1 || d_model < 1) {
    set_last_error("bad arguments");
    return DMS_ERR_INVALID_ARG;
  }
  const PoolView& v = pool->view;
  const int KC = (d_model + kProjRows - 1) / kProjRows;
  const int S = n_seqs < kProjMaxSeqs ? n_seqs : kProjMaxSeqs;
  *bytes = size_t(v.Hkv) * KC * S * (2 * v.D + 1) * 4;
  return DMS_OK;
}

extern "C" dms_status dms_project_append(dms_pool* pool, int layer, int n_seqs, const int32_t* seq_ids,
                                         const int64_t* pos, const void* x, int d_model,
                                         const void* w_kv, const void* w_evict, const float* b_evict,
                                         float threshold, void* workspace, size_t workspace_bytes,
                                         cudaStream_t stream) {
  if (!pool) {
    set_last_error("null pool");
    return DMS_ERR_INVALID_ARG;
  }
  const PoolView& v = pool->view;
  if (v.D != 128 || v.kv_dtype == DMS_F32) {
    set_last_error("dms_project_append needs head_dim 128 and a bf16 or FP8 pool");
    return DMS_ERR_UNSUPPORTED;
  }
  if (layer < 0 || layer >= v.L || n_seqs < 1 || n_seqs > v.Bmax || d_model < 1) {
    set_last_error("bad layer / n_seqs / d_model (%d, %d, %d)", layer, n_seqs, d_model);
    return DMS_ERR_INVALID_ARG;
  }
  if (!pos || !x || !w_kv || !w_evict || !workspace || (reinterpret_cast<uintptr_t>(w_kv) & 15) ||
      (reinterpret_cast<uintptr_t>(pos) & 7) || (reinterpret_cast<uintptr_t>(workspace) & 15)) {
    set_last_error("null pointer, or w_kv / workspace not 16-byte or pos not 8-byte aligned");
    return DMS_ERR_INVALID_ARG;
  }
  size_t need = 0;
  dms_project_workspace_bytes(pool, n_seqs, d_model, &need);
  if (workspace_bytes < need) {
    set_last_error("workspace has %zu bytes, needs %zu", workspace_bytes, need);
    return DMS_ERR_CAPACITY;
  }
  static bool attr = false;
  const size_t smem = proj_smem(128);
  if (!attr) {
    dms_status st = cuda_status(cudaFuncSetAttribute(project_append_kernel<128>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)),
                                "projection smem attribute");
    if (st != DMS_OK) return st;
    attr = true;
  }
  const int KC = (d_model + kProjRows - 1) / kProjRows;
  for (int s0 = 0; s0 < n_seqs; s0 += kProjMaxSeqs) {   // sequences in launches of 8
    const int S = n_seqs - s0 < kProjMaxSeqs ? n_seqs - s0 : kProjMaxSeqs;
    project_append_kernel<128><<<dim3(KC, v.Hkv), kProjThreads, smem, stream>>>(
        v, layer, S, seq_ids ? seq_ids + s0 : nullptr, pos + s0,
        static_cast<const __nv_bfloat16*>(x) + int64_t(s0) * d_model, d_model,
        static_cast<const __nv_bfloat16*>(w_kv), static_cast<const __nv_bfloat16*>(w_evict), b_evict,
        threshold, static_cast<float*>(workspace), KC);
    dms_status st = cuda_status(cudaGetLastError(), "project_append_kernel");
    if (st != DMS_OK) return st;
  }
  return DMS_OK;
}
