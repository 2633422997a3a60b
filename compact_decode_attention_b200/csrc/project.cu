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
// weights.  One thread-block cluster of kProjCluster CTAs per kv-head: CTA
// rank r streams rows [r * R, (r + 1) * R) of the head's K and V columns
// (a warp reads 512 bytes of one row, 16 rows in flight per warp) and of its
// predictor column, and keeps its partial sums in shared memory; after a
// cluster barrier the rank-0 CTA adds the ranks' partials in rank order
// through distributed shared memory (deterministic, no global workspace),
// rounds k and v, decides the flag and stores the rows.  The slot each token
// takes does not depend on its values or flag, so rank 0 does the append
// bookkeeping while the weights stream and only sets the ring's flag bit at
// the end.
#include <cooperative_groups.h>

#include "append_core.cuh"

namespace dms {

namespace cg = cooperative_groups;

constexpr int kProjCluster = 8;    // CTAs per kv-head (portable cluster size)
constexpr int kProjMaxSeqs = 8;    // sequences per launch (the host loops)
constexpr int kProjWarps = 16;
constexpr int kProjThreads = 32 * kProjWarps;

// dynamic shared memory (floats): x slice [S][R], cross-warp partials
// [warps][S][256], logit partials [warps][S], this CTA's partial [S][257],
// finished rows [S][2][D], slots
__host__ __device__ constexpr size_t proj_smem(int D, int S, int R) {
  return (size_t(S) * R + size_t(kProjWarps) * S * 256 + size_t(kProjWarps) * S + size_t(S) * (2 * D + 1) +
          size_t(S) * 2 * D) * 4 + size_t(S) * 3 * 4 + 64;
}

// S sequences per launch (1..kProjMaxSeqs), a compile-time count
template <int D, int S>
__global__ void __launch_bounds__(kProjThreads)
    project_append_kernel(PoolView v, int layer, const int32_t* seq_ids, const int64_t* pos,
                          const __nv_bfloat16* x, int dm, const __nv_bfloat16* w_kv,
                          const __nv_bfloat16* w_ev, const float* b_ev, float thr) {
  static_assert(2 * D == 256, "one warp covers the head's K and V columns with 16-byte loads");
  constexpr int NC = 2 * D + 1;
  // weight rows in flight per warp (fewer as the per-sequence accumulators grow)
  constexpr int kProjUnroll = S <= 2 ? 16 : S <= 4 ? 8 : 4;
  extern __shared__ float psm[];
  const int R = ((dm + kProjCluster - 1) / kProjCluster + 7) / 8 * 8;
  float* xs = psm;                                         // [S][R]
  float* red = xs + S * R;                                 // [warps][S][256]
  float* lred = red + kProjWarps * S * 256;                // [warps][S]
  float* cpart = lred + kProjWarps * S;                    // [S][NC]
  float* rows = cpart + S * NC;                            // [S][2][D]
  int* slots = reinterpret_cast<int*>(rows + S * 2 * D);   // [S][3]
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = int(cluster.block_rank());
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x / kProjCluster;
  const int Hkv = v.Hkv;
  const int d0 = rank * R, nd = max(0, min(R, dm - d0));
  for (int i = tid; i < S * R; i += kProjThreads) {
    const int s = i / R, d = i % R;
    xs[i] = d < nd ? __bfloat162float(x[int64_t(s) * dm + d0 + d]) : 0.f;
  }
  const int64_t ldw = int64_t(2) * Hkv * D;

  if (rank == 0 && warp < S && lane == 0) {   // bookkeeping of sequence `warp` (flag bit 0 for now)
    const int s = warp;
    const int b = seq_ids ? seq_ids[s] : s;
    const int64_t tpos = pos[s];
    AppendSlot r{-1, -1, 0};
    if (b < 0 || b >= v.Bmax || tpos < 0 || tpos >= (int64_t(1) << 31))
      report_error(v.hdr, DMS_DEVERR_BAD_SEQUENCE, layer, s, h);
    else
      r = append_bookkeeping(v, layer, b, h, v.head(layer, b, h), int(tpos), 0u);
    slots[s * 3 + 0] = r.slot;
    slots[s * 3 + 1] = r.prow;
    slots[s * 3 + 2] = r.opened;
  }

  // ---- K and V columns: lane covers 8 columns (lanes 0-15 K, 16-31 V) ----
  __syncthreads();  // x slice staged
  float acc[S][8];
#pragma unroll
  for (int s = 0; s < S; ++s)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[s][e] = 0.f;
  const int col = lane < 16 ? h * D + 8 * lane : (Hkv + h) * D + 8 * (lane - 16);
  for (int d = warp; d < nd; d += kProjWarps * kProjUnroll) {
    uint4 raw[kProjUnroll];
#pragma unroll
    for (int u = 0; u < kProjUnroll; ++u) {
      const int dd = d + kProjWarps * u;
      raw[u] = dd < nd ? __ldg(reinterpret_cast<const uint4*>(w_kv + int64_t(d0 + dd) * ldw + col))
                       : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kProjUnroll; ++u) {
      const int dd = d + kProjWarps * u;
      if (dd >= nd) break;
      const __nv_bfloat16* wv = reinterpret_cast<const __nv_bfloat16*>(&raw[u]);
      float wf[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) wf[e] = __bfloat162float(wv[e]);
#pragma unroll
      for (int s = 0; s < S; ++s) {
        const float xv = xs[s * R + dd];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[s][e] = fmaf(xv, wf[e], acc[s][e]);
      }
    }
  }
  // ---- eviction logit: thread t covers rows t, t + 256, ... of the chunk ----
  float lacc[S];
#pragma unroll
  for (int s = 0; s < S; ++s) lacc[s] = 0.f;
  for (int d = tid; d < nd; d += kProjThreads) {
    const float we = __bfloat162float(w_ev[int64_t(d0 + d) * Hkv + h]);
#pragma unroll
    for (int s = 0; s < S; ++s) lacc[s] = fmaf(xs[s * R + d], we, lacc[s]);
  }
#pragma unroll
  for (int s = 0; s < S; ++s) {
    float t = lacc[s];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    if (lane == 0) lred[warp * S + s] = t;
#pragma unroll
    for (int e = 0; e < 8; ++e) red[(warp * S + s) * 256 + 8 * lane + e] = acc[s][e];
  }
  __syncthreads();
  // ---- this CTA's partial (warps added in order) ----
  for (int i = tid; i < S * 256; i += kProjThreads) {
    const int s = i / 256, c = i % 256;
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kProjWarps; ++w) t += red[(w * S + s) * 256 + c];
    cpart[s * NC + c] = t;
  }
  if (tid < S) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kProjWarps; ++w) t += lred[w * S + tid];
    cpart[tid * NC + 2 * D] = t;
  }
  cluster.sync();   // every rank's partial is in its shared memory

  if (rank == 0) {
    // ---- add the ranks' partials in rank order, round, decide, store ----
    for (int i = tid; i < S * NC; i += kProjThreads) {
      float t = 0.f;
#pragma unroll
      for (int r = 0; r < kProjCluster; ++r) t += cluster.map_shared_rank(cpart, r)[i];
      const int s = i / NC, c = i % NC;
      if (c < 2 * D) rows[s * 2 * D + c] = __bfloat162float(__float2bfloat16_rn(t));  // input precision
      else lred[s] = t;                                                                    // logit
    }
    __syncthreads();
    for (int s = warp; s < S; s += kProjWarps) {
      const float lg = lred[s] + (b_ev ? b_ev[h] : 0.f);
      const int slot = slots[s * 3 + 0], prow = slots[s * 3 + 1], opened = slots[s * 3 + 2];
      if (slot < 0) continue;
      if (lane == 0 && lg > thr) {   // the flag bit of the ring entry written at the start
        const int b = seq_ids ? seq_ids[s] : s;
        v.ring[int64_t(v.head(layer, b, h)) * v.w + int(pos[s]) % v.w] |= 1u << 31;
      }
      store_row_from_float(v, layer, h, prow, opened, rows + s * 2 * D, rows + s * 2 * D + D, lane);
    }
  }
  cluster.sync();   // rank 0 has read every rank's shared memory
}

template <int S>
static dms_status launch_projection(const PoolView& v, int layer, const int32_t* ids, const int64_t* pos,
                                    const __nv_bfloat16* x, int dm, int R, const void* w_kv, const void* w_evict,
                                    const float* b_evict, float threshold, cudaStream_t stream) {
  const size_t smem = proj_smem(128, S, R);
  if (smem > 227 * 1024) {
    set_last_error("d_model %d too large for the projection's shared memory", dm);
    return DMS_ERR_UNSUPPORTED;
  }
  static FuncAttrCache smem_attr;   // per instantiation and device: the largest size set so far
  dms_status ast = ensure_func_attr(reinterpret_cast<const void*>(project_append_kernel<128, S>),
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem), smem_attr,
                                    "projection smem attribute");
  if (ast != DMS_OK) return ast;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kProjCluster * v.Hkv);
  cfg.blockDim = dim3(kProjThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr_c[1];
  attr_c[0].id = cudaLaunchAttributeClusterDimension;
  attr_c[0].val.clusterDim.x = kProjCluster;
  attr_c[0].val.clusterDim.y = 1;
  attr_c[0].val.clusterDim.z = 1;
  cfg.attrs = attr_c;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, project_append_kernel<128, S>, v, layer, ids, pos, x, dm,
                                        static_cast<const __nv_bfloat16*>(w_kv),
                                        static_cast<const __nv_bfloat16*>(w_evict), b_evict, threshold),
                     "project_append_kernel");
}

}  // namespace dms

using namespace dms;

extern "C" dms_status dms_project_workspace_bytes(const dms_pool* pool, int n_seqs, int d_model,
                                                  size_t* bytes) {
  if (!pool || !bytes || n_seqs < 1 || d_model < 1) {
    set_last_error("bad arguments");
    return DMS_ERR_INVALID_ARG;
  }
  *bytes = 0;   // the cluster reduces in distributed shared memory
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
  if (!pos || !x || !w_kv || !w_evict || (reinterpret_cast<uintptr_t>(w_kv) & 15) ||
      (reinterpret_cast<uintptr_t>(pos) & 7)) {
    set_last_error("null pointer, or w_kv not 16-byte or pos not 8-byte aligned");
    return DMS_ERR_INVALID_ARG;
  }
  (void)workspace;
  (void)workspace_bytes;
  const int R = ((d_model + kProjCluster - 1) / kProjCluster + 7) / 8 * 8;
  for (int s0 = 0; s0 < n_seqs; s0 += kProjMaxSeqs) {   // sequences in launches of up to 8
    const int S = n_seqs - s0 < kProjMaxSeqs ? n_seqs - s0 : kProjMaxSeqs;
    const int32_t* ids = seq_ids ? seq_ids + s0 : nullptr;
    const __nv_bfloat16* xs = static_cast<const __nv_bfloat16*>(x) + int64_t(s0) * d_model;
    dms_status st = DMS_OK;
    switch (S) {
      case 1: st = launch_projection<1>(v, layer, ids, pos + s0, xs, d_model, R, w_kv, w_evict, b_evict, threshold, stream); break;
      case 2: st = launch_projection<2>(v, layer, ids, pos + s0, xs, d_model, R, w_kv, w_evict, b_evict, threshold, stream); break;
      case 3: st = launch_projection<3>(v, layer, ids, pos + s0, xs, d_model, R, w_kv, w_evict, b_evict, threshold, stream); break;
      case 4: st = launch_projection<4>(v, layer, ids, pos + s0, xs, d_model, R, w_kv, w_evict, b_evict, threshold, stream); break;
      case 5: st = launch_projection<5>(v, layer, ids, pos + s0, xs, d_model, R, w_kv, w_evict, b_evict, threshold, stream); break;
      case 6: st = launch_projection<6>(v, layer, ids, pos + s0, xs, d_model, R, w_kv, w_evict, b_evict, threshold, stream); break;
      case 7: st = launch_projection<7>(v, layer, ids, pos + s0, xs, d_model, R, w_kv, w_evict, b_evict, threshold, stream); break;
      default: st = launch_projection<8>(v, layer, ids, pos + s0, xs, d_model, R, w_kv, w_evict, b_evict, threshold, stream); break;
    }
    if (st != DMS_OK) return st;
  }
  return DMS_OK;
}
