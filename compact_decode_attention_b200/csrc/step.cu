// Decode attention for calls with few heads, one thread-block cluster per
// head, and the decode step (append/evict fused with it) built on it.
//
// DMS decode is bound by reading each head's retained tokens ("Nvidia DMS
// ..." (stiva.ai), opening section; FastDMS page: faster decode from less
// KV).  A model issues one layer per call (layer l+1's query needs layer
// l's output), and one layer holds few heads (8 kv-heads at batch 1): the
// stream-K kernel then spends most of its time on fixed costs -- a scan of
// every head's held count before any copy, a block-table lookup after it,
// few CTAs streaming many blocks each, and cross-CTA merges through global
// memory with an arrival ticket.
//
// Here each head gets a cluster of C CTAs (C = 16, 8, 4, 2 or 1: as many as
// keep every cluster of the call resident at once).  CTA j of a head takes
// the head's blocks j, j + C, j + 2C, ...; its producer warp loads its
// block-table entries in the same round trip as the head's held count, so
// the first copies go out one memory round trip after the kernel may start,
// and a helper warp prefetches the CTA's blocks into L2 before the previous
// kernel has finished (a hint: nothing it reads is used afterwards).  Each
// CTA's consumer warps run the same unit compute as the stream-K kernel
// (attn_warp.cuh) and combine into one partial softmax state in the CTA's
// shared memory.  The CTA then sends it with TMA bulk copies between shared
// memories of the cluster, one per CTA (issued by one lane each): that
// CTA's slice of the head's outputs together with this CTA's (max, sum)
// pairs, completing bytes on the receiver's mbarrier.  A CTA waits (bounded)
// for its own barrier -- every CTA's piece landed -- and merges its slice by
// log-sum-exp from its own shared memory: no global workspace, no tickets,
// no remote loads.
//
// The fused step (dms_decode_step_layers) runs the append/evict of the
// step's token in the same launch.  Every CTA of a head reads the head's
// state from before the append (held count n, and the slot the step reuses:
// the retired slot of token t - w when it was flagged) and arrives at a
// cluster barrier; CTA 0's helper warp waits on it and only then appends
// (the same per-head code as dms_append_evict).  The same barrier tells
// every CTA, before its first copy into another CTA's shared memory, that
// the whole cluster runs.  The attention masks the reused slot (its row is
// being overwritten) and takes the new token as one more unit: the last CTA
// of the cluster writes the token's row, in the store's format, into a
// shared-memory stage and computes it like any staged block.  So the result
// is the attention over exactly the rows dms_append_evict then
// dms_decode_attn would see.  Rows a concurrent append may be writing are
// never read unmasked: the reused slot is masked and a new slot lies past
// every range read.
//
// Every mbarrier wait is bounded by the pool's wait limit.  The one cluster
// barrier is a hardware barrier that every thread of every CTA arrives at
// with the same instruction at the same point (a warp never splits over two
// arrive forms: a warp whose lanes arrived with two different forms left the
// barrier's phase count wrong and the cluster waiting for good) and waits on
// exactly once, so it cannot wait for a missing arrival.
#include <mutex>

#include "append_core.cuh"
#include "attn_warp.cuh"

namespace dms {

template <int KV, int D>
struct ClusterTraits {
  using A = AttnTraits<KV, D>;
  // Stages and consumer warps: a CTA of a small call holds a few blocks, so
  // a few stages in flight cover it, and at most 113 KB of shared memory
  // lets two CTAs share an SM (so a 16-CTA cluster needs 8 SMs of a GPC, and
  // the next launch's CTAs start under this one's).
  static constexpr int NS = KV == KV_F32 ? 2 : KV == KV_INT4 ? 6 : KV == KV_FP8 ? 6 : D == 128 ? 3 : 6;
  static constexpr int NCW = KV == KV_F32 ? 2 : 3;
  // consumer warps, then the producer warp, then a helper warp (prefetch
  // before the launch dependency resolves; the fused step's append)
  static constexpr int THREADS = 32 * (NCW + 2);
  static constexpr int kMaxC = 16;
  // Shared memory for a GQA group of g query heads: stages, the consumer
  // warps' states (g rows each), this CTA's partial (g rows, then max and
  // sum), and the receive buffer of the cluster merge (every CTA's slice of
  // g * D / C outputs with its 16 max/sum values), mbarriers, flags.
  static constexpr size_t smem(int g) {
    return size_t(NS) * A::STAGEB + size_t(NCW * g * D + 2 * NCW * 8) * 4 +
           size_t(2 * (g * D + 16 * kMaxC) + 8) * 4 + (2 * NS + 1) * 8 + 16 * 4;
  }
  static constexpr size_t SMEM_MAX = smem(8);
  static constexpr int CTAS_PER_SM = (KV == KV_F32 && D == 128) ? 1 : 2;   // registers are capped to match
  static_assert(NS % NCW == 0, "each stage must always belong to the same consumer warp");
  static_assert(SMEM_MAX <= 227 * 1024, "shared memory budget");
  // two CTAs per SM at the usual GQA groups (g <= 4)
  static_assert(CTAS_PER_SM == 1 || smem(4) + 1024 <= 228 * 1024 / 2, "two CTAs per SM");
};

struct ClusterParams {
  PoolView v;
  int l0, batch;
  const uint8_t* q;        // [nl, batch, Hq, D] q dtype
  uint8_t* out;            // same layout
  float scale_log2;
  // fused step only: the token at position pos of every head
  const uint8_t* knew;     // [nl, batch, Hkv, D] input dtype
  const uint8_t* vnew;
  const uint8_t* evict;    // [nl, batch, Hkv]
  int64_t pos;
};

__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
}
__device__ __forceinline__ void fence_acq_rel_cluster() {
  asm volatile("fence.acq_rel.cluster;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t dsmem_addr(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
// Bulk copy (TMA) of `bytes` from this CTA's shared memory to another
// CTA's (dst, completing `bytes` on that CTA's mbarrier mbar): both are
// shared::cluster addresses from dsmem_addr.
__device__ __forceinline__ void bulk_s2dsmem(uint32_t dst, uint32_t src, uint32_t bytes, uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "r"(src), "r"(bytes), "r"(mbar)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_and_wait_read() {
  asm volatile("cp.async.bulk.commit_group;\n\tcp.async.bulk.wait_group.read 0;" ::: "memory");
}

// The step's new token as row 0 of a staged block image, in the store's
// format (the same bytes dms_append_evict writes into the pool), so that the
// unit compute takes it like any held row.  One warp.
template <int KV, int D, typename InT>
__device__ __forceinline__ void stage_new_row(uint8_t* st, const InT* krow, const InT* vrow, float sK,
                                              float sV, int lane) {
  using T = AttnTraits<KV, D>;
  if constexpr (KV == KV_BF16 || KV == KV_F32) {
    // row 0: chunk c sits at chunk c ^ 0; the input is in the store's dtype
    constexpr int kChunks = D * T::ESZ / 16;
    for (int c = lane; c < 2 * kChunks; c += 32) {
      const uint8_t* src = reinterpret_cast<const uint8_t*>(c < kChunks ? krow : vrow) + (c % kChunks) * 16;
      *reinterpret_cast<uint4*>(st + (c < kChunks ? 0 : T::TILEB) + (c % kChunks) * 16) =
          *reinterpret_cast<const uint4*>(src);
    }
  } else if constexpr (KV == KV_FP8) {
    for (int d = lane; d < D; d += 32) {
      st[fp8k_byte(0, d)] = f32_to_e4m3(__fdiv_rn(in_to_f32(krow[d]), sK));
      st[T::TILEB + fp8v_byte(0, d)] = f32_to_e4m3(__fdiv_rn(in_to_f32(vrow[d]), sV));
    }
  } else {  // 4-bit: the other token columns' V scales must read 0 (probability 0 times a finite scale)
    uint32_t* vs = reinterpret_cast<uint32_t*>(st + T::TILEB + kInt4Nibbles);
    for (int c = lane; c < 4 * kBlockTokens * 2 / 4; c += 32) vs[c] = 0u;
    __syncwarp();
    float k4[4], v4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      k4[e] = in_to_f32(krow[4 * lane + e]);
      v4[e] = in_to_f32(vrow[4 * lane + e]);
    }
    store_row_int4_at(st, 0, T::TILEB, k4, v4, lane);
  }
}

template <int KV>
struct StoreOf {
  static constexpr int value = KV == KV_FP8 ? 1 : KV == KV_INT4 ? 2 : 0;
};

template <int KV, int D, typename InT, bool FUSED>
__global__ void __launch_bounds__(ClusterTraits<KV, D>::THREADS, ClusterTraits<KV, D>::CTAS_PER_SM)
    decode_cluster_kernel(const ClusterParams p) {
  using CT = ClusterTraits<KV, D>;
  using T = AttnTraits<KV, D>;
  using W = typename WarpSel<KV, D>::type;
  constexpr int NS = CT::NS, NCW = CT::NCW, kThreads = CT::THREADS, kCons = 32 * NCW;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* stages = smem;
  const int g = p.v.Hq / p.v.Hkv;
  float* s_ow = reinterpret_cast<float*>(smem + size_t(NS) * T::STAGEB);   // [NCW][g][D]
  float* s_mw = s_ow + NCW * g * D;
  float* s_lw = s_mw + NCW * 8;
  // the cluster merge: this CTA's partial laid out per receiving CTA r as
  // [chunk outputs of r's slice][max [8], sum [8]] (the source of one bulk
  // copy to each CTA), and the receive buffer of the same shape holding
  // every CTA's piece for this CTA's slice ([sender][chunk + 16])
  float* s_po = s_lw + NCW * 8;
  float* s_rx = s_po + g * D + 16 * CT::kMaxC;
  float* s_L = s_rx + g * D + 16 * CT::kMaxC;   // merged softmax sums [8]
  uint64_t* full = reinterpret_cast<uint64_t*>(s_L + 8);
  uint64_t* empty = full + NS;
  uint64_t* rxbar = empty + NS;        // completes when every CTA's piece has landed here
  int* s_misc = reinterpret_cast<int*>(rxbar + 1);
  volatile int* s_abort = s_misc;

  const PoolView& v = p.v;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int C = int(cluster_size()), j = int(cluster_rank());
  const int i = blockIdx.x / C;                      // head of the call
  const int h = i % v.Hkv, lb = i / v.Hkv;           // lb = layer-in-call * batch + b
  const int b = lb % p.batch, l = p.l0 + lb / p.batch;
  const int hd = v.head(l, b, h);
  const int t = int(p.pos);

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(rxbar, 1);
    if (C > 1)   // every CTA of the cluster sends this CTA its slice and its (max, sum) pairs
      mbar_arrive_expect_tx(rxbar, uint32_t(g * D + 16 * C) * 4);
    s_misc[0] = 0;
    s_misc[3] = 0;
    fence_mbar_init();
  }
  if constexpr (T::QB > 0) {  // fp32 path: query rows g..7 of every stage stay zero (padding)
    for (int s = 0; s < NS; ++s) {
      uint4* qa = reinterpret_cast<uint4*>(stages + size_t(s) * T::STAGEB + 2 * T::TILEB);
      for (int e = tid; e < T::QB / 16; e += kThreads) qa[e] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  pdl_launch_dependents();
  if (warp == NCW + 1) {
    // helper warp, before the previous kernel's writes are visible: prefetch
    // this CTA's blocks (and the head's state the producer reads next) into
    // L2 from the head's current count and block table.  A hint only --
    // values read here may be stale, nothing read here is used after the
    // wait, and only addresses inside the pool are touched -- so the loads
    // and copies after the wait find their lines in L2.
    if (lane == 0 && FUSED) {
      prefetch_l2(v.ring + int64_t(hd) * v.w + t % v.w);
      prefetch_l2(v.free_top + hd);
    }
    const int n_hint = __ldcg(v.n_slots + hd);
    const int nb_hint = units_of(max(0, n_hint));
    for (int64_t e = j + int64_t(lane) * C; e < nb_hint && e < v.mbh; e += 32 * int64_t(C)) {
      const int blk = __ldcg(v.bt + int64_t(hd) * v.mbh + e);
      if (blk >= 0 && blk < v.max_blocks)
        bulk_prefetch_l2(v.blocks + int64_t(blk) * v.block_bytes, uint32_t(v.block_bytes));
    }
  }
  pdl_wait_prerequisites();

  // ---- the head's state before this step's append: held count and the
  // slot the append reuses (producer warp, one round trip; the block-table
  // entries of this CTA's first 32 blocks load in the same trip) ----
  int bt_reg = 0;
  if (warp == NCW) {
    const int64_t e0 = j + int64_t(lane) * C;
    if (e0 < v.mbh) bt_reg = v.bt[int64_t(hd) * v.mbh + e0];
    if (lane == 0) {
      const int n = v.n_slots[hd];
      int hole = -1;
      if constexpr (FUSED) {
        const uint32_t e = v.ring[int64_t(hd) * v.w + t % v.w];
        const int ft = v.free_top[hd];
        if (t >= v.w && (e >> 31)) hole = int(e & 0x7fffffffu);
        else if (ft > 0) hole = v.free_stack[int64_t(hd) * v.free_cap + ft - 1];
      }
      s_misc[1] = n;
      s_misc[2] = hole;
      if (FUSED) fence_acq_rel_cluster();   // these reads come before the append (phase 1 below)
    }
  }
  __syncthreads();
  const int n_old = s_misc[1], hole = s_misc[2];
  // Cluster barrier, phase 1: this CTA has started and has read the state
  // the append changes.  Waiting on it tells a CTA that every CTA of its
  // cluster is running -- required before it writes into another CTA's
  // shared memory -- and, in CTA 0, that the append may begin (the thread
  // that read the state fenced its reads above).  Every thread executes the
  // same arrive instruction: a warp never splits over two arrive forms.
  if (C > 1) cluster_arrive_relaxed();
  const int nb = units_of(n_old);
  const int nreal = nb > j ? (nb - j + C - 1) / C : 0;
  const bool virt = FUSED && j == C - 1;
  const int nunits = nreal + (virt ? 1 : 0);
  const int qrow_bytes = g * D * T::QESZ;
  const uint8_t* qg = p.q + int64_t(lb) * v.Hq * D * T::QESZ + int64_t(h) * qrow_bytes;
  using InPtr = const InT*;
  const InT* krow = FUSED ? reinterpret_cast<InPtr>(p.knew) + int64_t(i) * D : nullptr;
  const InT* vrow = FUSED ? reinterpret_cast<InPtr>(p.vnew) + int64_t(i) * D : nullptr;
  float sK = 1.f, sV = 1.f;
  if constexpr (KV == KV_FP8) {
    sK = v.scales[(int64_t(l) * v.Hkv + h) * 2 + 0];
    sV = v.scales[(int64_t(l) * v.Hkv + h) * 2 + 1];
  }

  if (warp == NCW) {
    // ======================= producer =======================
    const uint64_t pol = policy_evict_first();
    const uint64_t qpol = policy_evict_last();
    int issued = 0;
    bool aborted = false;
    for (int k = 0; k < nunits; ++k) {
      if (k >= 32 && (k & 31) == 0) {   // the next 32 block-table entries
        const int64_t e = j + int64_t(k + lane) * C;
        bt_reg = e < v.mbh ? v.bt[int64_t(hd) * v.mbh + e] : 0;
      }
      const int blk = __shfl_sync(0xffffffffu, bt_reg, k & 31);
      const int s = k % NS;
      const uint32_t ph = (k / NS) & 1;
      bool ok = false;
      if (lane == 0 && !aborted) {
        ok = mbar_wait_bounded(&empty[s], ph ^ 1, s_abort, v.wait_ns) && !*s_abort;
        if (!ok) {
          if (!*s_abort) report_error(v.hdr, DMS_DEVERR_TIMEOUT, l, b, h);
          *s_abort = 1;
          aborted = true;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) continue;
      uint8_t* st = stages + size_t(s) * T::STAGEB;
      if (k < nreal) {
        const int bi = j + k * C;
        const int rows = min(kBlockTokens, n_old - bi * kBlockTokens);
        if (lane == 0) {
          if (!DMS_CHECK(blk >= 0 && blk < v.max_blocks && rows >= 1, v.hdr, 401, blk, rows)) {
            *s_abort = 1;
            aborted = true;
          } else {
            const uint8_t* src = v.blocks + int64_t(blk) * v.block_bytes;
            const uint32_t kbytes = uint32_t(rows) * T::ROWB;
            const bool whole = rows == kBlockTokens || KV == KV_INT4;
            const uint32_t vbytes = (whole || KV == KV_FP8) ? T::TILEB : kbytes;
            mbar_arrive_expect_tx(&full[s], (whole ? T::TILEB : kbytes) + vbytes +
                                                (T::QB > 0 ? qrow_bytes : 0));
            if (whole) {
              bulk_g2s(st, src, 2 * T::TILEB, &full[s], pol);
            } else {
              bulk_g2s(st, src, kbytes, &full[s], pol);
              bulk_g2s(st + T::TILEB, src + T::TILEB, vbytes, &full[s], pol);
            }
            if constexpr (T::QB > 0) bulk_g2s(st + 2 * T::TILEB, qg, qrow_bytes, &full[s], qpol);
            issued = k + 1;
          }
        }
      } else if constexpr (FUSED) {
        // the new token, written into the stage by this warp (generic
        // stores; the mbarrier arrive releases them to the consumer)
        stage_new_row<KV, D, InT>(st, krow, vrow, sK, sV, lane);
        if constexpr (T::QB > 0) {
          for (int e = lane; e < qrow_bytes / 16; e += 32)
            reinterpret_cast<uint4*>(st + 2 * T::TILEB)[e] = reinterpret_cast<const uint4*>(qg)[e];
        }
        fence_proxy_async_smem();   // before any later bulk copy into this stage
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&full[s]);
          issued = k + 1;
        }
      }
      aborted = __shfl_sync(0xffffffffu, aborted, 0);
    }
    __syncwarp();
    if (C > 1) cluster_wait();   // phase 1 (see above)
    // drain: no copy into this CTA's shared memory may be in flight at exit
    if (lane == 0) {
      volatile int never = 0;
      for (int kk = max(0, issued - NS); kk < issued; ++kk)
        mbar_wait_bounded(&full[kk % NS], (kk / NS) & 1, &never, v.wait_ns);
    }
    __syncwarp();
  } else if (warp == NCW + 1) {
    // ======================= helper =======================
    __syncwarp();
    if (C > 1) cluster_wait();   // phase 1
    if constexpr (FUSED) {
      if (j == 0) {   // the append, once every CTA of the head has read the old state
        const uint32_t flag = lane == 0 ? uint32_t(p.evict[i] != 0) : 0u;
        append_head_warp<InT, StoreOf<KV>::value>(v, l, b, h, hd, t, krow, vrow, flag, lane);
      }
    }
    __syncwarp();
  } else {
    // ======================= consumers =======================
    W st;
    st.reset();
    if constexpr (KV == KV_F32) st.g = g;
    st.scale = p.scale_log2;
    st.vscale = 1.f;
    if constexpr (KV == KV_FP8) {
      st.scale = p.scale_log2 * sK;
      st.vscale = sV;
    }
    if constexpr (KV != KV_F32) {
      if (warp < nunits) st.load_q(qg, g, lane);
    }
    for (int k = warp; k < nunits; k += NCW) {
      const int s = k % NS;
      const uint32_t ph = (k / NS) & 1;
      bool ok = false;
      if (!*s_abort) {
        ok = mbar_wait_bounded(&full[s], ph, s_abort, v.wait_ns);
        if (!ok && lane == 0) {
          *s_abort = 1;
          report_error(v.hdr, DMS_DEVERR_TIMEOUT, l, b, h);
        }
      }
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        int rows = 1, hr = -1;
        if (k < nreal) {
          const int bi = j + k * C;
          rows = min(kBlockTokens, n_old - bi * kBlockTokens);
          if (hole >= 0 && hole / kBlockTokens == bi) hr = hole % kBlockTokens;
        }
        st.unit(stages + size_t(s) * T::STAGEB, rows, lane, hr);
      }
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(&empty[s]);
    }
    st.write_state(s_ow + warp * g * D, s_mw + warp * 8, s_lw + warp * 8, g, lane);
    __syncwarp();
    if (C > 1) cluster_wait();   // phase 1: every CTA of the cluster runs (before the pushes below)
    consumer_bar<NCW>();
    // this CTA's partial over its warps (or the output, when the head has one CTA)
    const int64_t orow = int64_t(lb) * v.Hq + int64_t(h) * g;
    for (int idx = tid; idx < g * D; idx += kCons) {
      const int nn = idx / D, d = idx % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NCW; ++w) M = fmaxf(M, s_mw[w * 8 + nn]);
      float o = 0.f, L = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < NCW; ++w) {
          const float f = fast_exp2(s_mw[w * 8 + nn] - M);
          o += f * s_ow[(w * g + nn) * D + d];
          L += f * s_lw[w * 8 + nn];
        }
      }
      if (C == 1) {
        store_out<T::QESZ>(p.out, orow * D + idx, L > 0.f ? o / L : 0.f);
      } else {
        // output element idx is merged by CTA idx / chunk: push this CTA's
        // partial value to it, and this CTA's (max, sum) of query head nn
        // to every CTA of the cluster
        const int chunk = (g * D) / C, r = idx / chunk;
        s_po[r * (chunk + 16) + idx - r * chunk] = o;
        if (d == 0) {
          for (int q = 0; q < C; ++q) {
            s_po[q * (chunk + 16) + chunk + nn] = M;
            s_po[q * (chunk + 16) + chunk + 8 + nn] = L;
          }
        }
      }
    }
    if (C > 1) {
      // output element idx is merged by CTA idx / chunk: one bulk copy to
      // each CTA r of the cluster (lane r issues it) moves it this CTA's
      // slice of r's outputs and this CTA's (max, sum) pairs
      fence_proxy_async_smem();   // the generic writes above, before the bulk copies read them
      consumer_bar<NCW>();
      if (warp == 0 && lane < C) {
        const int piece = (g * D) / C + 16;
        bulk_s2dsmem(dsmem_addr(smem_u32(s_rx + j * piece), lane), smem_u32(s_po + lane * piece),
                     uint32_t(piece) * 4, dsmem_addr(smem_u32(rxbar), lane));
        bulk_commit_and_wait_read();   // the source stays valid until read
      }
    }
  }

  if (C > 1) {
    // ---- merge over the cluster: after this barrier every CTA holds, in its
    // own shared memory, every CTA's slice of the outputs it merges; CTA j
    // writes outputs [j*chunk, (j+1)*chunk).  Nothing reads another CTA's
    // memory after the barrier, so each CTA may leave when it is done. ----
    if (tid == 0) {   // every CTA's pieces have landed in this CTA's buffers
      volatile int never = 0;
      if (!mbar_wait_bounded(rxbar, 0, &never, v.wait_ns)) {
        report_error(v.hdr, DMS_DEVERR_TIMEOUT, l, b, h);
        s_misc[3] = 1;
      }
    }
    __syncthreads();
    if (warp == 0) {   // per query head: max over the C partials, their factors and sum (lanes = ranks)
      const int piece = (g * D) / C + 16, chunk = piece - 16;
      for (int nn = 0; nn < g; ++nn) {
        const float m = lane < C ? s_rx[lane * piece + chunk + nn] : -INFINITY;
        float M = m;
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        const float f = (lane < C && M != -INFINITY) ? fast_exp2(m - M) : 0.f;
        float L = lane < C ? f * s_rx[lane * piece + chunk + 8 + nn] : 0.f;
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
        __syncwarp();
        if (lane < C) s_rx[lane * piece + chunk + nn] = f;   // the max's slot now holds the factor
        if (lane == 0) s_L[nn] = L;
      }
    }
    __syncthreads();
    const int chunk = (g * D) / C, piece = chunk + 16;
    const int64_t orow = int64_t(lb) * v.Hq + int64_t(h) * g;
    const bool ok = s_misc[3] == 0;
    for (int e = tid; e < chunk; e += kThreads) {
      const int idx = j * chunk + e, nn = idx / D;
      float o = 0.f;
      for (int r = 0; r < C; ++r) o += s_rx[r * piece + chunk + nn] * s_rx[r * piece + e];
      const float L = s_L[nn];
      store_out<T::QESZ>(p.out, orow * D + idx, ok && L > 0.f ? o / L : 0.f);
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

// Most clusters of C CTAs of this kernel that can be resident at once on the
// current device (cached per kernel, device and C).
struct ClusterCapacity {
  std::mutex mu;
  int value[kAttrDevices][5];   // C = 1, 2, 4, 8, 16; 0 = not asked yet
};

template <typename K>
static int cluster_capacity(K kernel, size_t smem, int threads, int C, ClusterCapacity& cache) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kAttrDevices) return 0;
  const int ci = C == 1 ? 0 : C == 2 ? 1 : C == 4 ? 2 : C == 8 ? 3 : 4;
  std::lock_guard<std::mutex> lock(cache.mu);
  if (cache.value[dev][ci] == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    cache.value[dev][ci] = n > 0 ? n : -1;
  }
  return cache.value[dev][ci];
}

template <int KV, int D, typename InT, bool FUSED>
static dms_status cluster_setup(int* C_out, int n_heads, int g) {
  using CT = ClusterTraits<KV, D>;
  auto kernel = decode_cluster_kernel<KV, D, InT, FUSED>;
  static FuncAttrCache smem_attr, portable_attr;
  dms_status st = ensure_func_attr(reinterpret_cast<const void*>(kernel),
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, int(CT::SMEM_MAX), smem_attr,
                                   "cluster attn smem attribute");
  if (st != DMS_OK) return st;
  st = ensure_func_attr(reinterpret_cast<const void*>(kernel), cudaFuncAttributeNonPortableClusterSizeAllowed,
                        1, portable_attr, "cluster size attribute");
  if (st != DMS_OK) return st;
  static ClusterCapacity cap[9];   // per GQA group size
  int C = CT::kMaxC;
  while (C > 1 && cluster_capacity(kernel, CT::smem(g), CT::THREADS, C, cap[g]) < n_heads) C /= 2;
  *C_out = C;
  return DMS_OK;
}

template <int KV, int D, typename InT, bool FUSED>
static dms_status launch_cluster(const ClusterParams& prm, int n_heads, int C, cudaStream_t stream) {
  using CT = ClusterTraits<KV, D>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(n_heads * C));
  cfg.blockDim = dim3(CT::THREADS);
  cfg.dynamicSmemBytes = CT::smem(prm.v.Hq / prm.v.Hkv);
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
  return cuda_status(cudaLaunchKernelEx(&cfg, decode_cluster_kernel<KV, D, InT, FUSED>, prm),
                     "decode_cluster_kernel");
}

// Cluster size for a call over n_heads heads: the largest C with every
// cluster resident at once; below 2 the caller uses the stream-K kernel
// unless `force` (then clusters of one CTA run in waves).
template <int KV, int D, typename InT, bool FUSED>
static dms_status run_cluster(const ClusterParams& prm, int n_heads, bool force, cudaStream_t stream,
                              bool* done) {
  int C = 0;
  *done = false;
  dms_status st = cluster_setup<KV, D, InT, FUSED>(&C, n_heads, prm.v.Hq / prm.v.Hkv);
  if (st != DMS_OK || (C < 2 && !force)) return st;
  *done = true;
  return launch_cluster<KV, D, InT, FUSED>(prm, n_heads, C, stream);
}

// Try the cluster kernel for a call (attention only when knew is null, else
// the fused step).  *done = false: the call has too many heads for it.
dms_status cluster_attn(dms_pool* pool, int layer0, int n_layers, int batch, const void* q, void* out,
                        float sm_scale, const void* knew, const void* vnew, dms_dtype in_dtype,
                        const uint8_t* evict, int64_t pos, bool force, cudaStream_t stream,
                        bool* done) {
  const PoolView& v = pool->view;
  ClusterParams prm;
  prm.v = v;
  prm.l0 = layer0;
  prm.batch = batch;
  prm.q = static_cast<const uint8_t*>(q);
  prm.out = static_cast<uint8_t*>(out);
  const float sc = sm_scale > 0.f ? sm_scale : 1.0f / sqrtf(float(v.D));
  prm.scale_log2 = sc * 1.4426950408889634f;
  prm.knew = static_cast<const uint8_t*>(knew);
  prm.vnew = static_cast<const uint8_t*>(vnew);
  prm.evict = evict;
  prm.pos = pos;
  const int H = n_layers * batch * v.Hkv;
  using bf = __nv_bfloat16;
  if (!knew) {
    if (v.kv_dtype == DMS_BF16)
      return v.D == 128 ? run_cluster<KV_BF16, 128, bf, false>(prm, H, force, stream, done)
                        : run_cluster<KV_BF16, 64, bf, false>(prm, H, force, stream, done);
    if (v.kv_dtype == DMS_FP8_E4M3) return run_cluster<KV_FP8, 128, bf, false>(prm, H, force, stream, done);
    if (v.kv_dtype == DMS_INT4) return run_cluster<KV_INT4, 128, bf, false>(prm, H, force, stream, done);
    return v.D == 128 ? run_cluster<KV_F32, 128, float, false>(prm, H, force, stream, done)
                      : run_cluster<KV_F32, 64, float, false>(prm, H, force, stream, done);
  }
  const bool f32 = in_dtype == DMS_F32;
  if (v.kv_dtype == DMS_BF16)
    return v.D == 128 ? run_cluster<KV_BF16, 128, bf, true>(prm, H, force, stream, done)
                      : run_cluster<KV_BF16, 64, bf, true>(prm, H, force, stream, done);
  if (v.kv_dtype == DMS_FP8_E4M3)
    return f32 ? run_cluster<KV_FP8, 128, float, true>(prm, H, force, stream, done)
               : run_cluster<KV_FP8, 128, bf, true>(prm, H, force, stream, done);
  if (v.kv_dtype == DMS_INT4)
    return f32 ? run_cluster<KV_INT4, 128, float, true>(prm, H, force, stream, done)
               : run_cluster<KV_INT4, 128, bf, true>(prm, H, force, stream, done);
  return v.D == 128 ? run_cluster<KV_F32, 128, float, true>(prm, H, force, stream, done)
                    : run_cluster<KV_F32, 64, float, true>(prm, H, force, stream, done);
}

}  // namespace dms

using namespace dms;

extern "C" dms_status dms_decode_attn_plan(dms_pool* pool, int n_layers, int batch, int* kernel,
                                           int* cluster_size) {
  if (!pool || !kernel || !cluster_size || n_layers < 1 || batch < 1) {
    set_last_error("bad arguments");
    return DMS_ERR_INVALID_ARG;
  }
  const PoolView& v = pool->view;
  const int H = n_layers * batch * v.Hkv, g = v.Hq / v.Hkv;
  *kernel = DMS_ATTN_STREAM_K;
  *cluster_size = 0;
  if (pool->attn_kernel == DMS_ATTN_STREAM_K) return DMS_OK;
  int C = 0;
  using bf = __nv_bfloat16;
  dms_status st;
  if (v.kv_dtype == DMS_BF16)
    st = v.D == 128 ? cluster_setup<KV_BF16, 128, bf, false>(&C, H, g) : cluster_setup<KV_BF16, 64, bf, false>(&C, H, g);
  else if (v.kv_dtype == DMS_FP8_E4M3)
    st = cluster_setup<KV_FP8, 128, bf, false>(&C, H, g);
  else if (v.kv_dtype == DMS_INT4)
    st = cluster_setup<KV_INT4, 128, bf, false>(&C, H, g);
  else
    st = v.D == 128 ? cluster_setup<KV_F32, 128, float, false>(&C, H, g) : cluster_setup<KV_F32, 64, float, false>(&C, H, g);
  if (st != DMS_OK) return st;
  if (C >= 2 || pool->attn_kernel == DMS_ATTN_CLUSTER) {
    *kernel = DMS_ATTN_CLUSTER;
    *cluster_size = C;
  }
  return DMS_OK;
}

extern "C" dms_status dms_decode_step_layers(dms_pool* pool, int layer0, int n_layers, int batch,
                                             int64_t pos, const void* k, const void* v,
                                             dms_dtype in_dtype, const uint8_t* evict, const void* q,
                                             dms_dtype q_dtype, void* out, float sm_scale,
                                             void* workspace, size_t workspace_bytes,
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
  if (!k || !v || !evict || !q || !out || !workspace) {
    set_last_error("null k / v / evict / q / out / workspace");
    return DMS_ERR_INVALID_ARG;
  }
  const bool quant = pv.kv_dtype == DMS_FP8_E4M3 || pv.kv_dtype == DMS_INT4;
  if (!(in_dtype == DMS_F32 || in_dtype == DMS_BF16) || (!quant && int(in_dtype) != pv.kv_dtype)) {
    set_last_error("in_dtype %d does not match kv_dtype %d", int(in_dtype), pv.kv_dtype);
    return DMS_ERR_INVALID_ARG;
  }
  const dms_dtype want = pv.kv_dtype == DMS_F32 ? DMS_F32 : DMS_BF16;
  if (q_dtype != want) {
    set_last_error("q_dtype must be %s for this pool", want == DMS_F32 ? "DMS_F32" : "DMS_BF16");
    return DMS_ERR_INVALID_ARG;
  }
  if (((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(q)) & 15) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255)) {
    set_last_error("k, v and q must be 16-byte aligned and workspace 256-byte aligned");
    return DMS_ERR_INVALID_ARG;
  }
  size_t need = 0;
  dms_status st = dms_decode_workspace_bytes(pool, n_layers, batch, &need);
  if (st != DMS_OK) return st;
  if (workspace_bytes < need) {
    set_last_error("workspace has %zu bytes, needs %zu", workspace_bytes, need);
    return DMS_ERR_CAPACITY;
  }
  bool done = false;
  if (pool->attn_kernel != DMS_ATTN_STREAM_K) {
    st = cluster_attn(pool, layer0, n_layers, batch, q, out, sm_scale, k, v, in_dtype, evict, pos,
                      pool->attn_kernel == DMS_ATTN_CLUSTER, stream, &done);
    if (st != DMS_OK || done) return st;
  }
  // many heads: the append kernel, then the stream-K attention kernel
  st = dms_append_evict_layers(pool, layer0, n_layers, batch, pos, k, v, in_dtype, evict, stream);
  if (st != DMS_OK) return st;
  return dms_decode_attn_layers(pool, layer0, n_layers, batch, q, q_dtype, out, sm_scale, workspace,
                                workspace_bytes, stream);
}
