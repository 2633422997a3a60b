// dms_decode_attn: split-K flash decoding over the compact DMS store.
//
// DMS only changes which keys a query sees: each kv-head keeps its own
// ragged set of tokens (delayed eviction, "NVIDIA veröffentlicht
// Qwen3-8B-DMS-8x ..." (mindverse), section "Dynamic Memory Sparsification
// (DMS): Eine innovative Lösung"), and decode is bound by reading that set
// from memory ("Nvidia DMS ..." (stiva.ai), opening section; FastDMS page:
// faster decode from less KV).  The kernel therefore streams every held row
// of every head once and nothing else.
//
// Work split (stream-K over blocks): the held rows of all heads of the call,
// in (layer, sequence, kv-head) order, form U blocks of up to 64 rows.  A
// persistent grid of G CTAs (one per SM) takes the contiguous ranges
// [c*U/G', (c+1)*U/G') with G' = min(G, U), so every CTA moves the same
// bytes whatever the head lengths.  A CTA's piece of a head ends in a partial softmax state
// (m, l, o); a head cut by CTA boundaries is merged by log-sum-exp in the
// CTA that finishes it last (an atomic ticket -- nobody waits).  Partial id
// c + i is unique per (CTA c, head i) piece.
//
// Inside a CTA: the last warp is the producer.  It issues one 1-D TMA bulk
// copy per full block (K tile and V tile are adjacent in the pool, 32 KB for
// bf16 D=128) into a ring of NS shared-memory stages paced by mbarriers
// (expect-tx on "full", one arrive on "empty").  The NCW consumer warps
// before it take the stages round-robin (NS a multiple of NCW, see
// AttnTraits).  Each keeps its own online-softmax state for the current head,
// reads the head's query rows itself (the fp32 path: from the stage, where
// the producer copies them with the block), and computes on tensor cores with the GQA
// group as the N=8 side of mma.sync m16n8k16 (tokens as M): S^T = K Q^T,
// then O^T += V^T P^T, P moved from accumulator to operand layout with
// movmatrix.  The stored rows' 16-byte chunks are XOR-swizzled by row, so
// ldmatrix reads them without bank conflicts.  FP8-E4M3 rows are decoded to
// f16 in registers (exact) from a layout that gives each lane its fragment
// bytes in two 16-byte loads; fp32 rows use CUDA-core FMA.
//
// Every wait is bounded (the pool's wait limit, 1 s unless set); a timeout
// sets DMS_DEVERR_TIMEOUT and the CTA
// drains its in-flight copies and returns.
#include <math.h>

#include "attn_warp.cuh"

namespace dms {

struct AttnParams {
  PoolView v;
  int l0, nl, batch;
  const uint8_t* q;   // [nl, batch, Hq, D] q dtype
  uint8_t* out;       // same layout and dtype
  float scale_log2;   // sm_scale * log2(e)
  float* ws_o;        // [(G + Htot) * g * D]
  float* ws_ml;       // [(G + Htot) * g * 2]
  const int32_t* seq_ids;  // pool sequence of batch row b (device), or null: row b
  int G;
  StepSync sync;           // stepper counters (null pointers otherwise)
};

// head index i of the call -> pool head id, or -1 for a sequence id out of range
__device__ __forceinline__ int pool_head(const AttnParams& p, int i) {
  const int h = i % p.v.Hkv;
  const int lb = i / p.v.Hkv;  // li * batch + b
  const int b = lb % p.batch;
  const int seq = p.seq_ids ? p.seq_ids[b] : b;
  if (seq < 0 || seq >= p.v.Bmax) return -1;
  return p.v.head(p.l0 + lb / p.batch, seq, h);
}

// held rows of call head i (a bad sequence id holds none and is reported)
__device__ __forceinline__ int n_of(const AttnParams& p, int i) {
  const int hd = pool_head(p, i);
  if (hd < 0) {
    report_error(p.v.hdr, DMS_DEVERR_BAD_SEQUENCE, p.l0 + (i / p.v.Hkv) / p.batch, (i / p.v.Hkv) % p.batch,
                 i % p.v.Hkv);
    return 0;
  }
  return p.v.n_slots[hd];
}

// Fewest blocks a CTA's range holds when there are fewer than 8 per SM
// (one layer of the Qwen3-8B shapes per call: 966 -> 760 us a decode step of
// 36 such calls; the all-layer launch is unaffected).
constexpr int kMinUnitsPerCta = 8;

// CTA whose unit range holds unit u (U units cut into G ranges).
__device__ __forceinline__ int cta_of(int64_t u, int64_t U, int G) {
  return int(((u + 1) * G - 1) / U);
}


// ---------------------------------------------------------------------------
template <int KV, int D>
__global__ void __launch_bounds__(AttnTraits<KV, D>::THREADS, 1)
    decode_attn_kernel(const AttnParams p) {
  using T = AttnTraits<KV, D>;
  using W = typename WarpSel<KV, D>::type;
  constexpr int kNCW = T::NCW;
  constexpr int kAttnThreads = T::THREADS;
  constexpr int kCons = 32 * kNCW;   // consumer threads
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* stages = smem;
  float* s_ow = reinterpret_cast<float*>(smem + size_t(T::NS) * T::STAGEB);
  float* s_mw = s_ow + kNCW * 8 * D;
  float* s_lw = s_mw + kNCW * 8;
  uint64_t* full = reinterpret_cast<uint64_t*>(s_lw + kNCW * 8);
  uint64_t* empty = full + T::NS;
  int* s_misc = reinterpret_cast<int*>(empty + T::NS);
  volatile int* s_abort = s_misc;        // [0]
  int* s_scan = s_misc + 16;             // [kAttnThreads / 32]

  const PoolView& v = p.v;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = v.Hq / v.Hkv;
  const int Htot = p.nl * p.batch * v.Hkv;
  const int c = blockIdx.x, G = p.G;

  if (tid == 0) {
    for (int s = 0; s < T::NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    s_misc[0] = 0;
    fence_mbar_init();
  }
  if constexpr (T::QB > 0) {
    // fp32 path: query rows g..7 of every stage stay zero (padding)
    for (int s = 0; s < T::NS; ++s) {
      uint4* qa = reinterpret_cast<uint4*>(stages + size_t(s) * T::STAGEB + 2 * T::TILEB);
      for (int i = tid; i < T::QB / 16; i += kAttnThreads) qa[i] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();  // order these generic writes before later TMA writes
  }

  // everything above only touched shared memory; the pool state and the
  // queries may come from the kernel before this one (append/evict)
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  // stepper: the output buffer's previous copy-out must be done (thread 0;
  // the scan's barrier below holds the other threads)
  if (p.sync.drained && tid == 0 && !wait_counter_geq(p.sync.drained, p.sync.drained_value, v.wait_ns))
    report_error(v.hdr, DMS_DEVERR_TIMEOUT, p.l0, -1, c);
  // stepper: the last CTA to leave publishes the step as computed
  auto sync_exit = [&]() {
    if (p.sync.done && tid == 0) {
      __threadfence();
      if (atomicAdd(p.sync.exit_count, 1) == int(gridDim.x) - 1) {
        *p.sync.exit_count = 0;
        __threadfence();
        st_release_gpu(p.sync.done, p.sync.done_value);
      }
    }
  };

  // ---- find this CTA's unit range: per-thread head ranges + block scan ----
  const int per = (Htot + kAttnThreads - 1) / kAttnThreads;
  const int hb = min(Htot, tid * per), he = min(Htot, hb + per);
  // this thread's held counts, loaded once and together (kept in registers
  // when it has at most kCache heads; the walks below reuse them)
  constexpr int kCache = 4;
  const bool cached = per <= kCache;
  int ncache[kCache];
#pragma unroll
  for (int x = 0; x < kCache; ++x) ncache[x] = (cached && hb + x < he) ? n_of(p, hb + x) : 0;
  auto n_mine = [&](int i) {   // held count of head i in [hb, he)
    if (!cached) return n_of(p, i);
    int n = 0;
#pragma unroll
    for (int x = 0; x < kCache; ++x) n = i == hb + x ? ncache[x] : n;
    return n;
  };
  int su = 0;
  for (int i = hb; i < he; ++i) {
    const int n = n_mine(i);
    su += units_of(n);
    if (n == 0 && i % G == c) {  // no key at all: define the output as 0
      const int64_t orow = int64_t(i / v.Hkv) * v.Hq + int64_t(i % v.Hkv) * g;
      for (int e = 0; e < g * D; ++e) store_out<T::QESZ>(p.out, orow * D + e, 0.f);
    }
  }
  int incl = su;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) s_scan[warp] = incl;
  __syncthreads();
  int wbase = 0, U = 0;
  for (int k = 0; k < kAttnThreads / 32; ++k) {
    wbase += k < warp ? s_scan[k] : 0;
    U += s_scan[k];
  }
  const int excl = wbase + incl - su;
  // a CTA takes at least kMinUnitsPerCta blocks (with few blocks, e.g. one
  // layer per call, fewer CTAs and fewer cross-CTA merges are faster), so
  // that every CTA in [0, Geff) has a non-empty range
  const int Geff = min(G, (U + kMinUnitsPerCta - 1) / kMinUnitsPerCta);
  if (c >= Geff) {
    sync_exit();
    return;
  }
  const int u_beg = int((int64_t(c) * U) / Geff), u_end = int((int64_t(c + 1) * U) / Geff);
  if (u_beg < u_end && u_beg >= excl && u_beg < excl + su) {
    int pre = excl;
    for (int i = hb; i < he; ++i) {
      const int nu = units_of(n_mine(i));
      if (u_beg < pre + nu) {
        s_misc[1] = i;
        s_misc[2] = pre;
        break;
      }
      pre += nu;
    }
  }
  // the head holding the range's last unit, and where it starts
  if (u_beg < u_end && u_end - 1 >= excl && u_end - 1 < excl + su) {
    int pre = excl;
    for (int i = hb; i < he; ++i) {
      const int n = n_mine(i);
      const int nu = units_of(n);
      if (u_end - 1 < pre + nu) {
        s_misc[4] = i;
        s_misc[5] = pre;
        s_misc[6] = n;
        break;
      }
      pre += nu;
    }
  }
  __syncthreads();
  const int i0 = s_misc[1], p0 = s_misc[2];
  // Processing order: first this CTA's piece of its last head (segment A,
  // units [r, u_end)), then [u_beg, r) (segment B).  The range's two end
  // heads are usually shared with the neighbouring CTAs and need the
  // cross-CTA merge; this way both finish early and their merges overlap the
  // copies already in flight, and the CTA ends on a head of its own.
  const int iL = s_misc[4], pL = s_misc[5], nL = s_misc[6];
  const int r = max(u_beg, pL);
  const int nA = u_end - r;
  // producer: the block ids of segment A's first 32 units (below), loaded
  // now so that their round trip overlaps the window fill and its barrier
  int blkA = 0;
  if (warp == kNCW && r + lane < u_end) {
    const int bi = r + lane - pL;
    if (DMS_CHECK(iL < Htot && bi >= 0 && bi < v.mbh, v.hdr, 304, iL, bi))
      blkA = v.bt[int64_t(pool_head(p, iL)) * v.mbh + bi];
  }
  // held counts of heads i0 .. i0 + HEAD_WIN - 1 in shared memory, so that the
  // walks below need no dependent global loads (the scan just loaded them)
  int* s_nwin = s_misc + T::MISC_INTS;
  for (int i = max(hb, i0); i < min(he, i0 + T::HEAD_WIN); ++i) s_nwin[i - i0] = n_mine(i);
  __syncthreads();
  auto n_at = [&](int i) { return i - i0 < T::HEAD_WIN ? s_nwin[i - i0] : n_of(p, i); };
  const int qrow_bytes = g * D * T::QESZ;

  if (warp == kNCW) {
    // ======================= producer =======================
    const uint64_t pol = policy_evict_first();   // K/V rows: read once per step
    const uint64_t qpol = policy_evict_last();   // query rows: re-read per block
    int k = 0, issued = 0;
    bool aborted = false;
    // lane 0 issues unit k (block jblk, jrows rows, of head ji) into stage k % NS
    auto issue = [&](int jblk, int jrows, int ji) {
      if (lane == 0 && !aborted) {
        const int s = k % T::NS;
        const uint32_t ph = (k / T::NS) & 1;
        if (!DMS_CHECK(jblk >= 0 && jblk < v.max_blocks && jrows >= 1 && jrows <= kBlockTokens &&
                           ji >= 0 && ji < Htot, v.hdr, 302, jblk, jrows)) {
          aborted = true;
          *s_abort = 1;
        } else if (!mbar_wait_bounded(&empty[s], ph ^ 1, s_abort, v.wait_ns) || *s_abort) {
          aborted = true;
          if (!*s_abort) report_error(v.hdr, DMS_DEVERR_TIMEOUT, p.l0, -1, c);
          *s_abort = 1;
        } else {
          uint8_t* st = stages + size_t(s) * T::STAGEB;
          const uint8_t* src = v.blocks + int64_t(jblk) * v.block_bytes;
          const uint8_t* qsrc = p.q + int64_t(ji / v.Hkv) * v.Hq * D * T::QESZ +
                                int64_t(ji % v.Hkv) * qrow_bytes;
          const uint32_t kbytes = uint32_t(jrows) * T::ROWB;
          // 4-bit tiles keep their scales after the nibbles: always copied whole
          const bool whole = jrows == kBlockTokens || KV == KV_INT4;
          const uint32_t vbytes = (whole || KV == KV_FP8) ? T::TILEB : kbytes;
          mbar_arrive_expect_tx(&full[s], (whole ? T::TILEB : kbytes) + vbytes +
                                              (T::QB > 0 ? qrow_bytes : 0));
          if (whole) {
            bulk_g2s(st, src, 2 * T::TILEB, &full[s], pol);
          } else {
            bulk_g2s(st, src, kbytes, &full[s], pol);
            bulk_g2s(st + T::TILEB, src + T::TILEB, vbytes, &full[s], pol);
          }
          if constexpr (T::QB > 0) bulk_g2s(st + 2 * T::TILEB, qsrc, qrow_bytes, &full[s], qpol);
          issued = k + 1;
        }
      }
      ++k;
    };
    // segment A: one head, units [r, u_end)
    for (int ub = r; ub < u_end; ub += 32) {
      const int u = ub + lane;
      int blk = ub == r ? blkA : 0, rows = 0;
      if (u < u_end) {
        const int bi = u - pL;
        if (ub != r && DMS_CHECK(iL < Htot && bi >= 0 && bi < v.mbh, v.hdr, 304, iL, bi))
          blk = v.bt[int64_t(pool_head(p, iL)) * v.mbh + bi];
        rows = min(kBlockTokens, nL - bi * kBlockTokens);
      }
      const int cnt = min(32, u_end - ub);
      for (int j = 0; j < cnt; ++j) {
        const int jblk = __shfl_sync(0xffffffffu, blk, j);
        const int jrows = __shfl_sync(0xffffffffu, rows, j);
        issue(jblk, jrows, iL);
      }
      aborted = __shfl_sync(0xffffffffu, aborted, 0);
    }
    // segment B: units [u_beg, r), walking the heads from i0
    int i = i0, pp = p0, n = n_at(i0), nu = units_of(n);
    for (int ub = u_beg; ub < r; ub += 32) {
      const int u = ub + lane;
      int mi = i, mp = pp, mn = n, mnu = nu;
      int blk = 0, rows = 0;
      if (u < r) {
        while (u >= mp + mnu) {
          mp += mnu;
          ++mi;
          mn = n_at(mi);
          mnu = units_of(mn);
        }
        const int bi = u - mp;
        if (DMS_CHECK(mi < Htot && bi < v.mbh, v.hdr, 301, mi, bi))
          blk = v.bt[int64_t(pool_head(p, mi)) * v.mbh + bi];
        rows = min(kBlockTokens, mn - bi * kBlockTokens);
      }
      const int cnt = min(32, r - ub);
      for (int j = 0; j < cnt; ++j) {
        const int jblk = __shfl_sync(0xffffffffu, blk, j);
        const int jrows = __shfl_sync(0xffffffffu, rows, j);
        const int ji = __shfl_sync(0xffffffffu, mi, j);
        issue(jblk, jrows, ji);
      }
      const int last = cnt - 1;
      i = __shfl_sync(0xffffffffu, mi, last);
      pp = __shfl_sync(0xffffffffu, mp, last);
      n = __shfl_sync(0xffffffffu, mn, last);
      nu = __shfl_sync(0xffffffffu, mnu, last);
      aborted = __shfl_sync(0xffffffffu, aborted, 0);
    }
    // drain: the CTA may not leave while a copy into its shared memory is in flight
    if (lane == 0) {
      volatile int never = 0;
      for (int kk = max(0, issued - T::NS); kk < issued; ++kk)
        mbar_wait_bounded(&full[kk % T::NS], (kk / T::NS) & 1, &never, v.wait_ns);
    }
    return;
  }

  // ========================= consumers =========================
  W st;
  st.reset();
  if constexpr (KV == KV_F32) st.g = g;
  float* my_ow = s_ow + warp * 8 * D;
  float* my_mw = s_mw + warp * 8;
  float* my_lw = s_lw + warp * 8;
  int i = i0, pp = p0, n = n_at(i0), nu = units_of(n);
  bool have_q = false;
  auto set_head_scales = [&](int head_i) {
    st.scale = p.scale_log2;
    st.vscale = 1.f;
    if constexpr (KV == KV_FP8) {
      const int hkv = head_i % v.Hkv;
      const int lyr = p.l0 + (head_i / v.Hkv) / p.batch;
      st.scale = p.scale_log2 * v.scales[(int64_t(lyr) * v.Hkv + hkv) * 2 + 0];
      st.vscale = v.scales[(int64_t(lyr) * v.Hkv + hkv) * 2 + 1];
    }
  };
  set_head_scales(i);
  // Each warp takes every kNCW-th unit of the CTA's range (unit k of the
  // range lives in stage k % NS).  A head is finished (the warps' states
  // combined) once no warp has a unit of it left: every warp passes every
  // head end of the range, in order, so the consumer barriers match.
  auto finish_head = [&]() {
    st.write_state(my_ow, my_mw, my_lw, g, lane);
    consumer_bar<kNCW>();
    const int hd = pool_head(p, i);
    const int cf = cta_of(pp, U, Geff), cl = cta_of(int64_t(pp) + nu - 1, U, Geff);
    const bool whole = cf == cl;
    const int64_t orow = int64_t(i / v.Hkv) * v.Hq + int64_t(i % v.Hkv) * g;
    const int pid = c + i;
    (void)DMS_CHECK(i < Htot && pid < G + Htot && cf >= 0 && cl < Geff, v.hdr, 303, i, pid);
    for (int idx = tid; idx < g * D; idx += kCons) {
      const int nn = idx / D, d = idx % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kNCW; ++w) M = fmaxf(M, s_mw[w * 8 + nn]);
      float o = 0.f, L = 0.f;
#pragma unroll
      for (int w = 0; w < kNCW; ++w) {
        const float f = fast_exp2(s_mw[w * 8 + nn] - M);
        o += f * s_ow[(w * 8 + nn) * D + d];
        L += f * s_lw[w * 8 + nn];
      }
      if (whole) {
        store_out<T::QESZ>(p.out, orow * D + idx, o / L);
      } else {
        p.ws_o[(int64_t(pid) * g + nn) * D + d] = o;
        if (d == 0) {
          p.ws_ml[(int64_t(pid) * g + nn) * 2 + 0] = M;
          p.ws_ml[(int64_t(pid) * g + nn) * 2 + 1] = L;
        }
      }
    }
    if (!whole) {
      consumer_bar<kNCW>();
      if (tid == 0) {
        __threadfence();
        const int prev = atomicAdd(&v.tickets[hd], 1);
        s_misc[3] = prev == cl - cf;
      }
      consumer_bar<kNCW>();
      if (s_misc[3]) {
        __threadfence();
        for (int idx = tid; idx < g * D; idx += kCons) {
          const int nn = idx / D, d = idx % D;
          float M = -INFINITY;
          for (int cc = cf; cc <= cl; ++cc)
            M = fmaxf(M, __ldcg(&p.ws_ml[(int64_t(cc + i) * g + nn) * 2]));
          float o = 0.f, L = 0.f;
          for (int cc = cf; cc <= cl; ++cc) {
            const int64_t id = int64_t(cc + i) * g + nn;
            const float f = fast_exp2(__ldcg(&p.ws_ml[id * 2]) - M);
            o += f * __ldcg(&p.ws_o[id * D + d]);
            L += f * __ldcg(&p.ws_ml[id * 2 + 1]);
          }
          store_out<T::QESZ>(p.out, orow * D + idx, o / L);
        }
        if (tid == 0) v.tickets[hd] = 0;
      }
    }
    consumer_bar<kNCW>();
    st.reset();
    have_q = false;
  };
  // unit k of the processing order (rows rows of head i) -> this warp
  auto process_unit = [&](int k, int rows) {
    const int s = k % T::NS;
    const uint32_t ph = (k / T::NS) & 1;
    if constexpr (KV != KV_F32) {
      if (!have_q) {  // first block of this head for this warp: issue before the wait
        st.load_q(p.q + int64_t(i / v.Hkv) * v.Hq * D * T::QESZ + int64_t(i % v.Hkv) * qrow_bytes,
                  g, lane);
        have_q = true;
      }
    }
    bool ok = false;
    if (!*s_abort) {
      ok = mbar_wait_bounded(&full[s], ph, s_abort, v.wait_ns);
      if (!ok && lane == 0) {
        *s_abort = 1;
        report_error(v.hdr, DMS_DEVERR_TIMEOUT, p.l0, -1, c);
      }
    }
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      const uint8_t* stage = stages + size_t(s) * T::STAGEB;
      st.unit(stage, rows, lane);
    }
    // release the stage only after its copy was seen complete; after an
    // abort the producer issues nothing more and drains what it issued
    __syncwarp();
    if (ok && lane == 0) mbar_arrive(&empty[s]);
  };
  int k = warp;
  if (nA > 0) {               // segment A: the piece of head iL
    i = iL;
    pp = pL;
    n = nL;
    nu = units_of(nL);
    set_head_scales(i);
    for (; k < nA; k += kNCW) process_unit(k, min(kBlockTokens, n - (r + k - pp) * kBlockTokens));
    finish_head();
  }
  if (r > u_beg) {            // segment B: [u_beg, r), ending on the head boundary r
    i = i0;
    pp = p0;
    n = n_at(i0);
    nu = units_of(n);
    set_head_scales(i);
    bool done = false;
    for (; !done; k += kNCW) {
      const int u = u_beg + (k - nA);
      const int lim = u < r ? u : r;
      while (pp + nu <= lim) {  // head i has no unit at or after u
        finish_head();
        if (pp + nu >= r) {
          done = true;
          break;
        }
        do {                    // next head with a unit (empty heads have none)
          pp += nu;
          ++i;
          n = n_at(i);
          nu = units_of(n);
        } while (nu == 0 && i + 1 < Htot);
        set_head_scales(i);
      }
      if (done) break;
      if (u >= r) {
        finish_head();
        break;
      }
      process_unit(k, min(kBlockTokens, n - (u - pp) * kBlockTokens));
    }
  }
  sync_exit();  // after the last head's combine (its barriers ordered every consumer's writes)
}

template <int KV, int D>
static dms_status launch_attn(const AttnParams& prm, cudaStream_t stream) {
  using T = AttnTraits<KV, D>;
  static FuncAttrCache smem_attr;  // per instantiation, per device
  dms_status st = ensure_func_attr(reinterpret_cast<const void*>(decode_attn_kernel<KV, D>),
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, int(T::SMEM),
                                   smem_attr, "attn smem attribute");
  if (st != DMS_OK) return st;
  return cuda_status(launch_pdl(decode_attn_kernel<KV, D>, dim3(prm.G), dim3(T::THREADS), T::SMEM,
                                stream, prm),
                     "decode_attn_kernel");
}

}  // namespace dms

using namespace dms;

static size_t attn_workspace_bytes(const dms_pool* pool, int n_layers, int batch) {
  const PoolView& v = pool->view;
  const int g = v.Hq / v.Hkv;
  const size_t parts = size_t(pool->sm_count) + size_t(n_layers) * batch * v.Hkv;
  const size_t o_bytes = (parts * g * v.D * 4 + 255) & ~size_t(255);
  return o_bytes + parts * g * 2 * 4;
}

// Fill the kernel parameters and launch (arguments already checked).
static dms_status run_attn(dms_pool* pool, int layer0, int n_layers, int batch, const void* q,
                           void* out, float sm_scale, void* ws, const int32_t* seq_ids,
                           cudaStream_t stream, const StepSync& sync = StepSync{}) {
  const PoolView& v = pool->view;
  const int g = v.Hq / v.Hkv;
  const size_t parts = size_t(pool->sm_count) + size_t(n_layers) * batch * v.Hkv;
  AttnParams prm;
  prm.v = v;
  prm.l0 = layer0;
  prm.nl = n_layers;
  prm.batch = batch;
  prm.q = static_cast<const uint8_t*>(q);
  prm.out = static_cast<uint8_t*>(out);
  const float sc = sm_scale > 0.f ? sm_scale : 1.0f / sqrtf(float(v.D));
  prm.scale_log2 = sc * 1.4426950408889634f;
  prm.ws_o = static_cast<float*>(ws);
  prm.ws_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                       ((parts * g * v.D * 4 + 255) & ~size_t(255)));
  prm.seq_ids = seq_ids;
  prm.G = pool->sm_count;
  prm.sync = sync;
  if (!seq_ids && !sync.ready && !sync.drained && !sync.done && pool->attn_kernel != DMS_ATTN_STREAM_K) {
    // few heads: one cluster per head (csrc/step.cu)
    bool done = false;
    dms_status st = cluster_attn(pool, layer0, n_layers, batch, q, out, sm_scale, nullptr, nullptr,
                                 DMS_BF16, nullptr, 0, pool->attn_kernel == DMS_ATTN_CLUSTER, stream,
                                 &done);
    if (st != DMS_OK || done) return st;
  }
  if (v.kv_dtype == DMS_BF16) {
    return v.D == 128 ? launch_attn<KV_BF16, 128>(prm, stream) : launch_attn<KV_BF16, 64>(prm, stream);
  }
  if (v.kv_dtype == DMS_FP8_E4M3) return launch_attn<KV_FP8, 128>(prm, stream);
  if (v.kv_dtype == DMS_INT4) return launch_attn<KV_INT4, 128>(prm, stream);
  return v.D == 128 ? launch_attn<KV_F32, 128>(prm, stream) : launch_attn<KV_F32, 64>(prm, stream);
}

// The stepper's attention launch: arguments as for dms_decode_attn_layers
// (checked by the caller), plus the step counters.
dms_status dms::decode_attn_layers_synced(dms_pool* pool, int layer0, int n_layers, int batch,
                                          const void* q, void* out, float sm_scale, void* ws,
                                          cudaStream_t stream, const StepSync& sync) {
  return run_attn(pool, layer0, n_layers, batch, q, out, sm_scale, ws, nullptr, stream, sync);
}

extern "C" dms_status dms_decode_workspace_bytes(const dms_pool* pool, int n_layers, int batch,
                                                 size_t* bytes) {
  if (!pool || !bytes || n_layers < 1 || batch < 1) {
    set_last_error("bad arguments");
    return DMS_ERR_INVALID_ARG;
  }
  *bytes = attn_workspace_bytes(pool, n_layers, batch);
  return DMS_OK;
}

static dms_status decode_attn_checked(dms_pool* pool, int layer0, int n_layers, int batch,
                                      const void* q, dms_dtype q_dtype, void* out, float sm_scale,
                                      void* workspace, size_t workspace_bytes,
                                      const int32_t* seq_ids, cudaStream_t stream) {
  if (!pool) {
    set_last_error("null pool");
    return DMS_ERR_INVALID_ARG;
  }
  const PoolView& v = pool->view;
  if (layer0 < 0 || n_layers < 1 || layer0 + n_layers > v.L || batch < 1 || batch > v.Bmax) {
    set_last_error("bad layer range / batch (%d+%d, %d)", layer0, n_layers, batch);
    return DMS_ERR_INVALID_ARG;
  }
  if (!q || !out || !workspace) {
    set_last_error("null q / out / workspace");
    return DMS_ERR_INVALID_ARG;
  }
  const dms_dtype want = v.kv_dtype == DMS_F32 ? DMS_F32 : DMS_BF16;
  if (q_dtype != want) {
    set_last_error("q_dtype must be %s for this pool", want == DMS_F32 ? "DMS_F32" : "DMS_BF16");
    return DMS_ERR_INVALID_ARG;
  }
  if ((reinterpret_cast<uintptr_t>(q) & 15) || (reinterpret_cast<uintptr_t>(workspace) & 255)) {
    set_last_error("q must be 16-byte aligned and workspace 256-byte aligned");
    return DMS_ERR_INVALID_ARG;
  }
  const size_t need = attn_workspace_bytes(pool, n_layers, batch);
  if (workspace_bytes < need) {
    set_last_error("workspace has %zu bytes, needs %zu", workspace_bytes, need);
    return DMS_ERR_CAPACITY;
  }
  return run_attn(pool, layer0, n_layers, batch, q, out, sm_scale, workspace, seq_ids, stream);
}

extern "C" dms_status dms_decode_attn_layers(dms_pool* pool, int layer0, int n_layers, int batch,
                                             const void* q, dms_dtype q_dtype, void* out,
                                             float sm_scale, void* workspace,
                                             size_t workspace_bytes, cudaStream_t stream) {
  return decode_attn_checked(pool, layer0, n_layers, batch, q, q_dtype, out, sm_scale, workspace,
                             workspace_bytes, nullptr, stream);
}

extern "C" dms_status dms_decode_attn_seqs(dms_pool* pool, int layer0, int n_layers, int n_seqs,
                                           const int32_t* seq_ids, const void* q, dms_dtype q_dtype,
                                           void* out, float sm_scale, void* workspace,
                                           size_t workspace_bytes, cudaStream_t stream) {
  if (!seq_ids || (reinterpret_cast<uintptr_t>(seq_ids) & 3)) {
    set_last_error("seq_ids must be a non-null, 4-byte aligned device array");
    return DMS_ERR_INVALID_ARG;
  }
  return decode_attn_checked(pool, layer0, n_layers, n_seqs, q, q_dtype, out, sm_scale, workspace,
                             workspace_bytes, seq_ids, stream);
}

extern "C" dms_status dms_decode_attn(dms_pool* pool, int layer, int batch, const void* q,
                                      dms_dtype q_dtype, void* out, float sm_scale,
                                      void* workspace, size_t workspace_bytes,
                                      cudaStream_t stream) {
  return dms_decode_attn_layers(pool, layer, 1, batch, q, q_dtype, out, sm_scale, workspace,
                                workspace_bytes, stream);
}

// ---------------------------------------------------------------------------
// Decode attention for callers that cannot allocate device memory.
//
// Some callers have no way to obtain a workspace: a serving engine that has
// already handed every free byte of HBM to its KV pool, a plugin whose host
// framework exposes no device allocator, or a latency-critical path where
// cudaMalloc's device-wide synchronisation would stall other streams.  This
// entry point gives them the split-K scratch from a fixed array compiled into
// the library instead of a caller buffer.
//
// The array is kStaticWorkspaceBytes (16 MiB) of global memory on every GPU
// that loads the library, held until the process exits.  Host code cannot
// hand the array's name to a kernel (in host code it names a host-side
// stand-in, not device memory), so the first call on each device looks up
// its device address with cudaGetSymbolAddress while that device is current
// and caches it with the context it belongs to; make that first call (and
// the first after a device reset) before any stream capture.  Every call
// on a device shares the one array, which keeps the previous call's partial
// results: nothing in it has to start at zero (each launch writes every
// partial it later reads, and the merge tickets live in the pool), but calls
// whose kernels overlap on the GPU race on it and must be ordered.
// ---------------------------------------------------------------------------
#include <cuda.h>
#include <mutex>

namespace dms {

constexpr size_t kStaticWorkspaceBytes = size_t(16) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

// The address is looked up once per device and context: a device reset
// (cudaDeviceReset, or a caller that makes another driver context current)
// gives the array a new address in the new context, so the cache remembers
// which context its address belongs to and looks it up again when the
// current context differs.
struct StaticWsEntry {
  CUcontext ctx;
  void* addr;
};
static std::mutex g_static_ws_mutex;
static StaticWsEntry g_static_ws[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
static CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = []() -> CtxGetCurrentFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  return fn;
}

// Device address of g_static_workspace on the current device (set-up on
// the first call in a device's context; cudaGetSymbolAddress runs there).
static dms_status static_workspace_address(int device, void** addr) {
  if (device < 0 || device >= kMaxDevices) {
    set_last_error("device %d out of range for the fixed workspace table", device);
    return DMS_ERR_UNSUPPORTED;
  }
  CUcontext ctx = nullptr;
  CtxGetCurrentFn get = ctx_get_current_fn();
  if (!get || get(&ctx) != CUDA_SUCCESS) {
    set_last_error("cuCtxGetCurrent is not available");
    return DMS_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_static_ws_mutex);
  StaticWsEntry& e = g_static_ws[device];
  if (!e.addr || e.ctx != ctx) {
    void* p = nullptr;
    dms_status st = cuda_status(cudaGetSymbolAddress(&p, g_static_workspace),
                                "cudaGetSymbolAddress(g_static_workspace)");
    if (st != DMS_OK) return st;
    e.ctx = ctx;
    e.addr = p;
  }
  *addr = e.addr;
  return DMS_OK;
}

}  // namespace dms

extern "C" dms_status dms_decode_attn_layers_noalloc(dms_pool* pool, int layer0, int n_layers,
                                                     int batch, const void* q, dms_dtype q_dtype,
                                                     void* out, float sm_scale,
                                                     cudaStream_t stream) {
  if (!pool) {
    set_last_error("null pool");
    return DMS_ERR_INVALID_ARG;
  }
  const PoolView& v = pool->view;
  if (layer0 < 0 || n_layers < 1 || layer0 + n_layers > v.L || batch < 1 || batch > v.Bmax) {
    set_last_error("bad layer range / batch (%d+%d, %d)", layer0, n_layers, batch);
    return DMS_ERR_INVALID_ARG;
  }
  if (!q || !out) {
    set_last_error("null q / out");
    return DMS_ERR_INVALID_ARG;
  }
  const dms_dtype want = v.kv_dtype == DMS_F32 ? DMS_F32 : DMS_BF16;
  if (q_dtype != want) {
    set_last_error("q_dtype must be %s for this pool", want == DMS_F32 ? "DMS_F32" : "DMS_BF16");
    return DMS_ERR_INVALID_ARG;
  }
  if (reinterpret_cast<uintptr_t>(q) & 15) {
    set_last_error("q must be 16-byte aligned");
    return DMS_ERR_INVALID_ARG;
  }
  const size_t need = attn_workspace_bytes(pool, n_layers, batch);
  if (need > kStaticWorkspaceBytes) {
    set_last_error("this call needs %zu bytes of scratch; the fixed workspace holds %zu "
                   "(use dms_decode_attn_layers with a caller workspace, or fewer layers)",
                   need, kStaticWorkspaceBytes);
    return DMS_ERR_CAPACITY;
  }
  int dev = -1;
  dms_status st = cuda_status(cudaGetDevice(&dev), "cudaGetDevice");
  if (st != DMS_OK) return st;
  if (dev != pool->device) {
    set_last_error("current device %d is not the pool's device %d", dev, pool->device);
    return DMS_ERR_INVALID_ARG;
  }
  void* ws = nullptr;
  st = static_workspace_address(dev, &ws);
  if (st != DMS_OK) return st;
  return run_attn(pool, layer0, n_layers, batch, q, out, sm_scale, ws, nullptr, stream);
}

