// dms_prefill_attn: prompt attention under the DMS delayed-eviction mask,
// fused with the compaction of the prompt into the compact store.
//
// The delayed-eviction rule holds for every query, prompt queries included:
// query i sees key j <= i unless j is flagged and i - j >= w ("NVIDIA
// veröffentlicht Qwen3-8B-DMS-8x ..." (mindverse), section "Dynamic Memory
// Sparsification (DMS): Eine innovative Lösung"; "Nvidia DMS ..."
// (stiva.ai), section "Ключевое изобретение: delayed eviction").  The keys
// the last prompt query can see are exactly the rows the compact store keeps
// ("FastDMS: vLLM BF16/FP8보다 빠른 6.4x KV cache 압축" (molayo1419.me),
// opening paragraphs), so the kernel that streams the prompt's K/V tiles for
// attention also writes the kept rows into their slots.
//
// One CTA of 8 warps per (128-query tile, query head, sequence), two CTAs
// per SM (one CTA's softmax runs while the other's tensor cores work), heaviest
// (latest) query tiles first.  Per 128-key tile, on the 5th-generation
// tensor cores with accumulators in tensor memory:
//   S = Q K^T           (M = 128 queries, N = 128 keys, K = D)
//   threads r and r + 128 own query row r, 64 key columns each: masked
//   online softmax on S[r] (tcgen05.ld; the row maximum is combined through
//   shared memory), P[r] as bf16 into shared memory, O[r] rescaled in tensor
//   memory when the row maximum moved
//   O += P V            (M = 128 queries, N = D, K = 128 keys; V is read in
//                        its own [keys x D] layout as an MN-major operand)
// Tiles live in shared memory in the 128-byte-swizzled image of umma.cuh,
// filled by tensor-map (TMA) loads: the query tile once, then per key tile
// its keys into the one tile buffer and, once S has read them, its values
// into the same buffer while the softmax runs (about 100 KB a CTA, so that
// two fit on an SM).
//
// Which key tiles (bf16 store):
//   sparse (default)  the layer is compacted before this kernel.  A key
//       older than i0 - w + 1 is outside the window of every query of the
//       tile [i0, i0 + 128), so it is seen exactly when it carries no flag,
//       and the unflagged keys are what the store holds, in position order.
//       Keys before the band of tiles that holds i0 - w + 1 are therefore
//       read from the store as dense 128-key tiles (two 64-row blocks, masked
//       only past the last one), and only the band and the diagonal come
//       from the prompt with the full mask.  At a keep rate k and a prompt
//       of P >> w the tiles computed fall from about P^2 / 2 to about
//       k P^2 / 2 + P w.
//   dense  every causal tile from the prompt; the CTA of the first query
//       head of each kv-head group writes, at its diagonal key tile, the
//       tile's kept rows into the pool (slots from the prefix counts of the
//       plan kernel) and the window ring.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include "dms_internal.cuh"
#include "umma.cuh"

namespace dms {

constexpr int kPaTile = 128;      // queries per CTA and keys per tile
// threads per query row: each takes 128 / SPLIT key columns of S and D / SPLIT
// columns of O (32 at least, the width of one tensor-memory load).  Two beat
// one (the softmax issues from twice the warps) and four (more exchanges).
template <int D>
struct PaSplit {
  static constexpr int SPLIT = 2;
  static constexpr int THREADS = kPaTile * SPLIT;
};

template <int D>
struct PaSmem {
  static constexpr int TILE = kPaTile * D * 2;         // one [128 x D] bf16 tile
  static constexpr int Q = 0;                          // queries, K-major
  static constexpr int KV = Q + TILE;                  // keys (K-major), then values [keys x D] (MN-major B)
  static constexpr int P = KV + TILE;                  // [128 queries x 128 keys] bf16
  static constexpr int FLAGS = P + kPaTile * kPaTile * 2;  // 2 x 4 words of evict-flag bits
  static constexpr int BARS = FLAGS + 2 * kPaTile;     // mbarriers: S, O, Q, K, V
  static constexpr int MISC = BARS + 64;               // tmem base, scan
  static constexpr int RED = MISC + 128;               // [SPLIT parts][128 rows] floats
  static constexpr int BYTES = RED + PaSplit<D>::SPLIT * kPaTile * 4 + 1024;  // + alignment slack
};

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Paired fp32 arithmetic of sm_100 (one instruction for two lanes of
// values, each rounded as the scalar operation would be) and the
// three-input maximum.
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                      float c1) {
  uint64_t d;
  asm("{\n\t.reg .b64 ra, rb, rc;\n\tmov.b64 ra, {%1, %2};\n\tmov.b64 rb, {%3, %4};\n\t"
      "mov.b64 rc, {%5, %6};\n\tfma.rn.f32x2 %0, ra, rb, rc;\n\t}"
      : "=l"(d)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d0), "=f"(d1) : "l"(d));
}
__device__ __forceinline__ void fadd2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  uint64_t d;
  asm("{\n\t.reg .b64 ra, rb;\n\tmov.b64 ra, {%1, %2};\n\tmov.b64 rb, {%3, %4};\n\t"
      "add.rn.f32x2 %0, ra, rb;\n\t}"
      : "=l"(d)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d0), "=f"(d1) : "l"(d));
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Unflagged keys of head (b, hkv) before position bs (a multiple of 128 below
// P - w, so kept = unflagged there), from the kept-token prefix counts the
// layer's compaction left per 256-token chunk, plus the first 128 tokens of
// bs's chunk when bs is not a chunk start.  Every thread calls it (one block
// barrier); s_tmp holds 4 ints.
__device__ __forceinline__ int far_keys(const PoolView& v, const uint8_t* evict, int b, int hkv, int P, int bs,
                                        int tid, int* s_tmp) {
  const int c = bs >> 8;
  const int base = v.chunk_counts[(int64_t(b) * v.Hkv + hkv) * v.n_chunks_max + c];
  if (bs & 255) {
    if (tid < kPaTile) {
      const int j = (c << 8) + tid;
      const unsigned m = __ballot_sync(0xffffffffu, evict[(int64_t(b) * P + j) * v.Hkv + hkv] == 0);
      if ((tid & 31) == 0) s_tmp[tid >> 5] = __popc(m);
    }
    __syncthreads();
    return base + s_tmp[0] + s_tmp[1] + s_tmp[2] + s_tmp[3];
  }
  return base;
}

template <int D>
__global__ void __launch_bounds__(PaSplit<D>::THREADS, 2)
    prefill_attn_kernel(PoolView v, int layer, int seq0, int P, const __grid_constant__ CUtensorMap tq,
                        const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                        const __grid_constant__ CUtensorMap tpool, const uint8_t* evict,
                        __nv_bfloat16* out, float scale_log2, int n_qtiles, int compact, int sparse) {
  using S = PaSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // query row r of the tile, key-column part h (columns HC h .. HC h + HC - 1
  // of S, OC h .. of O); warps w, w + 4, ... share the tensor-memory lanes of
  // rows 32 (w & 3) .. + 31
  constexpr int SPLIT = PaSplit<D>::SPLIT, THREADS = PaSplit<D>::THREADS;
  constexpr int HC = kPaTile / SPLIT, OC = D / SPLIT;  // S and O columns per thread
  const int r = tid & (kPaTile - 1), h = tid >> 7;
  float* s_red = reinterpret_cast<float*>(smem + S::RED);
  const int qt = n_qtiles - 1 - int(blockIdx.x);  // heaviest query tiles first
  const int hq = blockIdx.y, b = blockIdx.z;
  const int g = v.Hq / v.Hkv, hkv = hq / g;
  const int i0 = qt * kPaTile;
  const int64_t q_stride = int64_t(v.Hq) * D, kv_stride = int64_t(v.Hkv) * D;
  (void)kv_stride;
  uint64_t* bar_s = reinterpret_cast<uint64_t*>(smem + S::BARS);
  uint64_t* bar_o = bar_s + 1;
  uint64_t* bar_q = bar_s + 2;
  uint64_t* bar_k = bar_s + 3;
  uint64_t* bar_v = bar_s + 4;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + S::MISC);
  int* s_scan = reinterpret_cast<int*>(smem + S::MISC) + 4;   // [8]
  int* s_cnt = reinterpret_cast<int*>(smem + S::MISC) + 12;   // [4] (far_keys)

  // tensor-map loads of one [128 x D] tile: boxes of 64 columns x 128 rows
  // with 128-byte swizzle (the operand image of umma.cuh); rows past the
  // prompt arrive as zeros.  One thread.
  auto load_tile = [&](uint8_t* dst, const CUtensorMap* map, int x0, int row0, uint64_t* bar) {
    mbar_arrive_expect_tx(bar, S::TILE);
#pragma unroll
    for (int kb = 0; kb < D / 64; ++kb)
      umma::tma_load_3d(dst + kb * kPaTile * 128, map, x0 + kb * 64, row0, b, bar);
  };
  // a far tile: the store's slots [128 k, 128 k + 128) of this head, two
  // 64-row blocks; each block's K (kv = 0) or V (kv = 1) rows are copied per
  // 64-column half into rows 0..63 / 64..127 of the tile.  The store's
  // 16-byte chunks are already XOR-swizzled by row (chunk c of row r at
  // c ^ (r & 7)), which is the operand image a 128-byte-swizzled box load
  // makes, so the copies use no swizzle of their own.
  auto load_far = [&](uint8_t* dst, int blk0, int blk1, int kv, uint64_t* bar) {
    mbar_arrive_expect_tx(bar, S::TILE);
#pragma unroll
    for (int kb = 0; kb < D / 64; ++kb) {
      umma::tma_load_4d(dst + kb * kPaTile * 128, &tpool, 0, kb, 0, 2 * blk0 + kv, bar);
      umma::tma_load_4d(dst + kb * kPaTile * 128 + 64 * 128, &tpool, 0, kb, 0, 2 * blk1 + kv, bar);
    }
  };
  // evict flag of key j0 + r of tile kt (loaded a tile ahead, packed later)
  auto flag_of = [&](int kt) -> uint8_t {
    const int j = kt * kPaTile + r;
    return (h == 0 && j < P) ? evict[(int64_t(b) * P + j) * v.Hkv + hkv] : 0;
  };
  uint32_t* s_fbits = reinterpret_cast<uint32_t*>(smem + S::FLAGS);  // [2][4]

  if (tid == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    mbar_init(bar_q, 1);
    mbar_init(bar_k, 1);
    mbar_init(bar_v, 1);
    fence_mbar_init();
  }
  __syncwarp();  // tcgen05.alloc is warp-collective: lane 0 rejoins first
  if (warp == 0) {
    umma::tmem_alloc(s_tmem, 256);
    umma::tmem_relinquish();
  }
  __syncthreads();  // barriers initialised before any thread waits on them
  if (tid == 0) load_tile(smem + S::Q, &tq, hq * D, i0, bar_q);

  // ---- the key tiles of this query tile ----
  // Every row i of the tile sees keys j < lo = i0 - w + 1 only when they carry
  // no evict flag (i - j >= w for all of them).  With `sparse`, keys before
  // the band [kt_lo * 128, i0 + 128) that holds lo are not read from the
  // prompt: the unflagged ones among them are the store's first n_far slots
  // (the store keeps them in position order), read as nf dense "far" tiles;
  // the band is read from the prompt with the full mask.  The store must
  // hold this head's prompt, which the counts check: its held count must
  // equal the kept count of the flags, and the far tiles' slots must exist;
  // otherwise every key tile comes from the prompt.
  int kt_lo = 0, nf = 0, n_far = 0;
  const int32_t* far_bt = v.bt + int64_t(v.head(layer, seq0 + b, hkv)) * v.mbh;
  if (sparse) {
    const int lo = i0 - v.w + 1;
    const int kl = lo > 0 ? lo / kPaTile : 0;
    if (kl > 0) {
      // a compaction that failed (this call's or an earlier one: the error
      // word is sticky) may have left a head's old rows in place
      if (tid == 0) s_scan[0] = *reinterpret_cast<volatile uint32_t*>(&v.hdr->error) != 0u;
      const int held = v.n_slots[v.head(layer, seq0 + b, hkv)];
      __syncthreads();
      const bool failed = s_scan[0] != 0;
      const int tf = far_keys(v, evict, b, hkv, P, kl * kPaTile, tid, s_cnt);
      const int nft = (tf + kPaTile - 1) / kPaTile;
      if (!failed && nft * kPaTile <= held && 2 * nft <= v.mbh) {
        kt_lo = kl;
        nf = nft;
        n_far = tf;
      }
    }
  }
  const int n_tiles = nf + (qt - kt_lo + 1);
  // block ids of far tile k (thread 0; the next tile's are loaded a tile ahead)
  int fb0 = 0, fb1 = 0, nb0 = 0, nb1 = 0;
  if (tid == 0) {
    if (nf > 0) {
      fb0 = far_bt[0];
      fb1 = far_bt[1];
      if (nf > 1) {
        nb0 = far_bt[2];
        nb1 = far_bt[3];
      }
      load_far(smem + S::KV, fb0, fb1, 0, bar_k);
    } else {
      load_tile(smem + S::KV, &tk, hkv * D, kt_lo * kPaTile, bar_k);
    }
  }
  auto flag_at = [&](int it) -> uint8_t { return it >= nf ? flag_of(kt_lo + it - nf) : 0; };
  uint8_t f_cur = flag_at(0);
  umma::fence_before_sync();
  __syncthreads();
  umma::fence_after_sync();
  const uint32_t tbase = *s_tmem;
  const uint32_t t_s = tbase, t_o = tbase + kPaTile;
  const uint32_t aQ = smem_u32(smem + S::Q), aP = smem_u32(smem + S::P);
  constexpr uint32_t idS = umma::idesc_bf16_f32(kPaTile, kPaTile);
  constexpr uint32_t idO = umma::idesc_bf16_f32_bmn(kPaTile, D);
  const int i = i0 + r;  // this thread's query row
  // running row maximum (log2 units); a large finite start instead of -inf
  // keeps exp2(s - m) free of a check (masked entries are -inf and give 0)
  float m = -1e30f, l = 0.f;
  volatile int never = 0;
  bool ok = true;

  for (int it = 0; it < n_tiles; ++it) {
    const bool far = it < nf;
    const int kt = far ? -1 : kt_lo + it - nf;
    const int cur = it & 1, j0 = kt * kPaTile;
    if (it > 0) {  // P V of tile it-1 is done: P and the tile buffer are free
      ok &= mbar_wait_bounded(bar_o, (it - 1) & 1, &never, v.wait_ns);
      __syncwarp();
      umma::fence_after_sync();
      if (tid == 0) {
        if (far) {
          fb0 = nb0;
          fb1 = nb1;
          if (it + 1 < nf) {  // ids of the next far tile, used one tile later
            nb0 = far_bt[2 * (it + 1)];
            nb1 = far_bt[2 * (it + 1) + 1];
          }
          load_far(smem + S::KV, fb0, fb1, 0, bar_k);
        } else {
          load_tile(smem + S::KV, &tk, hkv * D, j0, bar_k);
        }
      }
      __syncwarp();
    }
    {  // this tile's flags as 4 words of bits (bit c = key j0 + c flagged)
      const unsigned fw = __ballot_sync(0xffffffffu, f_cur != 0);
      if (lane == 0 && h == 0) s_fbits[cur * 4 + warp] = fw;
    }
    const uint8_t f_next = it + 1 < n_tiles ? flag_at(it + 1) : 0;
    if (it == 0) ok &= mbar_wait_bounded(bar_q, 0, &never, v.wait_ns);
    ok &= mbar_wait_bounded(bar_k, it & 1, &never, v.wait_ns);  // K of tile it landed
    __syncwarp();
    __syncthreads();
    const uint32_t aK = smem_u32(smem + S::KV), aV = aK;
    if (tid == 0) {
      umma::fence_after_sync();
#pragma unroll
      for (int k0 = 0; k0 < D; k0 += 16)
        umma::mma_bf16(t_s, umma::desc_k16(aQ, kPaTile, k0), umma::desc_k16(aK, kPaTile, k0), idS,
                       k0 > 0);
      umma::commit(bar_s);
    }
    ok &= mbar_wait_bounded(bar_s, it & 1, &never, v.wait_ns);
    __syncwarp();  // lanes leave the wait loop independently; tcgen05.ld is warp-collective
    umma::fence_after_sync();
    // S read the keys: the values of the same tile stream into the buffer
    // while the softmax runs
    if (tid == 0) {
      if (far) load_far(smem + S::KV, fb0, fb1, 1, bar_v);
      else load_tile(smem + S::KV, &tv, hkv * D, j0, bar_v);
    }
    __syncwarp();

    // ---- masked online softmax on query row i (log2 domain) ----
    // visibility of key j0 + c as bits: flag clear or inside the window
    // (c >= i - w + 1 - j0), causal (c <= i - j0), inside the prompt (c < P - j0)
    uint32_t vis[HC / 32];
    if (far) {  // every row sees the tile's first n_far - 128 it slots
      const int lim = n_far - it * kPaTile;
#pragma unroll
      for (int x = 0; x < HC / 32; ++x) {
        const int x_lt = lim - 32 * ((HC / 32) * h + x);
        vis[x] = x_lt <= 0 ? 0u : x_lt >= 32 ? ~0u : (1u << x_lt) - 1u;
      }
    } else {
      const int hi = i - j0, lo = i - v.w + 1 - j0, end = P - j0;
#pragma unroll
      for (int x = 0; x < HC / 32; ++x) {
        const int wd = (HC / 32) * h + x, c0 = 32 * wd;
        const int x_le = hi - c0, x_ge = lo - c0, x_lt = end - c0;
        const uint32_t le = x_le < 0 ? 0u : x_le >= 31 ? ~0u : (2u << x_le) - 1u;
        const uint32_t ge = x_ge <= 0 ? ~0u : x_ge >= 32 ? 0u : ~((1u << x_ge) - 1u);
        const uint32_t lt = x_lt <= 0 ? 0u : x_lt >= 32 ? ~0u : (1u << x_lt) - 1u;
        vis[x] = (~s_fbits[cur * 4 + wd] | ge) & le & lt;
      }
    }
    float s[HC];
#pragma unroll
    for (int cb = 0; cb < HC / 32; ++cb) {
      float x[32];
      umma::ld32(umma::taddr_of(t_s, warp, h * HC + cb * 32), x);
#pragma unroll
      for (int e = 0; e < 32; ++e) s[cb * 32 + e] = x[e];
    }
    umma::wait_ld();
    float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int c = 0; c < HC; ++c) {  // unscaled scores; the scale enters the exponent below
      s[c] = ((vis[c >> 5] >> (c & 31)) & 1u) ? s[c] : -INFINITY;
      mx4[c & 3] = fmaxf(mx4[c & 3], s[c]);
    }
    // the row maximum over the row's SPLIT threads (r, r + 128, ...)
    s_red[h * kPaTile + r] = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * scale_log2;
    __syncthreads();
    float mx = s_red[r];
#pragma unroll
    for (int x = 1; x < SPLIT; ++x) mx = fmaxf(mx, s_red[x * kPaTile + r]);
    // lazy rescaling: the running maximum only moves when the row maximum
    // grew by more than 8 (log2 units), so P stays <= 256 and O rarely needs
    // a round trip through tensor memory
    float alpha = 1.f;
    if (mx > m + 8.f) {
      alpha = fast_exp2(m - mx);
      m = mx;
    }
    float sum4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < HC; ++c) {
      const float p = fast_exp2(fmaf(s[c], scale_log2, -m));
      sum4[c & 3] += p;
      s[c] = p;
    }
    l = l * alpha + ((sum4[0] + sum4[1]) + (sum4[2] + sum4[3]));
#pragma unroll
    for (int ch = 0; ch < HC / 8; ++ch) {
      uint4 w4;
      w4.x = pack2_bf16(s[ch * 8 + 0], s[ch * 8 + 1]);
      w4.y = pack2_bf16(s[ch * 8 + 2], s[ch * 8 + 3]);
      w4.z = pack2_bf16(s[ch * 8 + 4], s[ch * 8 + 5]);
      w4.w = pack2_bf16(s[ch * 8 + 6], s[ch * 8 + 7]);
      *reinterpret_cast<uint4*>(smem + S::P + umma::sw128_offset(kPaTile, r, h * HC + ch * 8)) = w4;
    }
    // O row *= alpha when this warp has a row whose maximum moved
    if (it > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
      for (int cb = 0; cb < OC / 32; ++cb) {
        float o[32];
        umma::ld32(umma::taddr_of(t_o, warp, h * OC + cb * 32), o);
        umma::wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] *= alpha;
        umma::st32(umma::taddr_of(t_o, warp, h * OC + cb * 32), o);
      }
      umma::wait_st();
    }
    f_cur = f_next;
    fence_proxy_async_smem();  // P before the tensor cores read it
    umma::fence_before_sync();
    __syncthreads();
    if (tid == 0) {
      umma::fence_after_sync();
      ok &= mbar_wait_bounded(bar_v, it & 1, &never, v.wait_ns);  // V of tile it landed
#pragma unroll
      for (int k0 = 0; k0 < kPaTile; k0 += 16)
        umma::mma_bf16(t_o, umma::desc_k16(aP, kPaTile, k0), umma::desc_mn_k16(aV, kPaTile, k0), idO,
                       it > 0 || k0 > 0);
      umma::commit(bar_o);
    }
    __syncwarp();
  }
  ok &= mbar_wait_bounded(bar_o, (n_tiles - 1) & 1, &never, v.wait_ns);
  __syncwarp();
  umma::fence_after_sync();

  // ---- output row i ----
  // tcgen05.ld is warp-collective (.sync.aligned): every lane of the warp
  // executes it, also lanes whose query lies past the prompt; only the
  // stores are guarded
  {
    // the row sum over the row's SPLIT threads
    s_red[h * kPaTile + r] = l;
    __syncthreads();
    float lsum = s_red[r];
#pragma unroll
    for (int x = 1; x < SPLIT; ++x) lsum += s_red[x * kPaTile + r];
    const float inv = i < P ? 1.f / lsum : 0.f;
    __nv_bfloat16* dst = out + (int64_t(b) * P + i) * q_stride + int64_t(hq) * D + h * OC;
#pragma unroll
    for (int cb = 0; cb < OC / 32; ++cb) {
      float o[32];
      umma::ld32(umma::taddr_of(t_o, warp, h * OC + cb * 32), o);
      umma::wait_ld();
      if (i < P) {
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint4 w4;
          w4.x = pack2_bf16(o[e + 0] * inv, o[e + 1] * inv);
          w4.y = pack2_bf16(o[e + 2] * inv, o[e + 3] * inv);
          w4.z = pack2_bf16(o[e + 4] * inv, o[e + 5] * inv);
          w4.w = pack2_bf16(o[e + 6] * inv, o[e + 7] * inv);
          *reinterpret_cast<uint4*>(dst + cb * 32 + e) = w4;
        }
      }
    }
  }
  // ---- fused compaction: the diagonal key tile's kept rows into the pool ----
  // (its V rows are still in shared memory; its K rows come back into the
  // query buffer, which no product reads any more)
  if (compact && hq % g == 0 && v.hdr->prefill_go) {
    if (tid == 0) load_tile(smem + S::Q, &tk, hkv * D, qt * kPaTile, bar_q);
    __syncwarp();
    int* s_kept = reinterpret_cast<int*>(smem + S::P);  // P is no longer read
    const int hd = v.head(layer, seq0 + b, hkv);
    auto keep_of = [&](int j, uint8_t* fl) {
      const uint8_t f = j < P ? evict[(int64_t(b) * P + j) * v.Hkv + hkv] : 0;
      *fl = f;
      return j < P && (f == 0 || (P - 1 - j) < v.w);
    };
    uint8_t f = 0, f_unused = 0;
    const int j = i0 + r;
    const bool keep = keep_of(j, &f);
    const unsigned bm = __ballot_sync(0xffffffffu, keep);
    // the prefix counts cover 256-token chunks; a second-half tile adds the
    // kept count of the first half
    const bool first_half_keep = (qt & 1) ? keep_of(j - kPaTile, &f_unused) : false;
    const unsigned bm1 = __ballot_sync(0xffffffffu, first_half_keep);
    if (lane == 0 && h == 0) {
      s_scan[warp] = __popc(bm);
      s_scan[4 + warp] = __popc(bm1);
    }
    __syncthreads();
    int before = 0, nkept = 0, first_half = 0;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      before += w < warp ? s_scan[w] : 0;
      nkept += s_scan[w];
      first_half += s_scan[4 + w];
    }
    const int rank = before + __popc(bm & ((1u << lane) - 1u));
    const int base = v.chunk_counts[(int64_t(b) * v.Hkv + hkv) * v.n_chunks_max + (qt >> 1)] + first_half;
    const int32_t* table = v.bt + int64_t(hd) * v.mbh;
    if (keep && h == 0) {
      s_kept[rank] = r;
      if (j >= P - v.w) {
        const int slot = base + rank;
        const int64_t ri = int64_t(hd) * v.w + (j % v.w);
        v.ring[ri] = uint32_t(slot) | (uint32_t(f != 0) << 31);
        v.ring_row[ri] = table[slot / v.BT] * v.BT + slot % v.BT;
      }
    }
    ok &= mbar_wait_bounded(bar_q, 1, &never, v.wait_ns);  // K rows of the diagonal tile
    __syncwarp();
    __syncthreads();
    constexpr int CH = D / 8;
    for (int idx = tid; idx < nkept * CH; idx += THREADS) {
      const int kk = idx / CH, c = idx % CH;
      const int kr = s_kept[kk];
      const int slot = base + kk, row = slot % v.BT;
      const int blk = table[slot / v.BT];
      if (!DMS_CHECK(blk >= 0 && blk < v.max_blocks && slot / v.BT < v.mbh, v.hdr, 501, hd, slot)) continue;
      uint8_t* dst = v.blocks + int64_t(blk) * v.block_bytes + int64_t(row) * v.row_bytes + swz_chunk(c, row) * 16;
      const uint32_t so = umma::sw128_offset(kPaTile, kr, c * 8);
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(smem + S::Q + so);
      *reinterpret_cast<uint4*>(dst + v.tile_bytes) = *reinterpret_cast<const uint4*>(smem + S::KV + so);
    }
  }

  if (!ok && tid == 0) report_error(v.hdr, DMS_DEVERR_TIMEOUT, layer, seq0 + b, hq);
  umma::fence_before_sync();
  __syncthreads();
  if (warp == 0) umma::tmem_dealloc(tbase, 256);
}

// ---------------------------------------------------------------------------
// Two query heads of one kv-head per CTA (sparse reading, an even group
// size g).  The heads share every K and V tile; per key tile the MMA thread
// issues S_A = Q_A K^T and S_B = Q_B K^T, and the softmax of head A runs
// while S_B is computed, that of head B while P_A V is, so the tensor cores
// and the softmax warps work at the same time inside one CTA.  K and V have
// their own buffers: the next key tile loads as soon as both S products have
// read the current one, during the softmax; the values of a tile load once
// both P V products of the previous tile are done.  One CTA per SM (the four
// accumulators take all 512 tensor-memory columns).
//
// Warps 0-7 run head A's softmax, 8-15 head B's (two threads per query row,
// as above), warp 16 loads tiles and issues the MMAs (one thread).  The
// hand-offs are mbarriers: S ready (commit), P ready (one arrival per
// softmax warp), O done (commit), K and V buffers free (commit).
//
// FP8 and 4-bit stores hold quantised rows, while the prompt's attention runs
// on the bf16 keys and values; for them warp 17 fetches each old-key tile
// from the prompt instead: the compaction left the prompt position of every
// kept slot in the pool's scratch, so tile t is the prompt rows of slots
// [128 t, 128 t + 128), gathered 16 bytes at a time (cp.async) into the
// swizzled operand image, the keys by warp 17 and the values by warp 18.
// The MMA thread requests each tile (an mbarrier per K / V buffer) when it
// would have loaded it; the gather warp waits for its copies, fences them
// for the tensor cores and arrives on the buffer's full barrier.
constexpr int kPpThreads = 2 * 2 * kPaTile + 96;
constexpr int kPpMaxFarIds = 2048;   // far-tile block ids cached in shared memory

template <int D>
struct PpSmem {
  static constexpr int TILE = kPaTile * D * 2;
  static constexpr int QA = 0, QB = TILE, K = 2 * TILE, V = 3 * TILE;
  static constexpr int PA = 4 * TILE;                          // [128 queries x 128 keys] bf16
  static constexpr int PB = PA + kPaTile * kPaTile * 2;
  static constexpr int FLAGS = PB + kPaTile * kPaTile * 2;     // [2 heads][2][4] words
  static constexpr int BARS = FLAGS + 64;                      // 16 mbarriers
  static constexpr int MISC = BARS + 128;                      // tmem base, abort, counts
  static constexpr int RED = MISC + 256;                       // [2 heads][2 parts][128] floats
  static constexpr int IDS = RED + 2 * 2 * kPaTile * 4;        // far-tile block ids
  static constexpr int USED = IDS + kPpMaxFarIds * 4;
  // at least 116 KB, so that a second CTA never waits on an SM for tensor memory
  static constexpr int BYTES = (USED > 116 * 1024 ? USED : 116 * 1024) + 1024;
};

__device__ __forceinline__ void pp_group_bar(int grp) {
  asm volatile("bar.sync %0, 256;" ::"r"(1 + grp) : "memory");
}

// 16 bytes global -> shared, bypassing L1; completion by cp_async_wait_all
__device__ __forceinline__ void cp_async16(uint32_t smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_dst), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

template <int D>
__global__ void __launch_bounds__(kPpThreads, 1)
    prefill_pair_kernel(PoolView v, int layer, int seq0, int P, const __grid_constant__ CUtensorMap tq,
                        const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                        const __grid_constant__ CUtensorMap tpool, const uint8_t* evict,
                        __nv_bfloat16* out, float scale_log2, int n_qtiles, const __nv_bfloat16* kin,
                        const __nv_bfloat16* vin, int far_in) {
  using S = PpSmem<D>;
  constexpr int SPLIT = 2, HC = kPaTile / SPLIT, OC = D / SPLIT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qt = n_qtiles - 1 - int(blockIdx.x);  // heaviest query tiles first
  const int hq0 = 2 * int(blockIdx.y), b = blockIdx.z;
  const int g = v.Hq / v.Hkv, hkv = hq0 / g;
  const int i0 = qt * kPaTile;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::BARS);
  uint64_t* bar_q = bars + 0;
  uint64_t* bar_k = bars + 1;
  uint64_t* bar_v = bars + 2;
  uint64_t* bar_kfree = bars + 3;
  uint64_t* bar_vfree = bars + 4;
  uint64_t* bar_s = bars + 5;    // [2] S of head A / B computed
  uint64_t* bar_o = bars + 7;    // [2] P V of head A / B computed
  uint64_t* bar_p = bars + 9;    // [2] P of head A / B in shared memory
  uint64_t* bar_fin = bars + 11; // every MMA done (exit)
  uint64_t* req_k = bars + 12;   // far_in: the MMA thread asks for the next old-key tile's keys
  uint64_t* req_v = bars + 13;   // ... and values
  int* s_misc = reinterpret_cast<int*>(smem + S::MISC);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(s_misc);
  volatile int* s_abort = s_misc + 1;
  int* s_cnt = s_misc + 8;       // [4] (far_keys)
  int* s_ids = reinterpret_cast<int*>(smem + S::IDS);

  if (tid == 0) {
    for (int x = 0; x < 14; ++x) mbar_init(&bars[x], x == 9 || x == 10 ? 8 : 1);
    s_misc[1] = 0;
    s_misc[2] = *reinterpret_cast<volatile uint32_t*>(&v.hdr->error) != 0u;
    fence_mbar_init();
    // both query tiles, while the key schedule is worked out
    mbar_arrive_expect_tx(bar_q, 2 * S::TILE);
#pragma unroll
    for (int kb = 0; kb < D / 64; ++kb) {
      umma::tma_load_3d(smem + S::QA + kb * kPaTile * 128, &tq, hq0 * D + kb * 64, i0, b, bar_q);
      umma::tma_load_3d(smem + S::QB + kb * kPaTile * 128, &tq, (hq0 + 1) * D + kb * 64, i0, b, bar_q);
    }
  }
  if (warp == 16) {
    umma::tmem_alloc(s_tmem, 512);
    umma::tmem_relinquish();
  }

  // ---- the key tiles of this query tile (as in prefill_attn_kernel) ----
  // The store holds this head's prompt when the layer's compaction (just
  // before this kernel) succeeded for every head: the error word is clear
  // (it is sticky, so an earlier error also sends every tile to the prompt).
  int kt_lo = 0, nf = 0, n_far = 0;
  const int32_t* far_bt = v.bt + int64_t(v.head(layer, seq0 + b, hkv)) * v.mbh;
  {
    const int lo = i0 - v.w + 1;
    const int kl = lo > 0 ? lo / kPaTile : 0;
    if (kl > 0) {
      const int held = v.n_slots[v.head(layer, seq0 + b, hkv)];
      __syncthreads();   // s_misc[2] (error word, read by thread 0)
      const int tf = far_keys(v, evict, b, hkv, P, kl * kPaTile, tid, s_cnt);
      const int nft = (tf + kPaTile - 1) / kPaTile;
      if (!s_misc[2] && nft * kPaTile <= held && 2 * nft <= v.mbh) {
        kt_lo = kl;
        nf = nft;
        n_far = tf;
      }
    }
  }
  const int n_tiles = nf + (qt - kt_lo + 1);
  umma::fence_before_sync();
  __syncthreads();  // barriers initialised, tensor memory allocated
  umma::fence_after_sync();
  const uint32_t tbase = *s_tmem;

  if (warp == 16) {
    // ======================= loads and MMAs (one thread) =======================
    const bool cached = !far_in && 2 * nf <= kPpMaxFarIds;
    if (cached)
      for (int x = lane; x < 2 * nf; x += 32) s_ids[x] = far_bt[x];
    __syncwarp();
    if (lane == 0) {
      auto far_id = [&](int x) { return cached ? s_ids[x] : far_bt[x]; };
      auto load_tile = [&](uint8_t* dst, const CUtensorMap* map, int x0, int row0, uint64_t* bar) {
        mbar_arrive_expect_tx(bar, S::TILE);
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb)
          umma::tma_load_3d(dst + kb * kPaTile * 128, map, x0 + kb * 64, row0, b, bar);
      };
      // tile it's keys (kv = 0) or values (kv = 1) into dst
      auto load_kv = [&](int it, int kv, uint64_t* bar) {
        uint8_t* dst = smem + (kv ? S::V : S::K);
        if (it < nf && far_in) {
          mbar_arrive(kv ? req_v : req_k);   // warp 17 gathers it from the prompt
        } else if (it < nf) {
          const int blk0 = far_id(2 * it), blk1 = far_id(2 * it + 1);
          mbar_arrive_expect_tx(bar, S::TILE);
#pragma unroll
          for (int kb = 0; kb < D / 64; ++kb) {
            umma::tma_load_4d(dst + kb * kPaTile * 128, &tpool, 0, kb, 0, 2 * blk0 + kv, bar);
            umma::tma_load_4d(dst + kb * kPaTile * 128 + 64 * 128, &tpool, 0, kb, 0, 2 * blk1 + kv, bar);
          }
        } else {
          load_tile(dst, kv ? &tv : &tk, hkv * D, (kt_lo + it - nf) * kPaTile, bar);
        }
      };
      constexpr uint32_t idS = umma::idesc_bf16_f32(kPaTile, kPaTile);
      constexpr uint32_t idO = umma::idesc_bf16_f32_bmn(kPaTile, D);
      const uint32_t aQ[2] = {smem_u32(smem + S::QA), smem_u32(smem + S::QB)};
      const uint32_t aPb[2] = {smem_u32(smem + S::PA), smem_u32(smem + S::PB)};
      const uint32_t aK = smem_u32(smem + S::K), aV = smem_u32(smem + S::V);
      load_kv(0, 0, bar_k);
      load_kv(0, 1, bar_v);
      int nk = 1, nv = 1, wk = 0, wv = 0;   // loads issued / waited on
      bool qdone = false, ok = true;
      // S of head hh for tile it (its keys have landed)
      auto mma_s = [&](int hh) {
#pragma unroll
        for (int k0 = 0; k0 < D; k0 += 16)
          umma::mma_bf16(tbase + 256 * hh, umma::desc_k16(aQ[hh], kPaTile, k0), umma::desc_k16(aK, kPaTile, k0),
                         idS, k0 > 0);
        umma::commit(&bar_s[hh]);
      };
      auto mma_pv = [&](int hh, int it) {
#pragma unroll
        for (int k0 = 0; k0 < kPaTile; k0 += 16)
          umma::mma_bf16(tbase + 256 * hh + 128, umma::desc_k16(aPb[hh], kPaTile, k0),
                         umma::desc_mn_k16(aV, kPaTile, k0), idO, it > 0 || k0 > 0);
        umma::commit(&bar_o[hh]);
      };
      // Issue order: S_A(0) S_B(0), then per tile it: P_A V(it), S_A(it+1),
      // P_B V(it), S_B(it+1).  While head A's softmax of tile it + 1 runs, the
      // tensor cores compute head B's P V of tile it and S of tile it + 1,
      // and the other way round.
      ok = mbar_wait_bounded(bar_q, 0, s_abort, v.wait_ns);
      qdone = ok;
      ok = ok && mbar_wait_bounded(bar_k, 0, s_abort, v.wait_ns);
      if (ok) {
        wk = 1;
        umma::fence_after_sync();
        mma_s(0);
        mma_s(1);
        umma::commit(bar_kfree);   // phase 0: both S of tile 0 read the keys
        if (n_tiles > 1) {
          ok = mbar_wait_bounded(bar_kfree, 0, s_abort, v.wait_ns);
          if (ok) {
            load_kv(1, 0, bar_k);
            nk = 2;
          }
        }
      }
      for (int it = 0; it < n_tiles && ok; ++it) {
        const bool more = it + 1 < n_tiles;
        if (!(ok = mbar_wait_bounded(bar_v, it & 1, s_abort, v.wait_ns))) break;
        wv = it + 1;
        if (!(ok = mbar_wait_bounded(&bar_p[0], it & 1, s_abort, v.wait_ns))) break;
        umma::fence_after_sync();
        mma_pv(0, it);
        if (more) {
          if (!(ok = mbar_wait_bounded(bar_k, (it + 1) & 1, s_abort, v.wait_ns))) break;
          wk = it + 2;
          umma::fence_after_sync();
          mma_s(0);
        }
        if (!(ok = mbar_wait_bounded(&bar_p[1], it & 1, s_abort, v.wait_ns))) break;
        umma::fence_after_sync();
        mma_pv(1, it);
        umma::commit(bar_vfree);     // phase it: both P V of tile it read the values
        if (more) {
          mma_s(1);
          umma::commit(bar_kfree);   // phase it + 1: both S of tile it + 1 read the keys
          if (!(ok = mbar_wait_bounded(bar_vfree, it & 1, s_abort, v.wait_ns))) break;
          load_kv(it + 1, 1, bar_v);
          nv = it + 2;
          if (it + 2 < n_tiles) {
            if (!(ok = mbar_wait_bounded(bar_kfree, (it + 1) & 1, s_abort, v.wait_ns))) break;
            load_kv(it + 2, 0, bar_k);
            nk = it + 3;
          }
        }
      }
      if (!ok) {
        *s_abort = 1;
        report_error(v.hdr, DMS_DEVERR_TIMEOUT, layer, seq0 + b, hq0);
      }
      // drain: every MMA issued and every copy still landing, each wait bounded
      volatile int never = 0;
      umma::commit(bar_fin);
      mbar_wait_bounded(bar_fin, 0, &never, v.wait_ns);
      if (!qdone) mbar_wait_bounded(bar_q, 0, &never, v.wait_ns);
      if (nk > wk) mbar_wait_bounded(bar_k, (nk - 1) & 1, &never, v.wait_ns);
      if (nv > wv) mbar_wait_bounded(bar_v, (nv - 1) & 1, &never, v.wait_ns);
    }
    __syncwarp();
  } else if (warp >= 17) {
    // ============ old-key tiles from the prompt (quantised stores) ============
    // warp 17 gathers the keys, warp 18 the values
    const int kv = warp - 17;
    if (far_in && nf > 0) {
      constexpr int NCH = D / 8, RPP = 32 / NCH;   // 16-byte chunks per row, rows per pass
      const int32_t* pos = v.pos_of_slot + (int64_t(b) * v.Hkv + hkv) * (int64_t(v.mbh) * v.BT);
      const int64_t tok_elems = int64_t(v.Hkv) * D;
      bool ok = true;
      for (int t = 0; t < nf && ok; ++t) {
        int prow[4];   // prompt positions of the tile's rows lane, lane + 32, + 64, + 96
#pragma unroll
        for (int x = 0; x < 4; ++x) prow[x] = pos[int64_t(t) * kPaTile + 32 * x + lane];
        {
          if (lane == 0) {
            ok = mbar_wait_bounded(kv ? req_v : req_k, t & 1, s_abort, v.wait_ns);
            if (!ok) *s_abort = 1;
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          const __nv_bfloat16* src = (kv ? vin : kin) + int64_t(b) * P * tok_elems + int64_t(hkv) * D;
          const uint32_t dst = smem_u32(smem + (kv ? S::V : S::K));
          const int c = lane % NCH;
#pragma unroll
          for (int pss = 0; pss < 4 * NCH; ++pss) {   // RPP whole rows per pass, coalesced
            const int rr = pss * RPP + lane / NCH;
            const int x = (pss * RPP) >> 5;
            const int mine = x == 0 ? prow[0] : x == 1 ? prow[1] : x == 2 ? prow[2] : prow[3];
            const int prompt_row = __shfl_sync(0xffffffffu, mine, rr & 31);
            cp_async16(dst + umma::sw128_offset(kPaTile, rr, c * 8), src + int64_t(prompt_row) * tok_elems + c * 8);
          }
          cp_async_wait_all();
          fence_proxy_async_smem();   // the copies, before the tensor cores read them
          __syncwarp();
          if (lane == 0) mbar_arrive(kv ? bar_v : bar_k);
        }
      }
      if (!ok && lane == 0) report_error(v.hdr, DMS_DEVERR_TIMEOUT, layer, seq0 + b, hq0);
    }
    __syncwarp();
  } else {
    // ======================= softmax of head A (warps 0-7) or B (8-15) =======================
    const int G = warp >> 3;
    const int tg = tid & 255, r = tg & (kPaTile - 1), h = tg >> 7, wg = tg >> 5;
    const int i = i0 + r;
    const int hq = hq0 + G;
    uint32_t* fbits = reinterpret_cast<uint32_t*>(smem + S::FLAGS) + 8 * G;   // [2][4]
    float* red = reinterpret_cast<float*>(smem + S::RED) + 2 * kPaTile * G;   // [2 parts][128]
    uint8_t* Pbuf = smem + (G ? S::PB : S::PA);
    const uint32_t t_s = tbase + 256 * G, t_o = t_s + 128;
    auto flag_at = [&](int it) -> uint8_t {
      if (it < nf || h != 0) return 0;
      const int j = (kt_lo + it - nf) * kPaTile + r;
      return j < P ? evict[(int64_t(b) * P + j) * v.Hkv + hkv] : 0;
    };
    // a wait that gives up stops every other wait of the CTA at once
    auto wait_g = [&](uint64_t* bar, uint32_t parity) {
      if (mbar_wait_bounded(bar, parity, s_abort, v.wait_ns)) return true;
      *s_abort = 1;
      return false;
    };
    float m = -1e30f, l = 0.f;
    bool ok = true;
    uint8_t f_cur = flag_at(0);
    for (int it = 0; it < n_tiles; ++it) {
      const bool far = it < nf;
      const int cur = it & 1, j0 = (kt_lo + it - nf) * kPaTile;
      {
        const unsigned fw = __ballot_sync(0xffffffffu, f_cur != 0);
        if (lane == 0 && h == 0) fbits[cur * 4 + wg] = fw;
      }
      const uint8_t f_next = it + 1 < n_tiles ? flag_at(it + 1) : 0;
      // one warp of the head polls the mbarrier; the named barrier holds the
      // other seven without issuing (it also publishes the flag bits)
      if (wg == 0) ok &= wait_g(&bar_s[G], it & 1);
      __syncwarp();
      pp_group_bar(G);
      umma::fence_after_sync();
      uint32_t vis[HC / 32];
      if (far) {
        const int lim = n_far - it * kPaTile;
#pragma unroll
        for (int x = 0; x < HC / 32; ++x) {
          const int x_lt = lim - 32 * ((HC / 32) * h + x);
          vis[x] = x_lt <= 0 ? 0u : x_lt >= 32 ? ~0u : (1u << x_lt) - 1u;
        }
      } else {
        const int hi = i - j0, lo = i - v.w + 1 - j0, end = P - j0;
#pragma unroll
        for (int x = 0; x < HC / 32; ++x) {
          const int wd = (HC / 32) * h + x, c0 = 32 * wd;
          const int x_le = hi - c0, x_ge = lo - c0, x_lt = end - c0;
          const uint32_t le = x_le < 0 ? 0u : x_le >= 31 ? ~0u : (2u << x_le) - 1u;
          const uint32_t ge = x_ge <= 0 ? ~0u : x_ge >= 32 ? 0u : ~((1u << x_ge) - 1u);
          const uint32_t lt = x_lt <= 0 ? 0u : x_lt >= 32 ? ~0u : (1u << x_lt) - 1u;
          vis[x] = (~fbits[cur * 4 + wd] | ge) & le & lt;
        }
      }
      float s[HC];
#pragma unroll
      for (int cb = 0; cb < HC / 32; ++cb) {
        float x[32];
        umma::ld32(umma::taddr_of(t_s, warp, h * HC + cb * 32), x);
#pragma unroll
        for (int e = 0; e < 32; ++e) s[cb * 32 + e] = x[e];
      }
      umma::wait_ld();
      // mask only the 32-key words that are not wholly visible
#pragma unroll
      for (int x = 0; x < HC / 32; ++x) {
        if (vis[x] != ~0u) {
#pragma unroll
          for (int e = 0; e < 32; ++e) s[x * 32 + e] = ((vis[x] >> e) & 1u) ? s[x * 32 + e] : -INFINITY;
        }
      }
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < HC; c += 2) mx4[(c >> 1) & 3] = fmax3(mx4[(c >> 1) & 3], s[c], s[c + 1]);
      red[h * kPaTile + r] = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3])) * scale_log2;
      pp_group_bar(G);
      float mx = red[r];
#pragma unroll
      for (int x = 1; x < SPLIT; ++x) mx = fmaxf(mx, red[x * kPaTile + r]);
      float alpha = 1.f;
      if (mx > m + 8.f) {   // lazy rescaling, as in prefill_attn_kernel
        alpha = fast_exp2(m - mx);
        m = mx;
      }
      float sum4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < HC; c += 2) {
        float a0, a1;
        ffma2(a0, a1, s[c], s[c + 1], scale_log2, scale_log2, -m, -m);
        s[c] = fast_exp2(a0);
        s[c + 1] = fast_exp2(a1);
        const int q = (c >> 1) & 1;
        fadd2(sum4[2 * q], sum4[2 * q + 1], sum4[2 * q], sum4[2 * q + 1], s[c], s[c + 1]);
      }
      l = l * alpha + ((sum4[0] + sum4[1]) + (sum4[2] + sum4[3]));
      if (it > 0) {   // P V of the previous tile: P buffer free, O settled
        ok &= wait_g(&bar_o[G], (it - 1) & 1);
        __syncwarp();
        umma::fence_after_sync();
      }
#pragma unroll
      for (int ch = 0; ch < HC / 8; ++ch) {
        uint4 w4;
        w4.x = pack2_bf16(s[ch * 8 + 0], s[ch * 8 + 1]);
        w4.y = pack2_bf16(s[ch * 8 + 2], s[ch * 8 + 3]);
        w4.z = pack2_bf16(s[ch * 8 + 4], s[ch * 8 + 5]);
        w4.w = pack2_bf16(s[ch * 8 + 6], s[ch * 8 + 7]);
        *reinterpret_cast<uint4*>(Pbuf + umma::sw128_offset(kPaTile, r, h * HC + ch * 8)) = w4;
      }
      if (it > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
        for (int cb = 0; cb < OC / 32; ++cb) {
          float o[32];
          umma::ld32(umma::taddr_of(t_o, warp, h * OC + cb * 32), o);
          umma::wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= alpha;
          umma::st32(umma::taddr_of(t_o, warp, h * OC + cb * 32), o);
        }
        umma::wait_st();
      }
      fence_proxy_async_smem();   // P before the tensor cores read it
      umma::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_p[G]);
      f_cur = f_next;
    }
    if (wg == 0) ok &= wait_g(&bar_o[G], (n_tiles - 1) & 1);
    __syncwarp();
    pp_group_bar(G);   // the last P V is done; every thread has read the last row maxima
    umma::fence_after_sync();
    red[h * kPaTile + r] = l;
    pp_group_bar(G);
    float lsum = red[r];
#pragma unroll
    for (int x = 1; x < SPLIT; ++x) lsum += red[x * kPaTile + r];
    const float inv = i < P ? 1.f / lsum : 0.f;
    __nv_bfloat16* dst = out + (int64_t(b) * P + i) * (int64_t(v.Hq) * D) + int64_t(hq) * D + h * OC;
#pragma unroll
    for (int cb = 0; cb < OC / 32; ++cb) {
      float o[32];
      umma::ld32(umma::taddr_of(t_o, warp, h * OC + cb * 32), o);
      umma::wait_ld();
      if (i < P) {
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint4 w4;
          w4.x = pack2_bf16(o[e + 0] * inv, o[e + 1] * inv);
          w4.y = pack2_bf16(o[e + 2] * inv, o[e + 3] * inv);
          w4.z = pack2_bf16(o[e + 4] * inv, o[e + 5] * inv);
          w4.w = pack2_bf16(o[e + 6] * inv, o[e + 7] * inv);
          *reinterpret_cast<uint4*>(dst + cb * 32 + e) = w4;
        }
      }
    }
    if (!ok && tg == 0) report_error(v.hdr, DMS_DEVERR_TIMEOUT, layer, seq0 + b, hq);
  }
  umma::fence_before_sync();
  __syncthreads();
  if (warp == 16) umma::tmem_dealloc(tbase, 512);
}

}  // namespace dms

using namespace dms;

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library)
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// Tensor map of a [batch, P, H * D] bf16 tensor: boxes of 64 elements x 128
// rows x 1 sequence, 128-byte swizzle, zeros outside.
static dms_status encode_bf16_map(CUtensorMap* m, const void* base, int batch, int P, int HD) {
  auto enc = tensor_map_encoder();
  if (!enc) {
    set_last_error("cuTensorMapEncodeTiled is not available");
    return DMS_ERR_CUDA;
  }
  const cuuint64_t dims[3] = {cuuint64_t(HD), cuuint64_t(P), cuuint64_t(batch)};
  const cuuint64_t strides[2] = {cuuint64_t(HD) * 2, cuuint64_t(HD) * 2 * cuuint64_t(P)};
  const cuuint32_t box[3] = {64, cuuint32_t(kPaTile), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_last_error("cuTensorMapEncodeTiled failed (%d)", int(r));
    return DMS_ERR_CUDA;
  }
  return DMS_OK;
}

// Tensor map of the store's blocks as [2 * max_blocks tiles (block b's K
// tile is 2b, its V tile 2b + 1)][64 rows][D / 64 halves][64 bf16]: boxes of
// one 64-column half of 64 rows, no swizzle (the rows are stored swizzled).
static dms_status encode_store_map(CUtensorMap* m, const PoolView& pv) {
  auto enc = tensor_map_encoder();
  if (!enc) {
    set_last_error("cuTensorMapEncodeTiled is not available");
    return DMS_ERR_CUDA;
  }
  const cuuint64_t dims[4] = {64, cuuint64_t(pv.D / 64), cuuint64_t(kBlockTokens), cuuint64_t(2 * pv.max_blocks)};
  const cuuint64_t strides[3] = {128, cuuint64_t(pv.row_bytes), cuuint64_t(pv.tile_bytes)};
  const cuuint32_t box[4] = {64, 1, cuuint32_t(kBlockTokens), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, pv.blocks, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_last_error("cuTensorMapEncodeTiled (store) failed (%d)", int(r));
    return DMS_ERR_CUDA;
  }
  return DMS_OK;
}

extern "C" dms_status dms_prefill_attn(dms_pool* pool, int layer, int seq0, int batch, int prompt_len,
                                       const void* q, const void* k, const void* v,
                                       dms_dtype in_dtype, const uint8_t* evict, void* out,
                                       float sm_scale, cudaStream_t stream) {
  if (!pool) {
    set_last_error("null pool");
    return DMS_ERR_INVALID_ARG;
  }
  const PoolView& pv = pool->view;
  if (pv.kv_dtype == DMS_F32 || in_dtype != DMS_BF16 || (pv.D != 64 && pv.D != 128)) {
    set_last_error("dms_prefill_attn needs a bf16, FP8 or 4-bit pool, bf16 inputs and head_dim 64 or 128");
    return DMS_ERR_UNSUPPORTED;
  }
  if (layer < 0 || layer >= pv.L || seq0 < 0 || batch < 1 || seq0 + batch > pv.Bmax ||
      batch > 65535 || prompt_len < 1 || prompt_len > pool->cfg.max_context) {
    set_last_error("bad layer/sequences/prompt_len (%d, %d+%d, %d)", layer, seq0, batch, prompt_len);
    return DMS_ERR_INVALID_ARG;
  }
  if (!q || !k || !v || !evict || !out) {
    set_last_error("null pointer argument");
    return DMS_ERR_INVALID_ARG;
  }
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v) |
       reinterpret_cast<uintptr_t>(out)) & 15) {
    set_last_error("q, k, v and out must be 16-byte aligned");
    return DMS_ERR_INVALID_ARG;
  }
  // bf16 store, sparse (default): the layer is compacted first and the
  // attention kernel reads the old kept keys back from the store.  bf16
  // store, dense: the kept rows come from the attention kernel's tiles, after
  // the prefix counts and block tables of the plan kernel.  FP8 and 4-bit
  // stores quantise the rows: the layer is compacted first, as by
  // dms_compact_prefill_seqs (scales, plan, scatter), and the attention
  // kernel reads every key from the bf16 inputs.
  const bool bf16_store = pv.kv_dtype == DMS_BF16;
  const bool even_g = (pv.Hq / pv.Hkv) % 2 == 0;
  const int sparse = bf16_store && pool->prefill_mode == DMS_PREFILL_SPARSE &&
                     2 * pv.max_blocks <= int64_t(INT32_MAX) ? 1 : 0;
  // quantised stores: old kept keys gathered from the prompt by position
  // (two query heads per CTA only)
  const int far_in = !bf16_store && pool->prefill_mode == DMS_PREFILL_SPARSE && even_g && pv.pos_of_slot ? 1 : 0;
  const int fused = bf16_store && !sparse ? 1 : 0;
  CUtensorMap tpool;
  memset(&tpool, 0, sizeof(tpool));
  dms_status st = sparse ? encode_store_map(&tpool, pv) : DMS_OK;
  if (st != DMS_OK) return st;
  st = fused ? prefill_plan_launch(pool, layer, seq0, batch, prompt_len, evict, stream)
             : dms_compact_prefill_seqs(pool, layer, seq0, batch, prompt_len, k, v, in_dtype, evict, stream);
  if (st != DMS_OK) return st;
  const int n_qtiles = (prompt_len + kPaTile - 1) / kPaTile;
  const dim3 grid(n_qtiles, pv.Hq, batch);
  const float sc = sm_scale > 0.f ? sm_scale : 1.0f / sqrtf(float(pv.D));
  const float scale_log2 = sc * 1.4426950408889634f;
  CUtensorMap tq, tk, tv;
  st = encode_bf16_map(&tq, q, batch, prompt_len, pv.Hq * pv.D);
  if (st == DMS_OK) st = encode_bf16_map(&tk, k, batch, prompt_len, pv.Hkv * pv.D);
  if (st == DMS_OK) st = encode_bf16_map(&tv, v, batch, prompt_len, pv.Hkv * pv.D);
  if (st != DMS_OK) return st;
  auto ko = static_cast<__nv_bfloat16*>(out);
  if ((sparse && even_g) || far_in) {   // two query heads of a kv-head per CTA
    const dim3 grid2(n_qtiles, pv.Hq / 2, batch);
    if (pv.D == 128) {
      static FuncAttrCache smem_attr;  // per device
      st = ensure_func_attr(reinterpret_cast<const void*>(prefill_pair_kernel<128>),
                            cudaFuncAttributeMaxDynamicSharedMemorySize, int(PpSmem<128>::BYTES), smem_attr,
                            "prefill pair smem attribute");
      if (st != DMS_OK) return st;
      prefill_pair_kernel<128><<<grid2, kPpThreads, PpSmem<128>::BYTES, stream>>>(
          pv, layer, seq0, prompt_len, tq, tk, tv, tpool, evict, ko, scale_log2, n_qtiles,
          static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), far_in);
    } else {
      static FuncAttrCache smem_attr;  // per device
      st = ensure_func_attr(reinterpret_cast<const void*>(prefill_pair_kernel<64>),
                            cudaFuncAttributeMaxDynamicSharedMemorySize, int(PpSmem<64>::BYTES), smem_attr,
                            "prefill pair smem attribute");
      if (st != DMS_OK) return st;
      prefill_pair_kernel<64><<<grid2, kPpThreads, PpSmem<64>::BYTES, stream>>>(
          pv, layer, seq0, prompt_len, tq, tk, tv, tpool, evict, ko, scale_log2, n_qtiles,
          static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), far_in);
    }
    return cuda_status(cudaGetLastError(), "prefill_pair_kernel");
  }
  if (pv.D == 128) {
    static FuncAttrCache smem_attr, carveout_attr;  // per device
    st = ensure_func_attr(reinterpret_cast<const void*>(prefill_attn_kernel<128>),
                          cudaFuncAttributeMaxDynamicSharedMemorySize, int(PaSmem<128>::BYTES), smem_attr,
                          "prefill attn smem attribute");
    if (st != DMS_OK) return st;
    // two CTAs per SM: the whole shared-memory carveout
    st = ensure_func_attr(reinterpret_cast<const void*>(prefill_attn_kernel<128>),
                          cudaFuncAttributePreferredSharedMemoryCarveout, int(cudaSharedmemCarveoutMaxShared),
                          carveout_attr, "prefill attn carveout");
    if (st != DMS_OK) return st;
    prefill_attn_kernel<128><<<grid, PaSplit<128>::THREADS, PaSmem<128>::BYTES, stream>>>(
        pv, layer, seq0, prompt_len, tq, tk, tv, tpool, evict, ko, scale_log2, n_qtiles, fused, sparse);
  } else {
    static FuncAttrCache smem_attr, carveout_attr;  // per device
    st = ensure_func_attr(reinterpret_cast<const void*>(prefill_attn_kernel<64>),
                          cudaFuncAttributeMaxDynamicSharedMemorySize, int(PaSmem<64>::BYTES), smem_attr,
                          "prefill attn smem attribute");
    if (st != DMS_OK) return st;
    // two CTAs per SM: the whole shared-memory carveout
    st = ensure_func_attr(reinterpret_cast<const void*>(prefill_attn_kernel<64>),
                          cudaFuncAttributePreferredSharedMemoryCarveout, int(cudaSharedmemCarveoutMaxShared),
                          carveout_attr, "prefill attn carveout");
    if (st != DMS_OK) return st;
    prefill_attn_kernel<64><<<grid, PaSplit<64>::THREADS, PaSmem<64>::BYTES, stream>>>(
        pv, layer, seq0, prompt_len, tq, tk, tv, tpool, evict, ko, scale_log2, n_qtiles, fused, sparse);
  }
  return cuda_status(cudaGetLastError(), "prefill_attn_kernel");
}
