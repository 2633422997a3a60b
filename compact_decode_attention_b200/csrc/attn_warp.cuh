// Per-warp decode attention compute shared by the decode kernels: the
// online-softmax state of one consumer warp and the compute of one staged
// block ("unit") of up to 64 held rows, for every stored K/V format.
//
// DMS only changes which keys a query sees ("NVIDIA veröffentlicht
// Qwen3-8B-DMS-8x ..." (mindverse), section "Dynamic Memory Sparsification
// (DMS): Eine innovative Lösung"); a unit is plain softmax attention of the
// GQA group's queries over the unit's rows, accumulated online.
#pragma once

#include <math.h>

#include "dms_internal.cuh"

namespace dms {

enum { KV_F32 = 0, KV_BF16 = 1, KV_FP8 = 2, KV_INT4 = 3 };

// 4-bit codes: a LOP3 of the packed word with 0x64006400 turns the nibble
// at bits 0-3 (and 16-19) into the f16 value 1024 + n, and the nibble at
// bits 4-7 (and 20-23) into 1024 + 16 n; both are exact.  The offsets and
// the factor 16 are taken out in fp32 / on the other MMA operand.
// (w & mask) | magic as one LOP3: mask and magic come in registers (a LOP3
// takes a single immediate, and with two constants the compiler emits two).
__device__ __forceinline__ uint32_t lop3_and_or(uint32_t w, uint32_t mask, uint32_t magic) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(w), "r"(mask), "r"(magic));
  return r;
}
// The three decoding constants, held in registers for a warp's whole run
// (a warp shuffle hides their values from constant folding).
struct NibConsts {
  uint32_t lo, hi, magic;
  __device__ __forceinline__ void init() {
    lo = __shfl_sync(0xffffffffu, 0x000F000Fu, 0);
    hi = __shfl_sync(0xffffffffu, 0x00F000F0u, 0);
    magic = __shfl_sync(0xffffffffu, 0x64006400u, 0);
  }
};
__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  const __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// Stage ownership: unit k goes to stage k % NS and to consumer warp k % NCW.
// NS must be a multiple of NCW so that every stage always belongs to the same
// warp.  A parity wait only tells "this phase" from "the previous one"; if a
// stage were shared by two warps, one of them could start waiting two phases
// ahead of the barrier, see the older phase of the same parity as complete,
// and read (and release) a stage whose copy is still landing.
template <int KV, int D>
struct AttnTraits {
  static constexpr int ESZ = KV == KV_F32 ? 4 : KV == KV_BF16 ? 2 : 1;
  static constexpr int QESZ = KV == KV_F32 ? 4 : 2;  // q / out element bytes
  // 4-bit rows: 64 bytes of nibbles + 4 fp16 group scales (see DMS_INT4)
  static constexpr int ROWB = KV == KV_INT4 ? D / 2 + D / 16 : D * ESZ;
  static constexpr int TILEB = kBlockTokens * ROWB;
  // The fp32 path reads its query rows from the stage (QB bytes after the
  // tiles); the tensor-core paths load query fragments from global memory.
  static constexpr int QB = KV == KV_F32 ? 8 * D * QESZ : 0;
  static constexpr int STAGEB = 2 * TILEB + QB;
  // Tensor-core variants give every stage its own consumer warp (6 stages of
  // 34 KB for bf16 D=128, 8 for the others): with two consumer warps per SM
  // sub-partition one warp's MMA / ldmatrix latency hides behind the other's.
  // fp32 (68 KB or 34 KB stages): 3 or 4 stages and warps.
  // 4-bit stages are 9 KB: two per consumer warp keep 129 KB in flight;
  // 7 consumer warps + the producer leave two warps per SM sub-partition
  // (up to 255 registers a thread).
  // FP8 stages are 16 KB: two per consumer warp (6 warps, 192 KB in flight).
  static constexpr int NS = KV == KV_F32 ? (D == 128 ? 3 : 4)
                          : KV == KV_INT4 ? 14
                          : KV == KV_FP8 ? 12
                          : (KV == KV_BF16 && D == 128) ? 6 : 8;
  static constexpr int NCW = KV == KV_INT4 ? 7 : KV == KV_FP8 ? 6 : NS;   // consumer warps
  static constexpr int THREADS = 32 * (NCW + 1);       // + one producer warp
  static constexpr int COMBINE_FLOATS = NCW * 8 * D + 2 * NCW * 8;
  static constexpr int MISC_INTS = 16 + THREADS / 32;
  static constexpr int HEAD_WIN = 256;                 // held counts of the CTA's first heads
  static constexpr size_t SMEM = size_t(NS) * STAGEB + COMBINE_FLOATS * 4 + 2 * NS * 8 +
                                 MISC_INTS * 4 + HEAD_WIN * 4;
  static_assert(NS % NCW == 0, "each stage must always belong to the same consumer warp");
  static_assert(SMEM <= 227 * 1024, "shared memory budget");
  static_assert(STAGEB % 128 == 0, "stage alignment");
};

// Named barrier 1 among the consumer warps only (the producer never joins it).
template <int NCW>
__device__ __forceinline__ void consumer_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(32 * NCW) : "memory");
}

__device__ __forceinline__ int units_of(int n) { return (n + kBlockTokens - 1) / kBlockTokens; }

template <int QESZ>
__device__ __forceinline__ void store_out(uint8_t* out, int64_t idx, float x) {
  if constexpr (QESZ == 4) {
    reinterpret_cast<float*>(out)[idx] = x;
  } else {
    reinterpret_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(x);
  }
}

// ---------------------------------------------------------------------------
// Per-warp online-softmax state and unit compute, tensor-core paths
// ---------------------------------------------------------------------------
template <int KV, int D>
struct MmaWarp {
  static constexpr int KSTEPS = D / 16;  // QK^T k-steps over head_dim
  static constexpr int MTD = D / 16;     // PV m-tiles over head_dim
  using T = AttnTraits<KV, D>;
  float m[2], l[2];
  float o[MTD][4];
  uint32_t qf[KSTEPS][2];
  float scale;  // log2-domain score scale (includes the K scale for FP8)
  float vscale; // V scale (FP8), else 1
  // 4-bit stores only: per 32-element group g, minus the offset that the
  // 1024 + m n decoding adds to q . k for query columns 2(lane&3), +1 ...
  float cq[4][2];
  // ... and the one it adds to each output row of group g (accumulated like o)
  float eo[4][4];
  NibConsts nc;  // 4-bit decoding constants

  __device__ __forceinline__ void reset() {
    m[0] = m[1] = -INFINITY;
    l[0] = l[1] = 0.f;
#pragma unroll
    for (int i = 0; i < MTD; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    if constexpr (KV == KV_INT4) {
#pragma unroll
      for (int i = 0; i < 4; ++i) eo[i][0] = eo[i][1] = eo[i][2] = eo[i][3] = 0.f;
      nc.init();
    }
  }

  // Q^T B fragments of the group's query rows (row n = lane / 4 < g; the
  // rows past g are the zero padding of the N = 8 side), from global memory.
  __device__ __forceinline__ void load_q(const uint8_t* qg, int g, int lane) {
    const int n = lane >> 2, q2 = (lane & 3) * 2;
    const __nv_bfloat16* qrow = reinterpret_cast<const __nv_bfloat16*>(qg) + n * D;
    const bool real = n < g;
#pragma unroll
    for (int kt = 0; kt < KSTEPS; ++kt) {
      const uint32_t lo = real ? __ldg(reinterpret_cast<const unsigned int*>(qrow + kt * 16 + q2)) : 0u;
      const uint32_t hi = real ? __ldg(reinterpret_cast<const unsigned int*>(qrow + kt * 16 + 8 + q2)) : 0u;
      if constexpr (KV == KV_FP8) {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&lo));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hi));
        qf[kt][0] = pack_f16x2(a.x, a.y);
        qf[kt][1] = pack_f16x2(b.x, b.y);
      } else if constexpr (KV == KV_INT4) {
        // k-columns 8..15 of a k-step meet K nibbles decoded as 1024 + 16 n:
        // their query values enter divided by 16 (exact)
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&lo));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hi));
        qf[kt][0] = pack_f16x2(a.x, a.y);
        qf[kt][1] = pack_f16x2(b.x * 0.0625f, b.y * 0.0625f);
      } else {
        qf[kt][0] = lo;
        qf[kt][1] = hi;
      }
    }
    if constexpr (KV == KV_INT4) {
      // Sum over group g of q'_d (1024 + 8 m_d), q' the f16 operand and m_d
      // its nibble factor (1 or 16): what the decoding adds to the group's
      // dot product.  This lane holds query row lane/4; columns 2(lane&3),
      // 2(lane&3)+1 of the MMA accumulator need rows 2(lane&3) and +1.
#pragma unroll
      for (int gq = 0; gq < 4; ++gq) {
        float c = 0.f;
#pragma unroll
        for (int kt = 2 * gq; kt < 2 * gq + 2; ++kt) {
          const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&qf[kt][0]));
          const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&qf[kt][1]));
          c += 1032.f * (a.x + a.y) + 1152.f * (b.x + b.y);
        }
        c += __shfl_xor_sync(0xffffffffu, c, 1);
        c += __shfl_xor_sync(0xffffffffu, c, 2);
        cq[gq][0] = -__shfl_sync(0xffffffffu, c, 8 * (lane & 3));
        cq[gq][1] = -__shfl_sync(0xffffffffu, c, 8 * (lane & 3) + 4);
      }
    }
  }

  __device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                      uint32_t b1) {
    if constexpr (KV == KV_FP8 || KV == KV_INT4) mma_f16_16816(d, a, b0, b1);
    else mma_bf16_16816(d, a, b0, b1);
  }

  // A whole block (64 rows) takes a copy of the unit code with every row
  // check folded away; a head's last, partly filled block the general one.
  // `hole` (>= 0) is a row whose score is masked: a slot the same step
  // reuses for its new token, which reaches the softmax separately.
  __device__ __forceinline__ void unit(const uint8_t* stage, int rows, int lane, int hole = -1) {
    if (rows == kBlockTokens && hole < 0) unit_rows<true>(stage, kBlockTokens, lane, -1);
    else unit_rows<false>(stage, rows, lane, hole);
  }

  template <bool FULL>
  __device__ __forceinline__ void unit_rows(const uint8_t* stage, int rows_in, int lane, int hole_in) {
    const int rows = FULL ? kBlockTokens : rows_in;
    const int hole = FULL ? -1 : hole_in;
    const uint8_t* Ks = stage;
    const uint8_t* Vs = stage + T::TILEB;
    const int q = lane & 3, r8 = lane >> 2;
    float s[4][4];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) s[mt][0] = s[mt][1] = s[mt][2] = s[mt][3] = 0.f;
    // ---- S^T = K Q^T over the 64 rows (4 m-tiles of 16 tokens) ----
    // All four m-tiles are computed (rows past `rows` are masked to -inf
    // below), k-step outer, so each k-step issues four independent MMAs.
    if constexpr (KV == KV_BF16) {
      const uint32_t kbase = smem_u32(Ks);
#pragma unroll
      for (int kt = 0; kt < KSTEPS; ++kt) {
        const int ch = 2 * kt + (lane >> 4);
        uint32_t a[4][4];
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          const int row = mt * 16 + (lane & 15);
          ldmatrix_x4(a[mt], kbase + row * T::ROWB + (swz_chunk(ch, row) << 4));
        }
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) mma(s[mt], a[mt], qf[kt][0], qf[kt][1]);
      }
    }
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      if constexpr (KV == KV_FP8) {
        if (mt * 16 < rows) {  // FP8, D = 128: two 16-byte loads per row give all 8 k-steps
          const int r0 = mt * 16 + r8, r1 = r0 + 8;
          const uint4 a0lo = *reinterpret_cast<const uint4*>(Ks + r0 * 128 + (((2 * q) ^ (r0 & 7)) << 4));
          const uint4 a0hi = *reinterpret_cast<const uint4*>(Ks + r0 * 128 + (((2 * q + 1) ^ (r0 & 7)) << 4));
          const uint4 a1lo = *reinterpret_cast<const uint4*>(Ks + r1 * 128 + (((2 * q) ^ (r1 & 7)) << 4));
          const uint4 a1hi = *reinterpret_cast<const uint4*>(Ks + r1 * 128 + (((2 * q + 1) ^ (r1 & 7)) << 4));
          const uint32_t w0[8] = {a0lo.x, a0lo.y, a0lo.z, a0lo.w, a0hi.x, a0hi.y, a0hi.z, a0hi.w};
          const uint32_t w1[8] = {a1lo.x, a1lo.y, a1lo.z, a1lo.w, a1hi.x, a1hi.y, a1hi.z, a1hi.w};
#pragma unroll
          for (int kt = 0; kt < KSTEPS; ++kt) {
            uint32_t a[4];
            a[0] = e4m3x2_to_f16x2(uint16_t(w0[kt] & 0xffff));
            a[1] = e4m3x2_to_f16x2(uint16_t(w1[kt] & 0xffff));
            a[2] = e4m3x2_to_f16x2(uint16_t(w0[kt] >> 16));
            a[3] = e4m3x2_to_f16x2(uint16_t(w1[kt] >> 16));
            mma(s[mt], a, qf[kt][0], qf[kt][1]);
          }
        }
      }
    }
    if constexpr (KV == KV_INT4) {
      // one 16-byte load gives a lane its 32 K nibbles of a row: word g holds
      // group g (k-steps 2g and 2g+1).  Per group, two MMAs start from minus
      // the decoding offset, and the group's K scale multiplies the result.
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        {  // all four m-tiles: nibbles always decode to finite values
          const int r0 = mt * 16 + r8, r1 = r0 + 8;
          const uint4 k0 = *reinterpret_cast<const uint4*>(Ks + r0 * 64 + q * 16);
          const uint4 k1 = *reinterpret_cast<const uint4*>(Ks + r1 * 64 + q * 16);
          const uint2 c0 = *reinterpret_cast<const uint2*>(Ks + kInt4Nibbles + r0 * 8);
          const uint2 c1 = *reinterpret_cast<const uint2*>(Ks + kInt4Nibbles + r1 * 8);
          const uint32_t w0[4] = {k0.x, k0.y, k0.z, k0.w}, w1[4] = {k1.x, k1.y, k1.z, k1.w};
          const float2 s0a = __half22float2(*reinterpret_cast<const __half2*>(&c0.x));
          const float2 s0b = __half22float2(*reinterpret_cast<const __half2*>(&c0.y));
          const float2 s1a = __half22float2(*reinterpret_cast<const __half2*>(&c1.x));
          const float2 s1b = __half22float2(*reinterpret_cast<const __half2*>(&c1.y));
          const float ks0[4] = {s0a.x, s0a.y, s0b.x, s0b.y}, ks1[4] = {s1a.x, s1a.y, s1b.x, s1b.y};
#pragma unroll
          for (int gq = 0; gq < 4; ++gq) {
            float t[4];
            uint32_t a[4];
            a[0] = lop3_and_or(w0[gq], nc.lo, nc.magic);
            a[1] = lop3_and_or(w1[gq], nc.lo, nc.magic);
            a[2] = lop3_and_or(w0[gq], nc.hi, nc.magic);
            a[3] = lop3_and_or(w1[gq], nc.hi, nc.magic);
            mma_f16_16816_c(t, a, qf[2 * gq][0], qf[2 * gq][1], cq[gq][0], cq[gq][1], cq[gq][0],
                            cq[gq][1]);
            const uint32_t x0 = w0[gq] >> 8, x1 = w1[gq] >> 8;
            a[0] = lop3_and_or(x0, nc.lo, nc.magic);
            a[1] = lop3_and_or(x1, nc.lo, nc.magic);
            a[2] = lop3_and_or(x0, nc.hi, nc.magic);
            a[3] = lop3_and_or(x1, nc.hi, nc.magic);
            mma_f16_16816(t, a, qf[2 * gq + 1][0], qf[2 * gq + 1][1]);
            s[mt][0] = fmaf(ks0[gq], t[0], s[mt][0]);
            s[mt][1] = fmaf(ks0[gq], t[1], s[mt][1]);
            s[mt][2] = fmaf(ks1[gq], t[2], s[mt][2]);
            s[mt][3] = fmaf(ks1[gq], t[3], s[mt][3]);
          }
        }
      }
    }
    // ---- scale, mask rows past `rows`, online softmax ----
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      const int r0 = mt * 16 + r8;
      const bool v0 = r0 < rows && r0 != hole, v1 = r0 + 8 < rows && r0 + 8 != hole;
      s[mt][0] = v0 ? s[mt][0] * scale : -INFINITY;
      s[mt][1] = v0 ? s[mt][1] * scale : -INFINITY;
      s[mt][2] = v1 ? s[mt][2] * scale : -INFINITY;
      s[mt][3] = v1 ? s[mt][3] * scale : -INFINITY;
      mx0 = fmaxf(mx0, fmaxf(s[mt][0], s[mt][2]));
      mx1 = fmaxf(mx1, fmaxf(s[mt][1], s[mt][3]));
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    const float mn0 = fmaxf(m[0], mx0), mn1 = fmaxf(m[1], mx1);
    const float al0 = fast_exp2(m[0] - mn0), al1 = fast_exp2(m[1] - mn1);
    m[0] = mn0;
    m[1] = mn1;
    l[0] *= al0;
    l[1] *= al1;
#pragma unroll
    for (int md = 0; md < MTD; ++md) {
      o[md][0] *= al0;
      o[md][1] *= al1;
      o[md][2] *= al0;
      o[md][3] *= al1;
    }
    if constexpr (KV == KV_INT4) {
#pragma unroll
      for (int gq = 0; gq < 4; ++gq) {
        eo[gq][0] *= al0;
        eo[gq][1] *= al1;
        eo[gq][2] *= al0;
        eo[gq][3] *= al1;
      }
    }
    uint32_t pb[4][2];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      const float p0 = fast_exp2(s[mt][0] - mn0), p1 = fast_exp2(s[mt][1] - mn1);
      const float p2 = fast_exp2(s[mt][2] - mn0), p3 = fast_exp2(s[mt][3] - mn1);
      l[0] += p0 + p2;
      l[1] += p1 + p3;
      if constexpr (KV == KV_FP8 || KV == KV_INT4) {
        pb[mt][0] = movmatrix_trans(pack_f16x2(p0, p1));
        pb[mt][1] = movmatrix_trans(pack_f16x2(p2, p3));
      } else {
        pb[mt][0] = movmatrix_trans(pack_bf16x2(p0, p1));
        pb[mt][1] = movmatrix_trans(pack_bf16x2(p2, p3));
      }
    }
    // ---- O^T += V^T P^T ----
    if constexpr (KV == KV_INT4) {
      // V^T tile [D][64 tokens] of nibbles.  Per group g of 32 V elements:
      // the group's V scales of the tokens multiply the probabilities, tokens
      // 8..15 of each 16-token m-tile (nibbles decoded as 1024 + 16 n) take a
      // further 1/16, and a constant-A MMA accumulates what the decoding adds
      // to each output row of the group (1032 or 1152 times each weight),
      // taken off when the state is written.  Token columns past `rows` hold
      // scale 0 (a 4-bit block's V tile is cleared when it is opened) and
      // probability 0, so every m-tile is computed.  One 8-byte load per
      // output row gives a lane its nibbles of all 64 tokens.
      const uint32_t kSixteenth = 0x2C002C00u;       // f16x2 (1/16, 1/16)
      const uint32_t ac[4] = {0x64086408u, 0x64086408u, 0x64806480u, 0x64806480u};  // 1032, 1152
#pragma unroll
      for (int gq = 0; gq < 4; ++gq) {
        uint32_t b[4][2];
#pragma unroll
        for (int mt = 0; mt < 4; ++mt) {
          const int t0 = mt * 16 + 2 * q;
          const uint32_t sA = *reinterpret_cast<const uint32_t*>(Vs + kInt4Nibbles + gq * 128 + t0 * 2);
          const uint32_t sB = *reinterpret_cast<const uint32_t*>(Vs + kInt4Nibbles + gq * 128 + (t0 + 8) * 2);
          b[mt][0] = hmul2_u32(pb[mt][0], sA);
          b[mt][1] = hmul2_u32(hmul2_u32(pb[mt][1], kSixteenth), sB);
          mma(eo[gq], ac, b[mt][0], b[mt][1]);
        }
#pragma unroll
        for (int md = 2 * gq; md < 2 * gq + 2; ++md) {
          const int d0 = md * 16 + r8;
          const uint2 x0 = *reinterpret_cast<const uint2*>(Vs + d0 * 32 + q * 8);
          const uint2 x1 = *reinterpret_cast<const uint2*>(Vs + (d0 + 8) * 32 + q * 8);
#pragma unroll
          for (int mt = 0; mt < 4; ++mt) {
            uint32_t w0 = (mt >> 1) ? x0.y : x0.x, w1 = (mt >> 1) ? x1.y : x1.x;
            if (mt & 1) {
              w0 >>= 8;
              w1 >>= 8;
            }
            uint32_t a[4];
            a[0] = lop3_and_or(w0, nc.lo, nc.magic);
            a[1] = lop3_and_or(w1, nc.lo, nc.magic);
            a[2] = lop3_and_or(w0, nc.hi, nc.magic);
            a[3] = lop3_and_or(w1, nc.hi, nc.magic);
            mma(o[md], a, b[mt][0], b[mt][1]);
          }
        }
      }
      return;
    }
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      if (mt * 16 >= rows) break;
      const bool partial = mt * 16 + 16 > rows;
      const int t0 = mt * 16 + 2 * q;
      const uint32_t m01 = (t0 < rows ? 0x0000ffffu : 0u) | (t0 + 1 < rows ? 0xffff0000u : 0u);
      const uint32_t m23 = (t0 + 8 < rows ? 0x0000ffffu : 0u) | (t0 + 9 < rows ? 0xffff0000u : 0u);
      if constexpr (KV == KV_BF16) {
        const uint32_t vbase = smem_u32(Vs);
        const int row = mt * 16 + (lane & 7) + ((lane >> 4) << 3);
#pragma unroll
        for (int md = 0; md < MTD; ++md) {
          const int ch = 2 * md + ((lane >> 3) & 1);
          uint32_t a[4];
          ldmatrix_x4_trans(a, vbase + row * T::ROWB + (swz_chunk(ch, row) << 4));
          if (partial) {
            a[0] &= m01;
            a[1] &= m01;
            a[2] &= m23;
            a[3] &= m23;
          }
          mma(o[md], a, pb[mt][0], pb[mt][1]);
        }
      } else {  // FP8: V^T tile [D][64], 16 bytes per (d row, owner lane)
#pragma unroll
        for (int md = 0; md < MTD; ++md) {
          const int d0 = md * 16 + r8;
          const uint4 x0 = *reinterpret_cast<const uint4*>(Vs + d0 * 64 + q * 16);
          const uint4 x1 = *reinterpret_cast<const uint4*>(Vs + (d0 + 8) * 64 + q * 16);
          const uint32_t w0 = mt == 0 ? x0.x : mt == 1 ? x0.y : mt == 2 ? x0.z : x0.w;
          const uint32_t w1 = mt == 0 ? x1.x : mt == 1 ? x1.y : mt == 2 ? x1.z : x1.w;
          uint32_t a[4];
          a[0] = e4m3x2_to_f16x2(uint16_t(w0 & 0xffff));
          a[1] = e4m3x2_to_f16x2(uint16_t(w1 & 0xffff));
          a[2] = e4m3x2_to_f16x2(uint16_t(w0 >> 16));
          a[3] = e4m3x2_to_f16x2(uint16_t(w1 >> 16));
          if (partial) {
            a[0] &= m01;
            a[1] &= m01;
            a[2] &= m23;
            a[3] &= m23;
          }
          mma(o[md], a, pb[mt][0], pb[mt][1]);
        }
      }
    }
  }

  // Write this warp's state for query heads n < g into the combine area.
  __device__ __forceinline__ void write_state(float* ow, float* mw, float* lw, int g, int lane) {
    if constexpr (KV == KV_INT4) {
#pragma unroll
      for (int md = 0; md < MTD; ++md) {
        o[md][0] -= eo[md >> 1][0];
        o[md][1] -= eo[md >> 1][1];
        o[md][2] -= eo[md >> 1][2];
        o[md][3] -= eo[md >> 1][3];
      }
    }
    float l0 = l[0], l1 = l[1];
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
    const int n0 = (lane & 3) * 2, r8 = lane >> 2;
#pragma unroll
    for (int md = 0; md < MTD; ++md) {
      const int d = md * 16 + r8;
      if (n0 < g) {
        ow[n0 * D + d] = o[md][0] * vscale;
        ow[n0 * D + d + 8] = o[md][2] * vscale;
      }
      if (n0 + 1 < g) {
        ow[(n0 + 1) * D + d] = o[md][1] * vscale;
        ow[(n0 + 1) * D + d + 8] = o[md][3] * vscale;
      }
    }
    if (r8 == 0) {
      if (n0 < g) {
        mw[n0] = m[0];
        lw[n0] = l0;
      }
      if (n0 + 1 < g) {
        mw[n0 + 1] = m[1];
        lw[n0 + 1] = l1;
      }
    }
  }
};

// ---------------------------------------------------------------------------
// fp32 path (CUDA-core FMA; exact fp32 arithmetic, no TF32)
// ---------------------------------------------------------------------------
template <int D>
struct F32Warp {
  static constexpr int DPL = D / 32;  // output elements per lane per query head
  using T = AttnTraits<KV_F32, D>;
  float m[8], l[8];
  float o[8][DPL];
  const float* qrow;  // stage query rows (set per unit)
  float scale, vscale;
  int g;

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      m[n] = -INFINITY;
      l[n] = 0.f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) o[n][e] = 0.f;
    }
  }
  __device__ __forceinline__ void load_q(const uint8_t*, int, int) {}

  __device__ __forceinline__ float kval(const uint8_t* tile, int r, int d) const {
    return reinterpret_cast<const float*>(tile + r * T::ROWB + (swz_chunk(d >> 2, r) << 4))[d & 3];
  }

  __device__ __forceinline__ void unit(const uint8_t* stage, int rows, int lane, int hole = -1) {
    const uint8_t* Ks = stage;
    const uint8_t* Vs = stage + T::TILEB;
    const float* qs = reinterpret_cast<const float*>(stage + 2 * T::TILEB);
    float s[2][8];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int r = lane + 32 * hh;
#pragma unroll
      for (int n = 0; n < 8; ++n) s[hh][n] = 0.f;
      if (r < rows) {
        for (int d = 0; d < D; ++d) {
          const float kd = kval(Ks, r, d);
#pragma unroll
          for (int n = 0; n < 8; ++n)
            if (n < g) s[hh][n] = fmaf(qs[n * D + d], kd, s[hh][n]);
        }
      }
#pragma unroll
      for (int n = 0; n < 8; ++n) s[hh][n] = r < rows && r != hole ? s[hh][n] * scale : -INFINITY;
    }
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      if (n >= g) continue;
      float mx = fmaxf(s[0][n], s[1][n]);
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float mn = fmaxf(m[n], mx);
      const float al = fast_exp2(m[n] - mn);
      m[n] = mn;
      s[0][n] = fast_exp2(s[0][n] - mn);
      s[1][n] = fast_exp2(s[1][n] - mn);
      float ps = s[0][n] + s[1][n];
      for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l[n] = l[n] * al + ps;
#pragma unroll
      for (int e = 0; e < DPL; ++e) o[n][e] *= al;
    }
    for (int r = 0; r < rows; ++r) {
      float pr[8];
#pragma unroll
      for (int n = 0; n < 8; ++n) pr[n] = __shfl_sync(0xffffffffu, s[r >> 5][n], r & 31);
#pragma unroll
      for (int e = 0; e < DPL; ++e) {
        const float vd = kval(Vs, r, lane + 32 * e);
#pragma unroll
        for (int n = 0; n < 8; ++n)
          if (n < g) o[n][e] = fmaf(pr[n], vd, o[n][e]);
      }
    }
  }

  __device__ __forceinline__ void write_state(float* ow, float* mw, float* lw, int gg, int lane) {
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      if (n >= gg) continue;
#pragma unroll
      for (int e = 0; e < DPL; ++e) ow[n * D + lane + 32 * e] = o[n][e] * vscale;
      if (lane == 0) {
        mw[n] = m[n];
        lw[n] = l[n];
      }
    }
  }
};

template <int KV, int D>
struct WarpSel {
  using type = MmaWarp<KV, D>;
};
template <int D>
struct WarpSel<KV_F32, D> {
  using type = F32Warp<D>;
};

}  // namespace dms
