// Internal definitions shared by the libdms CUDA sources (not installed).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include <atomic>
#include <utility>

#include "dms.h"

namespace dms {

constexpr int kBlockTokens = 64;     // BT: rows per physical block
constexpr int kFreeStackCap = 4;     // per-head free slots awaiting reuse
constexpr int kPrefillChunk = 256;   // prompt tokens per compaction CTA
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // default limit of every device wait: 1 s

// Device-side header at the start of the pool buffer.
struct DevHeader {
  int32_t next_block;       // bump pointer into the block region
  int32_t block_stack_top;  // entries on the global free-block stack
  uint32_t error;           // DMS_DEVERR_* bits
  int32_t err_layer;        // first failing head, -1 when none
  int32_t err_seq;
  int32_t err_head;
  int32_t prefill_go;       // set by the prefill planner when the layer may be written
  int32_t pad;
};

// Everything a kernel needs to address the pool; passed by value.
struct PoolView {
  int32_t L, Bmax, Hq, Hkv, D, w, BT, kv_dtype;
  int32_t mbh;              // block table width (max blocks per head)
  int32_t free_cap;
  int32_t n_heads;
  int32_t n_chunks_max;     // prefill scratch: chunks per (b, h)
  int64_t max_blocks;
  uint64_t wait_ns;         // limit of every bounded device wait (dms_pool_set_wait_limit)
  int64_t row_bytes;        // D * elem size
  int64_t tile_bytes;       // BT * row_bytes
  int64_t block_bytes;      // 2 * tile_bytes
  uint8_t* blocks;
  int32_t* bt;
  int32_t* n_slots;
  int32_t* n_retained;
  uint32_t* ring;           // [n_heads][w] slot | flag << 31
  int32_t* ring_row;        // [n_heads][w] physical row (block * BT + row) of that slot
  int32_t* last_block;      // [n_heads] block of slot n_slots - 1 (-1 when empty)
  int32_t* free_top;
  int32_t* free_stack;
  int32_t* block_stack;
  float* scales;            // [L][Hkv][2] (K, V)
  int32_t* tickets;         // [n_heads] split-K merge tickets (self-resetting)
  DevHeader* hdr;
  int32_t* chunk_counts;    // prefill scratch [Bmax][Hkv][n_chunks_max]
  uint32_t* amax;           // prefill scratch [2][Hkv] (float bits, non-negative; left zeroed)
  int32_t* prefill_tickets; // prefill scratch [Bmax + 1] arrival counters (self-resetting)
  int32_t* pair_n;          // prefill scratch [Bmax][Hkv] kept tokens of each (sequence, head)
  int32_t* pair_base;       // prefill scratch [Bmax * Hkv + 1] first allocation index of each pair
  int32_t* pos_of_slot;     // prefill scratch, FP8 and 4-bit stores only (else null):
                            // [Bmax][Hkv][mbh * BT] prompt position of each kept slot
  void* stats;              // staging for dms_pool_stats

  __host__ __device__ __forceinline__ int head(int l, int b, int h) const {
    return (l * Bmax + b) * Hkv + h;
  }
};

// ------------------------------------------------------------------------
// error word
// ------------------------------------------------------------------------
__device__ __forceinline__ void report_error(DevHeader* hdr, uint32_t bit, int l, int b, int h) {
  atomicOr(&hdr->error, bit);
  if (atomicCAS(&hdr->err_layer, -1, l) == -1) {
    hdr->err_seq = b;
    hdr->err_head = h;
  }
}

// Bounds checks of DMS_DEBUG builds: a failed check records DMS_DEVERR_BOUNDS
// with (site, a, b) in the error fields and evaluates to false, so the caller
// skips the access.  Release builds compile the check away.
#ifdef DMS_DEBUG
#define DMS_CHECK(cond, hdr, site, a, b) \
  ((cond) ? true : (report_error((hdr), DMS_DEVERR_BOUNDS, (site), int(a), int(b)), false))
#else
#define DMS_CHECK(cond, hdr, site, a, b) true
#endif

// ------------------------------------------------------------------------
// stored-row layout
// ------------------------------------------------------------------------
// bf16 / fp32 rows: 16-byte chunk c of row r lives at chunk c ^ (r & 7).
__host__ __device__ __forceinline__ int swz_chunk(int c, int r) { return c ^ (r & 7); }

// FP8 K rows (D = 128): logical element d of row r is stored at byte
//   chunk' * 16 + (pos & 15),  pos = owner * 32 + kt * 4 + hi * 2 + lo,
//   owner = (d & 7) >> 1, kt = d >> 4, hi = (d >> 3) & 1, lo = d & 1,
//   chunk' = (pos >> 4) ^ (r & 7)
// so that lane (r, owner) of an m16n8k16 A fragment reads its 32 values as
// two conflict-free 16-byte loads.
__host__ __device__ __forceinline__ int fp8k_pos(int d) {
  return (((d & 7) >> 1) << 5) | ((d >> 4) << 2) | (((d >> 3) & 1) << 1) | (d & 1);
}
__host__ __device__ __forceinline__ int fp8k_byte(int r, int d) {
  const int pos = fp8k_pos(d);
  return r * 128 + ((((pos >> 4) ^ (r & 7)) << 4) | (pos & 15));
}
// FP8 V tiles are stored transposed, [D][BT]: token row r of element d sits
// at byte d * 64 + owner * 16 + kt * 4 + hi * 2 + lo with the same split of
// the token index r (owner = (r & 7) >> 1, kt = r >> 4, hi = (r >> 3) & 1).
__host__ __device__ __forceinline__ int fp8v_byte(int r, int d) {
  return d * 64 + ((((r & 7) >> 1) << 4) | ((r >> 4) << 2) | (((r >> 3) & 1) << 1) | (r & 1));
}

// 4-bit rows (head_dim 128): see DMS_INT4 in dms.h.  Byte offset of the
// 32-bit word holding element d of K row r, and the bit of its nibble;
// the same for token t of V element row d; scale offsets in a tile.
constexpr int kInt4Nibbles = 4096;  // nibble bytes of a tile; scales follow
__host__ __device__ __forceinline__ int int4k_word(int r, int d) {
  return r * 64 + (((d & 7) >> 1) << 4) + ((d >> 5) << 2);
}
__host__ __device__ __forceinline__ int int4k_shift(int d) {
  return 8 * ((d >> 4) & 1) + 4 * ((d >> 3) & 1) + 16 * (d & 1);
}
__host__ __device__ __forceinline__ int int4v_word(int d, int t) {
  return d * 32 + (((t & 7) >> 1) << 3) + ((t >> 5) << 2);
}
__host__ __device__ __forceinline__ int int4v_shift(int t) {
  return 8 * ((t >> 4) & 1) + 4 * ((t >> 3) & 1) + 16 * (t & 1);
}
__host__ __device__ __forceinline__ int int4k_scale(int r, int j) { return kInt4Nibbles + r * 8 + j * 2; }
__host__ __device__ __forceinline__ int int4v_scale(int t, int j) { return kInt4Nibbles + j * 128 + t * 2; }

// ------------------------------------------------------------------------
// PTX wrappers
// ------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait that may suspend the thread until the phase completes, for at
// most hint_ns (a waiting warp then takes no issue slots from the warps
// that work); it returns early when the phase completes.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Wait for the phase of `parity` to complete; gives up after limit_ns or
// when *abort becomes non-zero (checked at least every 0.1 ms).  Returns
// false when it gave up.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_suspend(bar, parity, 100000u)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// Step counters shared with copy streams (the stepper): the copy streams
// write and wait on them with stream memory operations, the kernels wait on
// and publish them, so that the compute stream holds nothing but kernels.
// A null pointer means no such condition.
struct StepSync {
  const int32_t* ready;    // append: inputs of this step landed once *ready >= ready_value
  int32_t ready_value;
  const int32_t* drained;  // attention: the output buffer's previous copy-out is done once
  int32_t drained_value;   //            *drained >= drained_value
  int32_t* done;           // attention: the last CTA to leave stores done_value
  int32_t done_value;
  int32_t* exit_count;     // attention: CTAs that left (the last one resets it)
};

__device__ __forceinline__ int32_t ld_acquire_gpu(const int32_t* p) {
  int32_t v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(int32_t* p, int32_t v) {
  asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Wait (one thread) until *p >= v; false after limit_ns.
__device__ __forceinline__ bool wait_counter_geq(const int32_t* p, int32_t v, uint64_t limit_ns) {
  if (ld_acquire_gpu(p) >= v) return true;
  const uint64_t t0 = globaltimer_ns();
  while (ld_acquire_gpu(p) < v) {
    if (globaltimer_ns() - t0 > limit_ns) return false;
    __nanosleep(200);
  }
  return true;
}

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy (TMA) accesses.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 1-D bulk copy global -> shared (TMA), completion counted on `bar`.
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gsrc, uint32_t bytes,
                                         uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// D += A(16x16, row) * B(16x8, col), bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Same shape with f16 inputs (the FP8 path decodes E4M3 to f16 exactly).
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D = A * B + C with C in registers of its own (f16 inputs).
__device__ __forceinline__ void mma_f16_16816_c(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                                uint32_t b1, float c0, float c1, float c2, float c3) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c0), "f"(c1), "f"(c2),
        "f"(c3));
}

// Programmatic dependent launch: let the next kernel of the stream be
// scheduled now / wait until every kernel this one depends on has finished
// and its writes are visible.  Both are no-ops without the launch attribute.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait_prerequisites() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Bring `bytes` (a multiple of 16) from p into L2, asynchronously (TMA bulk
// prefetch: no register written, nothing waits).
__device__ __forceinline__ void bulk_prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Bring the line holding p into L2 (no register written, nothing waits).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// 2^x with the hardware approximation (max rel. error ~2^-22).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Two E4M3 bytes (low byte = first element) -> f16x2, exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t x) {
  uint32_t y;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(y) : "h"(x));
  return y;
}

// E4M3 code of an fp32 value: round to nearest even, saturating to +-448.
__device__ __forceinline__ uint8_t f32_to_e4m3(float x) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}

// ------------------------------------------------------------------------
// host helpers
// ------------------------------------------------------------------------
void set_last_error(const char* fmt, ...);
// Launch with programmatic stream serialisation (PDL) allowed.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
dms_status cuda_status(cudaError_t e, const char* what);
int device_sm_count(int device);
// A kernel attribute (cudaFuncSetAttribute) takes effect on the current
// device only, so it is set once per device: the cache remembers, per
// device ordinal, the largest value set so far (a static object, zeroed at
// load).  Two threads making their first call at once both set it, which is
// harmless.  Devices past the table are set on every call.
constexpr int kAttrDevices = 64;
struct FuncAttrCache {
  std::atomic<int> value[kAttrDevices];
};
dms_status ensure_func_attr(const void* func, cudaFuncAttribute attr, int value,
                            FuncAttrCache& cache, const char* what);
}  // namespace dms
struct dms_pool;
namespace dms {
dms_status prefill_plan_launch(dms_pool* pool, int layer, int seq0, int batch, int prompt_len,
                               const uint8_t* evict, cudaStream_t stream);
// prefill compaction of a copy store (bf16 / fp32) in one launch (csrc/prefill_cluster.cu),
// for prompts of up to prefill_cluster_max_prompt() tokens
int prefill_cluster_max_prompt();
dms_status prefill_cluster_launch(dms_pool* pool, int layer, int seq0, int batch, int prompt_len,
                                  const void* k, const void* v, dms_dtype in_dtype, const uint8_t* evict,
                                  cudaStream_t stream);

}  // namespace dms

// The opaque host handle.
struct dms_pool {
  dms_pool_config cfg;
  dms_pool_layout_t layout;
  dms::PoolView view;
  void* base;
  size_t bytes;
  int device;
  int sm_count;
  int attn_kernel;  // DMS_ATTN_* (dms_pool_set_attn_kernel)
  int prefill_mode; // DMS_PREFILL_* (dms_pool_set_prefill_mode)
};

namespace dms {
// stepper launches with step counters (csrc/append.cu, csrc/attn.cu)
dms_status append_layers_synced(dms_pool* pool, int layer0, int n_layers, int batch, int64_t pos,
                                const void* k, const void* v, dms_dtype in_dtype,
                                const uint8_t* evict, cudaStream_t stream, const StepSync& sync);
dms_status decode_attn_layers_synced(dms_pool* pool, int layer0, int n_layers, int batch,
                                     const void* q, void* out, float sm_scale, void* ws,
                                     cudaStream_t stream, const StepSync& sync);
// one cluster per head for calls with few heads (csrc/step.cu): attention
// only when knew is null, else the fused decode step; *done = false when
// the call has too many heads for every cluster of two or more CTAs to be
// resident at once (force: launch with clusters of one CTA then)
dms_status cluster_attn(dms_pool* pool, int layer0, int n_layers, int batch, const void* q, void* out,
                        float sm_scale, const void* knew, const void* vnew, dms_dtype in_dtype,
                        const uint8_t* evict, int64_t pos, bool force, cudaStream_t stream,
                        bool* done);
}  // namespace dms
