// Pool creation, layout, reset and statistics for the compact DMS KV store.
//
// The store follows the FastDMS design of a compact KV store that reclaims
// the slots of physically evicted tokens, with per-layer, per-head variable
// token counts and partial block release ("FastDMS: vLLM BF16/FP8보다 빠른
// 6.4x KV cache 압축" (molayo1419.me), opening paragraphs and table "What's
// the catch?", row "PagedAttention / KV memory pool").  The pool is one
// caller-owned device buffer; this file only carves it and clears it.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>

#include "dms_internal.cuh"

namespace dms {

static thread_local std::string g_last_error;

void set_last_error(const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
}

dms_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return DMS_OK;
  set_last_error("%s: %s", what, cudaGetErrorString(e));
  return DMS_ERR_CUDA;
}

dms_status ensure_func_attr(const void* func, cudaFuncAttribute attr, int value,
                            FuncAttrCache& cache, const char* what) {
  int dev = -1;
  dms_status st = cuda_status(cudaGetDevice(&dev), "cudaGetDevice");
  if (st != DMS_OK) return st;
  const bool cached = dev >= 0 && dev < kAttrDevices;
  if (cached && cache.value[dev].load(std::memory_order_acquire) >= value) return DMS_OK;
  st = cuda_status(cudaFuncSetAttribute(func, attr, value), what);
  if (st != DMS_OK || !cached) return st;
  int old = cache.value[dev].load(std::memory_order_relaxed);
  while (old < value && !cache.value[dev].compare_exchange_weak(old, value, std::memory_order_release))
    ;
  return DMS_OK;
}

int device_sm_count(int device) {
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) return 0;
  return n;
}

static inline uint64_t align256(uint64_t x) { return (x + 255) & ~uint64_t(255); }

static int elem_bytes(int dt) { return dt == DMS_F32 ? 4 : dt == DMS_BF16 ? 2 : 1; }

// Validate a configuration and compute its layout.  Returns DMS_OK or
// DMS_ERR_INVALID_ARG / DMS_ERR_UNSUPPORTED with a message.
static dms_status plan_layout(const dms_pool_config* c, dms_pool_layout_t* lay) {
  if (!c || !lay) {
    set_last_error("null config");
    return DMS_ERR_INVALID_ARG;
  }
  if (c->n_layers < 1 || c->max_batch < 1 || c->n_kv_heads < 1 || c->n_q_heads < 1 ||
      c->window < 1 || c->max_blocks < 1 || c->max_context < 1) {
    set_last_error("config sizes must be positive");
    return DMS_ERR_INVALID_ARG;
  }
  if (c->n_q_heads % c->n_kv_heads != 0) {
    set_last_error("n_q_heads (%d) must be a multiple of n_kv_heads (%d)", c->n_q_heads,
                   c->n_kv_heads);
    return DMS_ERR_INVALID_ARG;
  }
  const int g = c->n_q_heads / c->n_kv_heads;
  if (g > 8) {
    set_last_error("GQA group %d > 8 is not built", g);
    return DMS_ERR_UNSUPPORTED;
  }
  if (c->kv_dtype != DMS_F32 && c->kv_dtype != DMS_BF16 && c->kv_dtype != DMS_FP8_E4M3 &&
      c->kv_dtype != DMS_INT4) {
    set_last_error("bad kv_dtype %d", c->kv_dtype);
    return DMS_ERR_INVALID_ARG;
  }
  if (c->head_dim != 64 && c->head_dim != 128) {
    set_last_error("head_dim %d not built (64, 128)", c->head_dim);
    return DMS_ERR_UNSUPPORTED;
  }
  if ((c->kv_dtype == DMS_FP8_E4M3 || c->kv_dtype == DMS_INT4) && c->head_dim != 128) {
    set_last_error("FP8 and 4-bit pools are built for head_dim 128 only");
    return DMS_ERR_UNSUPPORTED;
  }
  if (c->block_tokens != kBlockTokens) {
    set_last_error("block_tokens must be %d", kBlockTokens);
    return DMS_ERR_UNSUPPORTED;
  }
  if (c->max_blocks * kBlockTokens >= (int64_t(1) << 31) || c->max_context >= (int64_t(1) << 24)) {
    set_last_error("max_blocks * block_tokens must be < 2^31 and max_context < 2^24");
    return DMS_ERR_INVALID_ARG;
  }
  const int64_t n_heads = int64_t(c->n_layers) * c->max_batch * c->n_kv_heads;
  const int64_t mbh = (c->max_context + kBlockTokens - 1) / kBlockTokens;
  if (n_heads * mbh >= (int64_t(1) << 31) || n_heads * c->window >= (int64_t(1) << 31)) {
    set_last_error("pool tables exceed 2^31 entries");
    return DMS_ERR_INVALID_ARG;
  }
  const int64_t n_chunks = (c->max_context + kPrefillChunk - 1) / kPrefillChunk;
  // 4-bit rows: D/2 bytes of nibbles + one fp16 scale per 32 elements
  const int64_t row_bytes = c->kv_dtype == DMS_INT4 ? int64_t(c->head_dim) / 2 + c->head_dim / 16
                                                    : int64_t(c->head_dim) * elem_bytes(c->kv_dtype);

  memset(lay, 0, sizeof(*lay));
  uint64_t off = 0;
  lay->header = off;      off = align256(off + sizeof(DevHeader));
  lay->block_table = off; off = align256(off + uint64_t(n_heads) * mbh * 4);
  lay->n_slots = off;     off = align256(off + uint64_t(n_heads) * 4);
  lay->n_retained = off;  off = align256(off + uint64_t(n_heads) * 4);
  lay->ring = off;        off = align256(off + uint64_t(n_heads) * c->window * 4);
  lay->ring_row = off;    off = align256(off + uint64_t(n_heads) * c->window * 4);
  lay->last_block = off;  off = align256(off + uint64_t(n_heads) * 4);
  lay->free_top = off;    off = align256(off + uint64_t(n_heads) * 4);
  lay->free_stack = off;  off = align256(off + uint64_t(n_heads) * kFreeStackCap * 4);
  lay->block_stack = off; off = align256(off + uint64_t(c->max_blocks) * 4);
  lay->scales = off;      off = align256(off + uint64_t(c->n_layers) * c->n_kv_heads * 2 * 4);
  lay->tickets = off;     off = align256(off + uint64_t(n_heads) * 4);
  lay->scratch = off;
  off = align256(off + uint64_t(c->max_batch) * c->n_kv_heads * n_chunks * 4);  // chunk counts
  off = align256(off + uint64_t(2) * c->n_kv_heads * 4);                        // amax
  off = align256(off + uint64_t(c->max_batch + 1) * 4);                         // prefill tickets
  off = align256(off + uint64_t(c->max_batch) * c->n_kv_heads * 4);             // pair counts
  off = align256(off + (uint64_t(c->max_batch) * c->n_kv_heads + 1) * 4);       // pair bases
  if (c->kv_dtype == DMS_FP8_E4M3 || c->kv_dtype == DMS_INT4)                     // slot positions
    off = align256(off + uint64_t(c->max_batch) * c->n_kv_heads * mbh * kBlockTokens * 4);
  off = align256(off + sizeof(dms_pool_stats_t));                                // stats
  lay->blocks = off;
  lay->block_bytes = 2 * kBlockTokens * row_bytes;
  off += uint64_t(c->max_blocks) * lay->block_bytes;
  lay->total = align256(off);
  lay->row_bytes = row_bytes;
  lay->max_blocks_per_head = int32_t(mbh);
  lay->free_stack_cap = kFreeStackCap;
  lay->n_heads = int32_t(n_heads);
  lay->fp8_layout = c->kv_dtype == DMS_FP8_E4M3 ? 1 : c->kv_dtype == DMS_INT4 ? 2 : 0;
  return DMS_OK;
}

static PoolView make_view(const dms_pool_config& c, const dms_pool_layout_t& lay, void* base) {
  uint8_t* b = static_cast<uint8_t*>(base);
  PoolView v;
  memset(&v, 0, sizeof(v));
  v.L = c.n_layers;
  v.Bmax = c.max_batch;
  v.Hq = c.n_q_heads;
  v.Hkv = c.n_kv_heads;
  v.D = c.head_dim;
  v.w = c.window;
  v.BT = kBlockTokens;
  v.kv_dtype = c.kv_dtype;
  v.mbh = lay.max_blocks_per_head;
  v.free_cap = kFreeStackCap;
  v.n_heads = lay.n_heads;
  v.n_chunks_max = int32_t((c.max_context + kPrefillChunk - 1) / kPrefillChunk);
  v.max_blocks = c.max_blocks;
  v.wait_ns = kWaitLimitNs;
  v.row_bytes = lay.row_bytes;
  v.tile_bytes = kBlockTokens * lay.row_bytes;
  v.block_bytes = lay.block_bytes;
  v.blocks = b + lay.blocks;
  v.bt = reinterpret_cast<int32_t*>(b + lay.block_table);
  v.n_slots = reinterpret_cast<int32_t*>(b + lay.n_slots);
  v.n_retained = reinterpret_cast<int32_t*>(b + lay.n_retained);
  v.ring = reinterpret_cast<uint32_t*>(b + lay.ring);
  v.ring_row = reinterpret_cast<int32_t*>(b + lay.ring_row);
  v.last_block = reinterpret_cast<int32_t*>(b + lay.last_block);
  v.free_top = reinterpret_cast<int32_t*>(b + lay.free_top);
  v.free_stack = reinterpret_cast<int32_t*>(b + lay.free_stack);
  v.block_stack = reinterpret_cast<int32_t*>(b + lay.block_stack);
  v.scales = reinterpret_cast<float*>(b + lay.scales);
  v.tickets = reinterpret_cast<int32_t*>(b + lay.tickets);
  v.hdr = reinterpret_cast<DevHeader*>(b + lay.header);
  uint64_t s = lay.scratch;
  v.chunk_counts = reinterpret_cast<int32_t*>(b + s);
  s = align256(s + uint64_t(c.max_batch) * c.n_kv_heads * v.n_chunks_max * 4);
  v.amax = reinterpret_cast<uint32_t*>(b + s);
  s = align256(s + uint64_t(2) * c.n_kv_heads * 4);
  v.prefill_tickets = reinterpret_cast<int32_t*>(b + s);
  s = align256(s + uint64_t(c.max_batch + 1) * 4);
  v.pair_n = reinterpret_cast<int32_t*>(b + s);
  s = align256(s + uint64_t(c.max_batch) * c.n_kv_heads * 4);
  v.pair_base = reinterpret_cast<int32_t*>(b + s);
  s = align256(s + (uint64_t(c.max_batch) * c.n_kv_heads + 1) * 4);
  v.pos_of_slot = nullptr;
  if (c.kv_dtype == DMS_FP8_E4M3 || c.kv_dtype == DMS_INT4) {
    v.pos_of_slot = reinterpret_cast<int32_t*>(b + s);
    s = align256(s + uint64_t(c.max_batch) * c.n_kv_heads * uint64_t(lay.max_blocks_per_head) * kBlockTokens * 4);
  }
  v.stats = b + s;
  return v;
}

__global__ void init_header_kernel(DevHeader* hdr) {
  hdr->next_block = 0;
  hdr->block_stack_top = 0;
  hdr->error = 0;
  hdr->err_layer = -1;
  hdr->err_seq = -1;
  hdr->err_head = -1;
  hdr->prefill_go = 0;
}

static dms_status clear_pool(dms_pool* p, cudaStream_t stream) {
  // every bookkeeping region lies before the block region
  dms_status st = cuda_status(cudaMemsetAsync(p->base, 0, p->layout.blocks, stream), "clear pool");
  if (st != DMS_OK) return st;
  init_header_kernel<<<1, 1, 0, stream>>>(p->view.hdr);
  return cuda_status(cudaGetLastError(), "init_header_kernel");
}

// One CTA reduces the per-head counters into the staging dms_pool_stats_t.
__global__ void __launch_bounds__(1024) stats_kernel(PoolView v) {
  __shared__ long long s_ret[32], s_slots[32];
  __shared__ int s_min[32], s_max[32], s_ne[32];
  long long ret = 0, slots = 0;
  int mn = 0x7fffffff, mx = 0, ne = 0;
  for (int i = threadIdx.x; i < v.n_heads; i += blockDim.x) {
    const int r = v.n_retained[i];
    ret += r;
    slots += v.n_slots[i];
    if (r > 0) {
      mn = min(mn, r);
      mx = max(mx, r);
      ne += 1;
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    ret += __shfl_xor_sync(0xffffffffu, ret, o);
    slots += __shfl_xor_sync(0xffffffffu, slots, o);
    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    ne += __shfl_xor_sync(0xffffffffu, ne, o);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    s_ret[warp] = ret;
    s_slots[warp] = slots;
    s_min[warp] = mn;
    s_max[warp] = mx;
    s_ne[warp] = ne;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int nw = blockDim.x >> 5;
    for (int k = 1; k < nw; ++k) {
      ret += s_ret[k];
      slots += s_slots[k];
      mn = min(mn, s_min[k]);
      mx = max(mx, s_max[k]);
      ne += s_ne[k];
    }
    dms_pool_stats_t* o = static_cast<dms_pool_stats_t*>(v.stats);
    o->retained_tokens = ret;
    o->slots_in_use = slots;
    o->min_retained = ne ? mn : 0;
    o->max_retained = mx;
    o->heads_nonempty = ne;
    o->pad0 = 0;
    // an exhausted decode step may have bumped the counter past the pool
    const int64_t handed = v.hdr->next_block < v.max_blocks ? v.hdr->next_block : v.max_blocks;
    o->blocks_in_use = handed - v.hdr->block_stack_top;
    o->blocks_total = v.max_blocks;
    o->kv_bytes_in_use = o->blocks_in_use * v.block_bytes;
    o->kv_bytes_retained = ret * 2 * v.row_bytes;
    o->error_flags = v.hdr->error;
    o->error_layer = v.hdr->err_layer;
    o->error_seq = v.hdr->err_seq;
    o->error_head = v.hdr->err_head;
  }
}

}  // namespace dms

using namespace dms;

extern "C" {

const char* dms_status_string(dms_status s) {
  switch (s) {
    case DMS_OK: return "DMS_OK";
    case DMS_ERR_INVALID_ARG: return "DMS_ERR_INVALID_ARG";
    case DMS_ERR_CAPACITY: return "DMS_ERR_CAPACITY";
    case DMS_ERR_CUDA: return "DMS_ERR_CUDA";
    case DMS_ERR_UNSUPPORTED: return "DMS_ERR_UNSUPPORTED";
    case DMS_ERR_DEVICE: return "DMS_ERR_DEVICE";
  }
  return "DMS_ERR_UNKNOWN";
}

const char* dms_last_error(void) { return g_last_error.c_str(); }

dms_status dms_pool_bytes_required(const dms_pool_config* cfg, size_t* bytes) {
  if (!bytes) {
    set_last_error("null output");
    return DMS_ERR_INVALID_ARG;
  }
  dms_pool_layout_t lay;
  dms_status st = plan_layout(cfg, &lay);
  if (st != DMS_OK) return st;
  *bytes = lay.total;
  return DMS_OK;
}

dms_status dms_pool_create(const dms_pool_config* cfg, void* dev_buf, size_t bytes,
                           cudaStream_t stream, dms_pool** out) {
  if (!out || !dev_buf) {
    set_last_error("null buffer or output handle");
    return DMS_ERR_INVALID_ARG;
  }
  *out = nullptr;
  if (reinterpret_cast<uintptr_t>(dev_buf) & 255) {
    set_last_error("pool buffer must be 256-byte aligned");
    return DMS_ERR_INVALID_ARG;
  }
  dms_pool_layout_t lay;
  dms_status st = plan_layout(cfg, &lay);
  if (st != DMS_OK) return st;
  if (bytes < lay.total) {
    set_last_error("pool buffer has %zu bytes, config needs %llu", bytes,
                   (unsigned long long)lay.total);
    return DMS_ERR_CAPACITY;
  }
  int dev = 0;
  st = cuda_status(cudaGetDevice(&dev), "cudaGetDevice");
  if (st != DMS_OK) return st;
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, dev_buf) != cudaSuccess ||
      attr.type != cudaMemoryTypeDevice) {
    cudaGetLastError();
    set_last_error("pool buffer is not device memory");
    return DMS_ERR_INVALID_ARG;
  }
  dms_pool* p = new (std::nothrow) dms_pool;
  if (!p) {
    set_last_error("host handle allocation failed");
    return DMS_ERR_CAPACITY;
  }
  p->cfg = *cfg;
  p->layout = lay;
  p->base = dev_buf;
  p->bytes = bytes;
  p->device = dev;
  p->sm_count = device_sm_count(dev);
  p->attn_kernel = DMS_ATTN_AUTO;
  p->prefill_mode = DMS_PREFILL_SPARSE;
  p->view = make_view(*cfg, lay, dev_buf);
  st = clear_pool(p, stream);
  if (st != DMS_OK) {
    delete p;
    return st;
  }
  *out = p;
  return DMS_OK;
}

dms_status dms_pool_destroy(dms_pool* pool) {
  delete pool;
  return DMS_OK;
}

dms_status dms_pool_reset(dms_pool* pool, cudaStream_t stream) {
  if (!pool) {
    set_last_error("null pool");
    return DMS_ERR_INVALID_ARG;
  }
  return clear_pool(pool, stream);
}

dms_status dms_pool_set_wait_limit(dms_pool* pool, uint64_t limit_ns) {
  if (!pool || limit_ns < 1000 || limit_ns > 60000000000ull) {
    set_last_error("wait limit must be between 1 us and 60 s (got %llu ns)",
                   (unsigned long long)limit_ns);
    return DMS_ERR_INVALID_ARG;
  }
  pool->view.wait_ns = limit_ns;
  return DMS_OK;
}

dms_status dms_pool_set_attn_kernel(dms_pool* pool, int kind) {
  if (!pool || kind < DMS_ATTN_AUTO || kind > DMS_ATTN_CLUSTER) {
    set_last_error("null pool or unknown attention kernel %d", kind);
    return DMS_ERR_INVALID_ARG;
  }
  pool->attn_kernel = kind;
  return DMS_OK;
}

dms_status dms_pool_set_prefill_mode(dms_pool* pool, int mode) {
  if (!pool || (mode != DMS_PREFILL_SPARSE && mode != DMS_PREFILL_DENSE)) {
    set_last_error("null pool or unknown prefill mode %d", mode);
    return DMS_ERR_INVALID_ARG;
  }
  pool->prefill_mode = mode;
  return DMS_OK;
}

dms_status dms_pool_layout(const dms_pool* pool, dms_pool_layout_t* out) {
  if (!pool || !out) {
    set_last_error("null pool or output");
    return DMS_ERR_INVALID_ARG;
  }
  *out = pool->layout;
  return DMS_OK;
}

dms_status dms_pool_stats(dms_pool* pool, dms_pool_stats_t* out, cudaStream_t stream) {
  if (!pool || !out) {
    set_last_error("null pool or output");
    return DMS_ERR_INVALID_ARG;
  }
  stats_kernel<<<1, 1024, 0, stream>>>(pool->view);
  dms_status st = cuda_status(cudaGetLastError(), "stats_kernel");
  if (st != DMS_OK) return st;
  st = cuda_status(cudaMemcpyAsync(out, pool->view.stats, sizeof(*out), cudaMemcpyDeviceToHost,
                                   stream),
                   "stats copy");
  if (st != DMS_OK) return st;
  st = cuda_status(cudaStreamSynchronize(stream), "stats sync");
  if (st != DMS_OK) return st;
  if (out->error_flags != 0) {
    set_last_error("device error word 0x%x (layer %d seq %d head %d)", out->error_flags,
                   out->error_layer, out->error_seq, out->error_head);
    return DMS_ERR_DEVICE;
  }
  return DMS_OK;
}

}  // extern "C"
