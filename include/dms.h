/*
 * dms.h -- C ABI of libdms: compact-KV decode for Dynamic Memory
 * Sparsification (DMS) on NVIDIA B200 (sm_100a).
 *
 * What the library computes
 * -------------------------
 * DMS learns, per attention head, which tokens to evict, and evicts them
 * with a delay: a token flagged for eviction stays visible for a window of w
 * tokens and is removed afterwards ("NVIDIA veröffentlicht Qwen3-8B-DMS-8x
 * mit innovativer Speicherkompression für verbesserte Inferenzzeiten"
 * (mindverse), section "Dynamic Memory Sparsification (DMS): Eine innovative
 * Lösung", w = 512; "Nvidia DMS: сжатие памяти LLM в 8 раз" (stiva.ai),
 * section "Ключевое изобретение: delayed eviction").  For the query at
 * position t, key j of kv-head h is visible unless evict[j,h] and t-j >= w.
 * FastDMS stores only the visible tokens in a compact KV store that reclaims
 * the slots of evicted tokens ("FastDMS: vLLM BF16/FP8보다 빠른 6.4x KV
 * cache 압축" (molayo1419.me), opening paragraphs), with per-layer,
 * per-head variable token counts instead of fixed pages (same page, table
 * "What's the catch?", row "PagedAttention / KV memory pool").
 *
 * The pool
 * --------
 * One caller-provided device buffer holds every (layer, sequence, kv-head)
 * "head" of the store:
 *   - physical blocks of BT = block_tokens token rows; block = [K tile
 *     BT x D][V tile BT x D] in the pool's kv dtype.  A row of bf16/fp32 is
 *     stored with its 16-byte chunks permuted: chunk c of row r sits at
 *     chunk c ^ (r & 7) (the shared-memory image the attention kernel
 *     reads, conflict free).  The FP8 layout is given in dms_pool_layout_t.
 *   - per head: a block table (logical slot s lives in block
 *     table[s / BT], row s % BT), n_slots (slots ever handed out),
 *     n_retained (tokens held), a window ring of w entries
 *     (slot | flag << 31 for the last w positions; entry t mod w holds
 *     token t) with a parallel ring of physical rows (block * BT + row),
 *     the block of the head's last slot, and a LIFO free-slot stack;
 *   - a global free-block stack and bump counter, FP8 scales, an error word.
 * Slots of one head are dense: a retired slot is reused by the same step's
 * new token, so the held tokens are exactly slots [0, n_slots).
 *
 * Conventions
 * -----------
 * - Ownership: the caller allocates every device buffer (pool, inputs,
 *   outputs, workspace) and owns every stream.  libdms never allocates
 *   device memory; a dms_pool is a small host handle.
 * - Asynchrony: every call enqueues its kernels on the given stream and
 *   returns; argument errors are reported at once, device-side errors
 *   (pool exhausted, table overflow, a wait that timed out) set bits of the
 *   pool's error word, read back by dms_pool_stats.  No kernel traps or
 *   waits without a time limit.
 * - Calls on one pool must be ordered (one stream, or events between
 *   streams): compaction, append, release and the fused projection share
 *   the pool's block counters and the planner's scratch, whatever layer
 *   they touch.  Pointers are device pointers unless marked host.
 * - Layouts are row-major, C order.  B = batch (sequences 0..B-1 of the
 *   pool, B <= max_batch), P = prompt length, Hq / Hkv query / kv heads,
 *   g = Hq / Hkv (query head hq reads kv head hq / g), D = head_dim.
 */
#ifndef DMS_H
#define DMS_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DMS_OK = 0,
  DMS_ERR_INVALID_ARG = 1,   /* bad pointer, size, dtype, layer range ... */
  DMS_ERR_CAPACITY = 2,      /* buffer too small for the requested pool    */
  DMS_ERR_CUDA = 3,          /* a CUDA runtime call failed                 */
  DMS_ERR_UNSUPPORTED = 4,   /* valid but not built (e.g. head_dim 96)     */
  DMS_ERR_DEVICE = 5         /* the pool's device error word is non-zero   */
} dms_status;

typedef enum { DMS_F32 = 0, DMS_BF16 = 1, DMS_FP8_E4M3 = 2, DMS_INT4 = 3 } dms_dtype;

/* Bits of the device error word (dms_pool_stats_t.error_flags). */
#define DMS_DEVERR_BLOCKS_EXHAUSTED 0x1u  /* global block pool ran out; write skipped   */
#define DMS_DEVERR_HEAD_TABLE_FULL  0x2u  /* a head outgrew max_context; write skipped   */
#define DMS_DEVERR_FREE_STACK_FULL  0x4u  /* per-head free stack overflow                */
#define DMS_DEVERR_TIMEOUT          0x8u  /* a bounded wait gave up; outputs invalid     */
#define DMS_DEVERR_LAYER_NOT_EMPTY  0x10u /* prefill into a layer that already holds data */
#define DMS_DEVERR_BOUNDS           0x20u /* DMS_DEBUG builds: an index failed its check  */
#define DMS_DEVERR_BAD_SEQUENCE     0x40u /* a device sequence id or position out of range; that head skipped */

typedef struct {
  int32_t n_layers;
  int32_t max_batch;
  int32_t n_q_heads;
  int32_t n_kv_heads;
  int32_t head_dim;       /* 64 or 128 */
  int32_t window;         /* delay window w >= 1 (512 in the pages)        */
  int32_t block_tokens;   /* BT; 64 is the only value built                */
  int32_t kv_dtype;       /* dms_dtype of the stored K/V                    */
  int64_t max_blocks;     /* physical blocks shared by all heads            */
  int64_t max_context;    /* most tokens one head may hold (table width)    */
} dms_pool_config;

typedef struct dms_pool dms_pool;  /* opaque host handle */

/* Byte offsets of each region inside the pool buffer, for inspection by
 * tests and tools (the pool is plain device memory). */
typedef struct {
  uint64_t header, blocks, block_table, n_slots, n_retained, ring, ring_row, last_block,
           free_top, free_stack, block_stack, scales, tickets, scratch, total;
  int64_t block_bytes;          /* bytes of one block (K tile + V tile)      */
  int64_t row_bytes;            /* bytes of one stored row (D * elem size)   */
  int32_t max_blocks_per_head;  /* block table width                         */
  int32_t free_stack_cap;       /* per-head free stack capacity              */
  int32_t n_heads;              /* n_layers * max_batch * n_kv_heads         */
  int32_t fp8_layout;           /* 1: FP8 rows use the permuted layout below; 2: 4-bit rows (below) */
} dms_pool_layout_t;

/* DMS_INT4 pools (head_dim 128 only): a stored row is 128 signed 4-bit codes
 * q in [-7, 7], kept as the nibble q + 8, with one fp16 scale per group of 32
 * elements (scale = fp16(amax / 7), q = rint(x / scale); the stored value is
 * q * scale).  row_bytes = 72 (64 bytes of nibbles + 4 scales).  A block is
 *   K tile: [64 rows x 64 B nibbles][64 rows x 4 fp16 scales]
 *   V tile: [128 element rows x 32 B nibbles, token-major][4 groups x 64 tokens fp16 scales]
 * Nibble placement (the attention kernel's MMA fragments come out of one
 * 16-byte load per row): element d of K row r lies in the 32-bit word at
 * byte r*64 + q*16 + (kt>>1)*4 with q = (d&7)>>1, kt = d>>4, at bit
 * 8*(kt&1) + 4*((d>>3)&1) + 16*(d&1); token t of V element row d lies in
 * the word at byte d*32 + q*8 + (m>>1)*4 with q = (t&7)>>1, m = t>>4, at bit
 * 8*(m&1) + 4*((t>>3)&1) + 16*(t&1).  Scale of K row r, group j: byte
 * 4096 + r*8 + j*2; of V token t, group j: byte 4096 + j*128 + t*2.
 * Decode attention on a 4-bit pool multiplies each code by its scale in
 * fp16 and runs the dot products on fp16 operands with fp32 accumulation
 * (the query is rounded to fp16 too), so stored values and queries must
 * stay within the fp16 range (|x| <= 65504).
 * Source: the pages pair token eviction with lower-bit KV (FastDMS page,
 * paragraph after the speed table, and its comparison with 4-bit KV) but
 * give no 4-bit format; the symmetric per-group format above is the plain
 * reading. */

typedef struct {
  int64_t retained_tokens;      /* sum of n_retained over all heads           */
  int64_t slots_in_use;         /* sum of n_slots                             */
  int32_t min_retained;         /* over heads with n_retained > 0             */
  int32_t max_retained;
  int32_t heads_nonempty;
  int32_t pad0;
  int64_t blocks_in_use;        /* handed out and not returned                */
  int64_t blocks_total;
  int64_t kv_bytes_in_use;      /* blocks_in_use * block_bytes                */
  int64_t kv_bytes_retained;    /* retained_tokens * 2 * row_bytes            */
  uint32_t error_flags;         /* DMS_DEVERR_* bits                          */
  int32_t error_layer;          /* first failing head (or -1)                 */
  int32_t error_seq;
  int32_t error_head;
} dms_pool_stats_t;

/* Human-readable name of a status code (static string). */
const char* dms_status_string(dms_status s);

/* Last host-side error message of the calling thread ("" if none). */
const char* dms_last_error(void);

/* Bytes of device memory a pool with this configuration needs.  Pure host
 * computation.  Returns DMS_ERR_INVALID_ARG for an invalid config. */
dms_status dms_pool_bytes_required(const dms_pool_config* cfg, size_t* bytes);

/* Carve a pool out of dev_buf (caller-owned, >= bytes_required, 256-byte
 * aligned) and clear its bookkeeping on `stream`.  *out receives a host
 * handle that must be released with dms_pool_destroy.  The device must be
 * current.  Source: compact store with slot reclaim and per-head ragged
 * counts (FastDMS page, opening paragraphs and table "What's the catch?"). */
dms_status dms_pool_create(const dms_pool_config* cfg, void* dev_buf, size_t bytes,
                           cudaStream_t stream, dms_pool** out);

/* Free the host handle only (the buffer stays the caller's). */
dms_status dms_pool_destroy(dms_pool* pool);

/* Clear every head, the block stack and the error word (async on stream). */
dms_status dms_pool_reset(dms_pool* pool, cudaStream_t stream);

/* Limit of every bounded wait in the kernels launched on this pool from now
 * on (default 1 s; 1 us .. 60 s, else DMS_ERR_INVALID_ARG).  A wait that
 * runs out sets DMS_DEVERR_TIMEOUT in the error word and its kernel returns
 * (no kernel waits without a limit).  The waits are the stepper's step
 * counters and the attention kernels' copy barriers; a shorter limit makes a
 * stalled producer (a copy that never lands, a signal that never comes)
 * surface sooner.  Host-side setting of the handle: not stream-ordered. */
dms_status dms_pool_set_wait_limit(dms_pool* pool, uint64_t limit_ns);

/* Which kernel decode attention uses (host setting of the handle, applied to
 * calls made after it):
 *   DMS_ATTN_AUTO      one thread-block cluster per head (up to 16 CTAs per
 *                      head, partials merged in distributed shared memory)
 *                      when every cluster of at least 2 CTAs of the call can
 *                      be resident at once -- calls with few heads, e.g. one
 *                      layer at a small batch; else the stream-K kernel
 *                      (the held blocks of all heads cut evenly over one CTA
 *                      per SM, merged through the workspace).  The default.
 *   DMS_ATTN_STREAM_K  always the stream-K kernel.
 *   DMS_ATTN_CLUSTER   always the cluster kernel (clusters of one CTA, in
 *                      waves, when the call has more heads than fit).
 * Both compute the same attention (rounding order aside).  The calls with
 * device sequence lists (_seqs) and the stepper always use stream-K. */
#define DMS_ATTN_AUTO 0
#define DMS_ATTN_STREAM_K 1
#define DMS_ATTN_CLUSTER 2
dms_status dms_pool_set_attn_kernel(dms_pool* pool, int kind);

/* How dms_prefill_attn reads the keys of a bf16 pool (host setting of the
 * handle, applied to calls made after it):
 *   DMS_PREFILL_SPARSE  the layer is compacted first (as by
 *                       dms_compact_prefill_seqs); then, for a tile of 128
 *                       queries, keys older than every query's window are
 *                       read from the compact store (only the unflagged ones
 *                       exist there, in position order) as dense 128-key
 *                       tiles, and only the tiles holding the window edge,
 *                       the diagonal and the keys between are read from the
 *                       prompt with the full mask.  The default.
 *   DMS_PREFILL_DENSE   every causal key tile is read from the prompt and
 *                       masked; the kernel stores each diagonal tile's kept
 *                       rows itself.
 * Both give the same attention (rounding order aside) and the same store.
 * FP8 and 4-bit pools hold quantised rows, while the prompt's attention runs
 * on the bf16 inputs: in sparse mode their old kept keys are gathered from
 * the prompt by the positions their compaction records (an even group size
 * g only; otherwise, and in dense mode, every causal tile is read). */
#define DMS_PREFILL_SPARSE 0
#define DMS_PREFILL_DENSE 1
dms_status dms_pool_set_prefill_mode(dms_pool* pool, int mode);

/* The kernel a decode attention call over n_layers x batch heads of this
 * pool would use now (*kernel = DMS_ATTN_CLUSTER or DMS_ATTN_STREAM_K) and,
 * for the cluster kernel, its CTAs per head (*cluster_size; 0 for stream-K).
 * For the plain calls (dms_decode_attn_layers, dms_decode_step_layers); the
 * current device must be the pool's.  Host query, nothing is launched. */
dms_status dms_decode_attn_plan(dms_pool* pool, int n_layers, int batch, int* kernel,
                                int* cluster_size);

/* Region offsets of the pool buffer. */
dms_status dms_pool_layout(const dms_pool* pool, dms_pool_layout_t* out);

/* Prefill compaction of one layer (DMS delayed eviction applied at the end
 * of the prompt, t = P - 1): for every sequence b < batch and kv-head h,
 * keeps position j iff evict[b,j,h] == 0 or P-1-j < w, writes the kept K/V
 * rows to slots 0.. in position order, sets n_slots = n_retained = kept
 * count and fills the window ring with positions max(0,P-w)..P-1.
 * For an FP8 pool the per-(layer, kv-head) scales become amax/448 over all
 * P*batch rows of that head (before eviction), K and V separately, and rows
 * are stored as e4m3(x / scale) (round to nearest even, saturating).  A
 * 4-bit pool quantises each kept row with its own group scales (DMS_INT4).
 *   k, v   [batch, P, Hkv, D]  in_dtype (DMS_F32 or DMS_BF16)
 *   evict  [batch, P, Hkv]     uint8, non-zero = flagged
 * The layer must be empty (fresh pool or after dms_pool_reset), else the
 * device sets DMS_DEVERR_LAYER_NOT_EMPTY and writes nothing.  in_dtype
 * must equal kv_dtype, or be F32/BF16 for an FP8 or 4-bit pool.  (FP8: the scales
 * are only set when the layer has none yet; see dms_compact_prefill_seqs.)
 * Source: compaction = the compact store of the FastDMS page; eviction
 * before FP8 quantisation = the same page's FP8 paragraph. */
dms_status dms_compact_prefill(dms_pool* pool, int layer, int batch, int prompt_len,
                               const void* k, const void* v, dms_dtype in_dtype,
                               const uint8_t* evict, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Continuous batching.  Sequences start, decode and finish independently:
 * each occupies one of the pool's max_batch sequence slots, has its own
 * position, and on release gives its whole blocks back to the global
 * free-block stack (the pool of per-head variable token counts of the
 * FastDMS page, table "What's the catch?", row "PagedAttention / KV memory
 * pool"; its memory figures count real allocator memory, paragraph before
 * the memory table).  The calls below take device arrays so that a step can
 * be captured in a CUDA graph; a sequence id or position out of range sets
 * DMS_DEVERR_BAD_SEQUENCE and that head is skipped.
 * ------------------------------------------------------------------------ */

/* dms_compact_prefill for sequence slots [seq0, seq0 + batch) of a layer
 * (inputs indexed 0..batch-1).  Those slots must be empty in that layer
 * (fresh, reset, or released).  FP8: the first prefill into a layer sets
 * its scales from the amax of its own rows; later prefills of other
 * sequences of that layer reuse them and saturate, like decode tokens. */
dms_status dms_compact_prefill_seqs(dms_pool* pool, int layer, int seq0, int batch,
                                    int prompt_len, const void* k, const void* v,
                                    dms_dtype in_dtype, const uint8_t* evict,
                                    cudaStream_t stream);

/* dms_append_evict_layers with a list of sequences, each at its own
 * position: batch row r of k, v [n_layers, n_seqs, Hkv, D] and evict
 * [n_layers, n_seqs, Hkv] is the token at position pos[r] of sequence slot
 * seq_ids[r].  seq_ids int32 [n_seqs] and pos int64 [n_seqs] are device
 * arrays; the ids must be distinct.  Each sequence's positions must
 * increase by one per step from its prompt length.  A new block comes from
 * the global free-block stack first (blocks of released sequences), then
 * from the never-used tail of the pool. */
dms_status dms_append_evict_seqs(dms_pool* pool, int layer0, int n_layers, int n_seqs,
                                 const int32_t* seq_ids, const int64_t* pos, const void* k,
                                 const void* v, dms_dtype in_dtype, const uint8_t* evict,
                                 cudaStream_t stream);

/* dms_decode_attn_layers over a list of sequences: row r of q, out
 * [n_layers, n_seqs, Hq, D] belongs to sequence slot seq_ids[r] (int32
 * device array).  Workspace as for dms_decode_attn_layers with batch =
 * n_seqs. */
dms_status dms_decode_attn_seqs(dms_pool* pool, int layer0, int n_layers, int n_seqs,
                                const int32_t* seq_ids, const void* q, dms_dtype q_dtype,
                                void* out, float sm_scale, void* workspace,
                                size_t workspace_bytes, cudaStream_t stream);

/* Prompt attention under the delayed-eviction mask, fused with compaction:
 * for sequences [seq0, seq0 + batch) of a layer, out[b, i, hq] =
 * softmax(sm_scale * q[b, i, hq] . K^T) V over the keys j <= i that query i
 * can see (j unflagged, or i - j < w; kv-head hq / g), and the layer's kept
 * prompt rows are written into the pool exactly as dms_compact_prefill_seqs
 * writes them (the kernel that streams each K/V tile for attention also
 * stores the tile's kept rows).
 *   q, out  [batch, P, Hq, D]  bf16      k, v  [batch, P, Hkv, D]  bf16
 *   evict   [batch, P, Hkv]    uint8     sm_scale <= 0 selects 1/sqrt(D)
 * Needs a bf16, FP8 or 4-bit pool with head_dim 64 or 128 (else
 * DMS_ERR_UNSUPPORTED).  A bf16 pool is compacted first and its old kept
 * keys are read back from the store (DMS_PREFILL_SPARSE, the default), or
 * filled by the attention kernel itself (DMS_PREFILL_DENSE, see
 * dms_pool_set_prefill_mode); an FP8 or 4-bit pool is compacted first, as by
 * dms_compact_prefill_seqs, and the attention reads the bf16 inputs (old kept
 * keys gathered by position in sparse mode).
 * The sequences must be empty in that layer (else DMS_DEVERR_LAYER_NOT_EMPTY
 * and nothing is stored; the outputs are still computed).  Runs on the
 * tensor cores (tcgen05, accumulators in tensor memory).
 * Source: the mask holds for every query (mindverse page, DMS section;
 * stiva.ai page, "delayed eviction"); compaction as dms_compact_prefill. */
dms_status dms_prefill_attn(dms_pool* pool, int layer, int seq0, int batch, int prompt_len,
                            const void* q, const void* k, const void* v, dms_dtype in_dtype,
                            const uint8_t* evict, void* out, float sm_scale, cudaStream_t stream);

/* Workspace bytes dms_project_append needs: 0 (its partial sums are reduced
 * in distributed shared memory); kept so callers can size generically. */
dms_status dms_project_workspace_bytes(const dms_pool* pool, int n_seqs, int d_model,
                                       size_t* bytes);

/* The model's K/V projection of one decode token per sequence with the
 * eviction decision and the append fused into its epilogue.  For sequence
 * row s (slot seq_ids[s], or s when seq_ids is null; position pos[s]) and
 * kv-head h:
 *   k = bf16(x[s] W_kv[:, h*D : (h+1)*D])
 *   v = bf16(x[s] W_kv[:, (Hkv+h)*D : (Hkv+h+1)*D])
 *   flag = x[s] . w_evict[:, h] + b_evict[h] > threshold
 * then the token is appended exactly as dms_append_evict_seqs appends it.
 *   x        [n_seqs, d_model]       bf16
 *   w_kv     [d_model, 2 * Hkv * D]  bf16, row-major, 16-byte aligned
 *   w_evict  [d_model, Hkv]          bf16 (the predictor's weights: an input)
 *   b_evict  [Hkv] float, or null;   seq_ids int32 / pos int64 [n_seqs] device
 * fp32 accumulation, k and v rounded to nearest-even bf16.  Needs head_dim 128
 * and a bf16, FP8 or 4-bit pool.  workspace may be null (no scratch is needed).
 * Runs as one thread-block cluster of 8 CTAs per kv-head.
 * Source: a learned per-head predictor decides which tokens to evict
 * (mindverse page, DMS section); decode runs the projection step by step. */
dms_status dms_project_append(dms_pool* pool, int layer, int n_seqs, const int32_t* seq_ids,
                              const int64_t* pos, const void* x, int d_model, const void* w_kv,
                              const void* w_evict, const float* b_evict, float threshold,
                              void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* End sequences: for every layer and kv-head of the n_seqs sequence slots in
 * seq_ids (int32 device array, distinct ids), push every block they hold on
 * the global free-block stack and return their counters to empty, so the
 * slots can be prefilled again and the blocks reused by any sequence.
 * Calls that touch these sequences must be ordered before it. */
dms_status dms_release_seqs(dms_pool* pool, int n_seqs, const int32_t* seq_ids,
                            cudaStream_t stream);

/* One decode step at position `pos` (= t) for layers [layer0, layer0 +
 * n_layers): for every (layer, b, h): if t >= w and token t-w was flagged,
 * its slot goes onto the head's free stack (delayed eviction retires it);
 * token t takes the top free slot, else slot n_slots (a new block when the
 * slot starts one); its K/V row is written (FP8: with the prefill scale,
 * saturating); ring[t mod w] = slot | flag << 31.
 *   k, v   [n_layers, batch, Hkv, D]  in_dtype
 *   evict  [n_layers, batch, Hkv]     uint8
 * Positions must increase by one per step from the prompt length.
 * Source: delayed eviction (mindverse page, section "Dynamic Memory
 * Sparsification (DMS): Eine innovative Lösung"), slot reclaim (FastDMS
 * page, opening paragraphs). */
dms_status dms_append_evict_layers(dms_pool* pool, int layer0, int n_layers, int batch,
                                   int64_t pos, const void* k, const void* v,
                                   dms_dtype in_dtype, const uint8_t* evict,
                                   cudaStream_t stream);

/* Single-layer form of dms_append_evict_layers (k, v [batch, Hkv, D]). */
dms_status dms_append_evict(dms_pool* pool, int layer, int batch, int64_t pos,
                            const void* k, const void* v, dms_dtype in_dtype,
                            const uint8_t* evict, cudaStream_t stream);

/* Workspace bytes dms_decode_attn_layers needs for n_layers x batch. */
dms_status dms_decode_workspace_bytes(const dms_pool* pool, int n_layers, int batch,
                                      size_t* bytes);

/* Decode attention over the compact store for layers [layer0, layer0 +
 * n_layers): out[l,b,hq] = softmax(sm_scale * q[l,b,hq] . K_h^T) V_h over
 * the n_slots held rows of kv-head h = hq / g (the query's own token
 * included, appended before this call).  Split-K flash decoding: the held
 * rows of all heads form one list of BT-row blocks that is cut evenly over
 * a persistent grid; partial softmax states are merged by log-sum-exp.
 *   q, out     [n_layers, batch, Hq, D]  q_dtype (DMS_BF16 or DMS_F32;
 *              F32 only for an F32 pool); out has q's dtype
 *   sm_scale   <= 0 selects 1/sqrt(D)
 *   workspace  >= dms_decode_workspace_bytes, 256-byte aligned; no
 *              initialisation needed; must not be shared by concurrent calls
 * Source: attention over each head's retained tokens only (mindverse page,
 * DMS section; FastDMS page, speed claim at 8K context). */
dms_status dms_decode_attn_layers(dms_pool* pool, int layer0, int n_layers, int batch,
                                  const void* q, dms_dtype q_dtype, void* out, float sm_scale,
                                  void* workspace, size_t workspace_bytes,
                                  cudaStream_t stream);

/* One whole decode step at position `pos` for layers [layer0, layer0 +
 * n_layers): the result of dms_append_evict_layers(k, v, evict) followed by
 * dms_decode_attn_layers(q) -- the new token is stored exactly as the
 * append stores it and the attention covers the same rows -- in one launch
 * when the call has few heads (the cluster kernel: every CTA of a head reads
 * the head's state from before the append, a cluster barrier orders that
 * before the append, the slot the append reuses is masked and the new token
 * enters the attention from the inputs); otherwise the two kernels run in
 * turn.  The form a model issues layer by layer (layer l+1's query needs
 * layer l's output).  Arguments as for the two calls:
 *   k, v   [n_layers, batch, Hkv, D]  in_dtype;   evict [n_layers, batch, Hkv]
 *   q, out [n_layers, batch, Hq, D]   q_dtype;    workspace as for
 *   dms_decode_attn_layers (used only when the two kernels run).
 * Source: delayed eviction and the attention over each head's retained
 * tokens (mindverse page, DMS section); slot reclaim (FastDMS page, opening
 * paragraphs). */
dms_status dms_decode_step_layers(dms_pool* pool, int layer0, int n_layers, int batch, int64_t pos,
                                  const void* k, const void* v, dms_dtype in_dtype,
                                  const uint8_t* evict, const void* q, dms_dtype q_dtype, void* out,
                                  float sm_scale, void* workspace, size_t workspace_bytes,
                                  cudaStream_t stream);

/* Single-layer form of dms_decode_attn_layers (q, out [batch, Hq, D]). */
dms_status dms_decode_attn(dms_pool* pool, int layer, int batch, const void* q,
                           dms_dtype q_dtype, void* out, float sm_scale, void* workspace,
                           size_t workspace_bytes, cudaStream_t stream);

/* dms_decode_attn_layers for callers that cannot allocate device memory
 * (an engine that gave all free HBM to its KV pool, a plugin without access
 * to an allocator, a path that must not pay cudaMalloc's synchronisation).
 * The pages have no counterpart: this is a library convenience.  The
 * split-K scratch comes from a fixed 16 MiB array in the library's device
 * globals (present on every GPU that loads the library until exit) instead
 * of a caller workspace; calls needing more return DMS_ERR_CAPACITY.  The
 * first call on a device looks up the array's device address (make it
 * before any stream capture); after a device reset, or in another driver
 * context, the next call looks it up again in the context then current (make
 * that call before any capture too).  All calls on a device share the array:
 * nothing in it must start at zero, but calls whose kernels overlap on the
 * GPU race and must be ordered -- also calls on different pools or streams,
 * since the array is per device.  The current device must be the pool's. */
dms_status dms_decode_attn_layers_noalloc(dms_pool* pool, int layer0, int n_layers, int batch,
                                          const void* q, dms_dtype q_dtype, void* out,
                                          float sm_scale, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Decode steps fed from host memory
 *
 * A stepper runs whole decode steps (dms_append_evict_layers, then
 * dms_decode_attn_layers over the same layers) on inputs that live in host
 * memory, and copies each step's output back to host memory.  Every step
 * is one packed host->device copy, the two kernels and one device->host
 * copy; the copies run on two streams of the stepper's own, with four
 * staging and four output buffers in rotation against the caller's compute
 * stream, so the copies of one step overlap the kernels of its neighbours.  The pages have no counterpart: this is the
 * serving-side plumbing around the method's decode step.
 * ------------------------------------------------------------------------ */
typedef struct dms_stepper dms_stepper;  /* opaque host handle */

/* Packed host input of one step: four segments, each starting at a
 * multiple of 256 bytes,
 *   k      [n_layers, batch, Hkv, D]  in dtype (DMS_F32 for an F32 pool,
 *   v      [n_layers, batch, Hkv, D]   else DMS_BF16)
 *   q      [n_layers, batch, Hq, D]   same dtype
 *   evict  [n_layers, batch, Hkv]     uint8
 * The host output of one step is out [n_layers, batch, Hq, D] (q's dtype). */
typedef struct {
  size_t k, v, q, evict;  /* byte offsets of the segments */
  size_t in_bytes;        /* bytes of one packed host input */
  size_t out_bytes;       /* bytes of one host output */
  size_t device_bytes;    /* device buffer dms_stepper_create needs */
} dms_stepper_layout_t;

dms_status dms_stepper_layout(const dms_pool* pool, int n_layers, int batch,
                              dms_stepper_layout_t* out);

/* Create a stepper for layers [layer0, layer0 + n_layers) and sequences
 * 0..batch-1 of the pool.  device_buf (>= layout.device_bytes, 256-byte
 * aligned, owned by the caller, no initialisation) holds four input staging
 * buffers, four output buffers, 256 bytes of step counters and the attention
 * workspace.  `stream` is
 * the compute stream the kernels run on; the stepper creates two copy
 * streams and its events (no device memory).  The pool's device must be
 * current.  sm_scale as for dms_decode_attn_layers. */
dms_status dms_stepper_create(dms_pool* pool, int layer0, int n_layers, int batch,
                              float sm_scale, void* device_buf, size_t device_bytes,
                              cudaStream_t stream, dms_stepper** out);

/* Enqueue the decode step at position pos: host_in (layout.in_bytes, host)
 * -> device, append/evict + decode attention, output -> host_out
 * (layout.out_bytes, host).  Returns at once.  Both host buffers should be
 * page-locked (pinned) for the copies to be asynchronous, must stay valid
 * and unchanged (host_in) / unread (host_out) until the step has finished
 * (dms_stepper_join, then synchronise).  Positions follow the rules of
 * dms_append_evict_layers. */
dms_status dms_stepper_step(dms_stepper* st, int64_t pos, const void* host_in, void* host_out);

/* Host-side fault injection for failure-detection tests (the pages have no
 * counterpart).  DMS_FAULT_DROP_INPUT_SIGNAL: the next dms_stepper_step
 * copies its inputs but does not signal "inputs staged" to the device, as if
 * the copy engine's completion message were lost; that step's append kernel
 * waits for the signal until the pool's wait limit (dms_pool_set_wait_limit),
 * then sets DMS_DEVERR_TIMEOUT, and the step runs on (its outputs are
 * invalid).  Nothing faults, traps or hangs: later steps signal as usual.
 * Returns DMS_ERR_UNSUPPORTED when the stepper uses events (no driver stream
 * memory operations), where there is no signal to drop. */
#define DMS_FAULT_DROP_INPUT_SIGNAL 1
dms_status dms_stepper_inject_fault(dms_stepper* st, int fault);

/* Make `stream` wait for every step enqueued so far, output copies
 * included. */
dms_status dms_stepper_join(dms_stepper* st, cudaStream_t stream);

/* Wait for the stepper's work, then release its streams, events and the
 * host handle (device_buf stays the caller's). */
dms_status dms_stepper_destroy(dms_stepper* st);

/* Reduce the pool's counters on the device and copy them to *out (host).
 * Synchronises `stream`.  Returns DMS_ERR_DEVICE when the error word is
 * non-zero (*out is filled either way).  Source: real allocator memory,
 * not theoretical KV bytes (FastDMS page, paragraph before the memory
 * table). */
dms_status dms_pool_stats(dms_pool* pool, dms_pool_stats_t* out, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DMS_H */
