/*
 * dms_synth.h -- seeded synthetic workload generator (device side).
 *
 * Not part of the method: it only draws the random K/V/Q values and
 * eviction flags of the synthetic workloads on the GPU, where the largest
 * ones (8.6 GB of prompt K/V per layer) must be made.  It is the bit-exact
 * twin of the NumPy module `synth`:
 *   hash(key, n)   = mix64(key + n * 0x9E3779B97F4A7C15), mix64 = the
 *                    SplitMix64 finaliser (Steele, Lea, Flood, OOPSLA 2014)
 *   key(seed, s)   = mix64(seed ^ (s << 56)), s: 0 = K, 1 = V, 2 = Q, 3 = flags
 *   counter        = layer << 52 | b << 44 | pos << 20 | head << 12 | d << 2 | k
 *   normal         = (sum of the twelve 16-bit fields of hash words k = 0,1,2
 *                    - 393210) * 2^-16 in fp32; bf16 by round-to-nearest-even
 *   evict          = (hash word of d = k = 0) >> 40 >= thr[layer, head]
 * Host errors are returned as dms_status; nothing is allocated.
 */
#ifndef DMS_SYNTH_H
#define DMS_SYNTH_H

#include "dms.h"

#ifdef __cplusplus
extern "C" {
#endif

/* out[l, b, p, h, d] for l < n_layers (layer index layer0 + l), b < batch,
 * p < n_pos (position pos0 + p), h < n_heads, d < head_dim; dtype DMS_F32 or
 * DMS_BF16. */
dms_status dms_synth_normal(uint64_t seed, int stream_id, int layer0, int n_layers, int batch,
                            int64_t pos0, int n_pos, int n_heads, int head_dim, dms_dtype dtype,
                            void* out, cudaStream_t stream);

/* out[l, b, p, h] uint8 eviction flags; thr[l * n_heads + h] (device int32)
 * holds the 24-bit keep threshold of layer layer0 + l, kv-head h. */
dms_status dms_synth_flags(uint64_t seed, int layer0, int n_layers, int batch, int64_t pos0,
                           int n_pos, int n_heads, const int32_t* thr, uint8_t* out,
                           cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DMS_SYNTH_H */
