// Device twin of the seeded synthetic workload generator (NumPy module
// `synth`).  It draws random numbers only -- none of the method's arithmetic
// lives here -- and must reproduce the NumPy values bit for bit:
//   hash(key, n) = mix64(key + n * 0x9E3779B97F4A7C15), mix64 = the
//   SplitMix64 finaliser (Steele, Lea, Flood, OOPSLA 2014, "Mix13");
//   key = mix64(seed ^ (stream << 56));
//   counter = layer << 52 | b << 44 | pos << 20 | head << 12 | d << 2 | k;
//   normal = (sum of twelve 16-bit fields of words k = 0..2 - 393210) * 2^-16.
#include "dms_internal.cuh"
#include "dms_synth.h"

namespace dms {

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t hash64(uint64_t key, uint64_t n) {
  return mix64(key + n * 0x9E3779B97F4A7C15ull);
}

__device__ __forceinline__ uint64_t counter_of(uint64_t layer, uint64_t b, uint64_t pos,
                                               uint64_t head, uint64_t d) {
  return (layer << 52) | (b << 44) | (pos << 20) | (head << 12) | (d << 2);
}

template <typename OutT>
__global__ void synth_normal_kernel(uint64_t key, int layer0, int nl, int batch, int64_t pos0,
                                    int n_pos, int nh, int D, OutT* out) {
  const int64_t total = int64_t(nl) * batch * n_pos * nh * D;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < total;
       e += int64_t(gridDim.x) * blockDim.x) {
    int64_t r = e;
    const int d = int(r % D);
    r /= D;
    const int h = int(r % nh);
    r /= nh;
    const int64_t p = pos0 + r % n_pos;
    r /= n_pos;
    const int b = int(r % batch);
    const int l = layer0 + int(r / batch);
    const uint64_t base = counter_of(l, b, p, h, d);
    int sum = 0;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      const uint64_t w = hash64(key, base | uint64_t(k));
      sum += int(w & 0xffff) + int((w >> 16) & 0xffff) + int((w >> 32) & 0xffff) + int(w >> 48);
    }
    const float x = __int2float_rn(sum - 393210) * (1.0f / 65536.0f);
    if constexpr (sizeof(OutT) == 4) {
      out[e] = x;
    } else {
      out[e] = __float2bfloat16_rn(x);
    }
  }
}

__global__ void synth_flags_kernel(uint64_t key, int layer0, int nl, int batch, int64_t pos0,
                                   int n_pos, int nh, const int32_t* thr, uint8_t* out) {
  const int64_t total = int64_t(nl) * batch * n_pos * nh;
  for (int64_t e = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; e < total;
       e += int64_t(gridDim.x) * blockDim.x) {
    int64_t r = e;
    const int h = int(r % nh);
    r /= nh;
    const int64_t p = pos0 + r % n_pos;
    r /= n_pos;
    const int b = int(r % batch);
    const int li = int(r / batch);
    const uint64_t w = hash64(key, counter_of(layer0 + li, b, p, h, 0));
    const int u24 = int(w >> 40);
    out[e] = u24 >= thr[li * nh + h] ? 1 : 0;
  }
}

static uint64_t host_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

static bool synth_dims_ok(int layer0, int nl, int batch, int64_t pos0, int n_pos, int nh, int D) {
  return layer0 >= 0 && nl >= 1 && layer0 + nl <= 4096 && batch >= 1 && batch <= 256 &&
         pos0 >= 0 && n_pos >= 1 && pos0 + n_pos <= (int64_t(1) << 24) && nh >= 1 && nh <= 256 &&
         D >= 1 && D <= 1024;
}

static int grid_for(int64_t total) {
  const int64_t blocks = (total + 255) / 256;
  return int(blocks < 148 * 16 ? blocks : 148 * 16);
}

}  // namespace dms

using namespace dms;

extern "C" dms_status dms_synth_normal(uint64_t seed, int stream_id, int layer0, int n_layers,
                                       int batch, int64_t pos0, int n_pos, int n_heads,
                                       int head_dim, dms_dtype dtype, void* out,
                                       cudaStream_t stream) {
  if (!out || stream_id < 0 || stream_id > 255 ||
      !synth_dims_ok(layer0, n_layers, batch, pos0, n_pos, n_heads, head_dim)) {
    set_last_error("dms_synth_normal: bad arguments");
    return DMS_ERR_INVALID_ARG;
  }
  const uint64_t key = host_mix64(seed ^ (uint64_t(stream_id) << 56));
  const int64_t total = int64_t(n_layers) * batch * n_pos * n_heads * head_dim;
  if (dtype == DMS_F32) {
    synth_normal_kernel<float><<<grid_for(total), 256, 0, stream>>>(
        key, layer0, n_layers, batch, pos0, n_pos, n_heads, head_dim, static_cast<float*>(out));
  } else if (dtype == DMS_BF16) {
    synth_normal_kernel<__nv_bfloat16><<<grid_for(total), 256, 0, stream>>>(
        key, layer0, n_layers, batch, pos0, n_pos, n_heads, head_dim,
        static_cast<__nv_bfloat16*>(out));
  } else {
    set_last_error("dms_synth_normal: dtype must be DMS_F32 or DMS_BF16");
    return DMS_ERR_INVALID_ARG;
  }
  return cuda_status(cudaGetLastError(), "synth_normal_kernel");
}

extern "C" dms_status dms_synth_flags(uint64_t seed, int layer0, int n_layers, int batch,
                                      int64_t pos0, int n_pos, int n_heads, const int32_t* thr,
                                      uint8_t* out, cudaStream_t stream) {
  if (!out || !thr || !synth_dims_ok(layer0, n_layers, batch, pos0, n_pos, n_heads, 1)) {
    set_last_error("dms_synth_flags: bad arguments");
    return DMS_ERR_INVALID_ARG;
  }
  const uint64_t key = host_mix64(seed ^ (uint64_t(3) << 56));
  const int64_t total = int64_t(n_layers) * batch * n_pos * n_heads;
  synth_flags_kernel<<<grid_for(total), 256, 0, stream>>>(key, layer0, n_layers, batch, pos0,
                                                          n_pos, n_heads, thr, out);
  return cuda_status(cudaGetLastError(), "synth_flags_kernel");
}
