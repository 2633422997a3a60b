// Decode steps fed from host memory (dms_stepper_*).
//
// Per step: one packed host->device copy of (k, v, q, evict) on the h2d
// stream, append/evict and decode attention on the caller's compute stream,
// one device->host copy of the output on the d2h stream.  kStepperDepth
// staging buffers and as many output buffers rotate between steps (D =
// kStepperDepth):
//   h2d(n)      after  kernels(n-D)   (staging[n % D] free again)
//   kernels(n)  after  h2d(n), d2h(n-D) (output[n % D] free)
//   d2h(n)      after  kernels(n)
// The compute stream holds only the kernels, so that the append of step
// n+1 starts under the attention of step n (programmatic launch); the copy
// streams wait on and set step counters in device memory (stream memory
// operations), the append kernel waits for its inputs and the attention
// kernel for its output buffer, and the attention's last CTA publishes the
// step as computed.  Without the driver's stream memory operations the
// same order is kept with events on all three streams.  With D = 4 the input
// copy of step n is issued three steps ahead of the kernels that free its
// buffer, so the waits find their conditions met (with two buffers the copy
// waited for kernels(n-2) and the compute stream for the copy, about 11 us a
// step on the Qwen3-8B ctx-8K workload).
#include <cuda.h>
#include <new>

#include "dms_internal.cuh"

namespace dms {

constexpr int kStepperDepth = 4;

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

static dms_status stepper_layout(const dms_pool* pool, int n_layers, int batch,
                                 dms_stepper_layout_t* o) {
  const PoolView& v = pool->view;
  const size_t esz = v.kv_dtype == DMS_F32 ? 4 : 2;
  const size_t kv = size_t(n_layers) * batch * v.Hkv * v.D * esz;
  const size_t qb = size_t(n_layers) * batch * v.Hq * v.D * esz;
  const size_t eb = size_t(n_layers) * batch * v.Hkv;
  o->k = 0;
  o->v = align256(kv);
  o->q = o->v + align256(kv);
  o->evict = o->q + align256(qb);
  o->in_bytes = o->evict + align256(eb);
  o->out_bytes = qb;
  size_t ws = 0;
  dms_status st = dms_decode_workspace_bytes(pool, n_layers, batch, &ws);
  if (st != DMS_OK) return st;
  // + 256 bytes of step counters (ready, done, drained, exit count)
  o->device_bytes = kStepperDepth * (o->in_bytes + align256(qb)) + 256 + align256(ws);
  return DMS_OK;
}

// cuStreamWaitValue32 / cuStreamWriteValue32 through the runtime's driver
// entry point (no link against the driver library); null when unavailable
typedef CUresult (*StreamValueFn)(CUstream, CUdeviceptr, cuuint32_t, unsigned int);
static StreamValueFn stream_value_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<StreamValueFn>(p);
}

}  // namespace dms

using namespace dms;

struct dms_stepper {
  dms_pool* pool;
  int layer0, n_layers, batch;
  float sm_scale;
  dms_dtype dtype;
  dms_stepper_layout_t lay;
  uint8_t* stage[kStepperDepth];
  uint8_t* out[kStepperDepth];
  void* ws;
  size_t ws_bytes;
  cudaStream_t compute, h2d, d2h;
  cudaEvent_t staged[kStepperDepth], computed[kStepperDepth], drained[kStepperDepth];
  int64_t steps;
  // step counters in device memory: [0] steps staged, [1] steps computed,
  // [2] steps copied out, [3] attention CTAs that left (self-resetting)
  int32_t* counters;
  StreamValueFn wait_value, write_value;  // both non-null: counter protocol
  bool drop_input_signal;                 // injected fault: skip the next "staged" write
};

extern "C" dms_status dms_stepper_layout(const dms_pool* pool, int n_layers, int batch,
                                         dms_stepper_layout_t* out) {
  if (!pool || !out || n_layers < 1 || batch < 1) {
    set_last_error("bad arguments");
    return DMS_ERR_INVALID_ARG;
  }
  return stepper_layout(pool, n_layers, batch, out);
}

static void stepper_release(dms_stepper* s) {
  for (int j = 0; j < kStepperDepth; ++j) {
    if (s->staged[j]) cudaEventDestroy(s->staged[j]);
    if (s->computed[j]) cudaEventDestroy(s->computed[j]);
    if (s->drained[j]) cudaEventDestroy(s->drained[j]);
  }
  if (s->h2d) cudaStreamDestroy(s->h2d);
  if (s->d2h) cudaStreamDestroy(s->d2h);
  delete s;
}

extern "C" dms_status dms_stepper_create(dms_pool* pool, int layer0, int n_layers, int batch,
                                         float sm_scale, void* device_buf, size_t device_bytes,
                                         cudaStream_t stream, dms_stepper** out) {
  if (!pool || !out || !device_buf) {
    set_last_error("null pool / out / device_buf");
    return DMS_ERR_INVALID_ARG;
  }
  const PoolView& v = pool->view;
  if (layer0 < 0 || n_layers < 1 || layer0 + n_layers > v.L || batch < 1 || batch > v.Bmax) {
    set_last_error("bad layer range / batch (%d+%d, %d)", layer0, n_layers, batch);
    return DMS_ERR_INVALID_ARG;
  }
  if (reinterpret_cast<uintptr_t>(device_buf) & 255) {
    set_last_error("device_buf must be 256-byte aligned");
    return DMS_ERR_INVALID_ARG;
  }
  dms_stepper_layout_t lay;
  dms_status st = stepper_layout(pool, n_layers, batch, &lay);
  if (st != DMS_OK) return st;
  if (device_bytes < lay.device_bytes) {
    set_last_error("device_buf has %zu bytes, needs %zu", device_bytes, lay.device_bytes);
    return DMS_ERR_CAPACITY;
  }
  int dev = -1;
  st = cuda_status(cudaGetDevice(&dev), "cudaGetDevice");
  if (st != DMS_OK) return st;
  if (dev != pool->device) {
    set_last_error("current device %d is not the pool's device %d", dev, pool->device);
    return DMS_ERR_INVALID_ARG;
  }
  dms_stepper* s = new (std::nothrow) dms_stepper();
  if (!s) {
    set_last_error("out of host memory");
    return DMS_ERR_CAPACITY;
  }
  s->pool = pool;
  s->layer0 = layer0;
  s->n_layers = n_layers;
  s->batch = batch;
  s->sm_scale = sm_scale;
  s->dtype = v.kv_dtype == DMS_F32 ? DMS_F32 : DMS_BF16;
  s->lay = lay;
  uint8_t* b = static_cast<uint8_t*>(device_buf);
  for (int j = 0; j < kStepperDepth; ++j) {
    s->stage[j] = b;
    b += lay.in_bytes;
  }
  for (int j = 0; j < kStepperDepth; ++j) {
    s->out[j] = b;
    b += align256(lay.out_bytes);
  }
  s->counters = reinterpret_cast<int32_t*>(b);
  b += 256;
  s->ws = b;
  s->ws_bytes = device_bytes - size_t(b - static_cast<uint8_t*>(device_buf));
  s->wait_value = stream_value_fn("cuStreamWaitValue32");
  s->write_value = stream_value_fn("cuStreamWriteValue32");
  if (!s->wait_value || !s->write_value) s->wait_value = s->write_value = nullptr;
  s->compute = stream;
  st = cuda_status(cudaStreamCreateWithFlags(&s->h2d, cudaStreamNonBlocking), "stepper h2d stream");
  if (st == DMS_OK)
    st = cuda_status(cudaStreamCreateWithFlags(&s->d2h, cudaStreamNonBlocking), "stepper d2h stream");
  for (int j = 0; j < kStepperDepth && st == DMS_OK; ++j) {
    st = cuda_status(cudaEventCreateWithFlags(&s->staged[j], cudaEventDisableTiming), "stepper event");
    if (st == DMS_OK)
      st = cuda_status(cudaEventCreateWithFlags(&s->computed[j], cudaEventDisableTiming), "stepper event");
    if (st == DMS_OK)
      st = cuda_status(cudaEventCreateWithFlags(&s->drained[j], cudaEventDisableTiming), "stepper event");
  }
  if (st == DMS_OK)
    st = cuda_status(cudaMemsetAsync(s->counters, 0, 256, stream), "stepper counters");
  if (st == DMS_OK) st = cuda_status(cudaStreamSynchronize(stream), "stepper counters");
  if (st != DMS_OK) {
    stepper_release(s);
    return st;
  }
  *out = s;
  return DMS_OK;
}

extern "C" dms_status dms_stepper_step(dms_stepper* s, int64_t pos, const void* host_in,
                                       void* host_out) {
  if (!s || !host_in || !host_out) {
    set_last_error("null stepper / host_in / host_out");
    return DMS_ERR_INVALID_ARG;
  }
  const int j = int(s->steps % kStepperDepth);
  const bool reuse = s->steps >= kStepperDepth;
  const dms_stepper_layout_t& L = s->lay;
  uint8_t* stg = s->stage[j];
  dms_status st = DMS_OK;
  if (s->wait_value) {
    // Counter protocol: the compute stream holds only the two kernels, so
    // the append of step n+1 and the attention of step n stay chained by
    // programmatic launch; the copy streams wait on and set device counters.
    const int32_t n = int32_t(s->steps);
    auto dptr = [&](int i) { return CUdeviceptr(reinterpret_cast<uintptr_t>(s->counters + i)); };
    auto drv = [&](CUresult r, const char* what) {
      if (r == CUDA_SUCCESS) return DMS_OK;
      set_last_error("%s failed (%d)", what, int(r));
      return DMS_ERR_CUDA;
    };
    // host -> device once the kernels of step n-D are done with the buffer
    if (reuse)
      st = drv(s->wait_value(s->h2d, dptr(1), cuuint32_t(n - kStepperDepth + 1), CU_STREAM_WAIT_VALUE_GEQ),
               "stepper wait (computed)");
    if (st == DMS_OK)
      st = cuda_status(cudaMemcpyAsync(stg, host_in, L.in_bytes, cudaMemcpyHostToDevice, s->h2d),
                       "stepper input copy");
    if (st == DMS_OK && !s->drop_input_signal)
      st = drv(s->write_value(s->h2d, dptr(0), cuuint32_t(n + 1), CU_STREAM_WRITE_VALUE_DEFAULT),
               "stepper write (staged)");
    s->drop_input_signal = false;
    StepSync in{};
    in.ready = s->counters + 0;
    in.ready_value = n + 1;
    StepSync att{};
    att.drained = reuse ? s->counters + 2 : nullptr;
    att.drained_value = n - kStepperDepth + 1;
    att.done = s->counters + 1;
    att.done_value = n + 1;
    att.exit_count = s->counters + 3;
    if (st == DMS_OK)
      st = append_layers_synced(s->pool, s->layer0, s->n_layers, s->batch, pos, stg + L.k, stg + L.v,
                                s->dtype, stg + L.evict, s->compute, in);
    if (st == DMS_OK)
      st = decode_attn_layers_synced(s->pool, s->layer0, s->n_layers, s->batch, stg + L.q, s->out[j],
                                     s->sm_scale, s->ws, s->compute, att);
    // device -> host once the step is computed
    if (st == DMS_OK)
      st = drv(s->wait_value(s->d2h, dptr(1), cuuint32_t(n + 1), CU_STREAM_WAIT_VALUE_GEQ),
               "stepper wait (computed)");
    if (st == DMS_OK)
      st = cuda_status(cudaMemcpyAsync(host_out, s->out[j], L.out_bytes, cudaMemcpyDeviceToHost, s->d2h),
                       "stepper output copy");
    if (st == DMS_OK)
      st = drv(s->write_value(s->d2h, dptr(2), cuuint32_t(n + 1), CU_STREAM_WRITE_VALUE_DEFAULT),
               "stepper write (drained)");
    if (st == DMS_OK) st = cuda_status(cudaEventRecord(s->drained[j], s->d2h), "stepper record");
    if (st == DMS_OK) ++s->steps;
    return st;
  }
  // host -> device: the staging buffer is free once the kernels of step n-D ran
  if (reuse) st = cuda_status(cudaStreamWaitEvent(s->h2d, s->computed[j], 0), "stepper wait");
  if (st == DMS_OK)
    st = cuda_status(cudaMemcpyAsync(stg, host_in, L.in_bytes, cudaMemcpyHostToDevice, s->h2d),
                     "stepper input copy");
  if (st == DMS_OK) st = cuda_status(cudaEventRecord(s->staged[j], s->h2d), "stepper record");
  // kernels: after the input landed and the output buffer's previous copy-out
  if (st == DMS_OK) st = cuda_status(cudaStreamWaitEvent(s->compute, s->staged[j], 0), "stepper wait");
  if (st == DMS_OK && reuse)
    st = cuda_status(cudaStreamWaitEvent(s->compute, s->drained[j], 0), "stepper wait");
  if (st == DMS_OK)
    st = dms_append_evict_layers(s->pool, s->layer0, s->n_layers, s->batch, pos, stg + L.k, stg + L.v,
                                 s->dtype, stg + L.evict, s->compute);
  if (st == DMS_OK)
    st = dms_decode_attn_layers(s->pool, s->layer0, s->n_layers, s->batch, stg + L.q, s->dtype,
                                s->out[j], s->sm_scale, s->ws, s->ws_bytes, s->compute);
  if (st == DMS_OK) st = cuda_status(cudaEventRecord(s->computed[j], s->compute), "stepper record");
  // device -> host
  if (st == DMS_OK) st = cuda_status(cudaStreamWaitEvent(s->d2h, s->computed[j], 0), "stepper wait");
  if (st == DMS_OK)
    st = cuda_status(cudaMemcpyAsync(host_out, s->out[j], L.out_bytes, cudaMemcpyDeviceToHost, s->d2h),
                     "stepper output copy");
  if (st == DMS_OK) st = cuda_status(cudaEventRecord(s->drained[j], s->d2h), "stepper record");
  if (st == DMS_OK) ++s->steps;
  return st;
}

extern "C" dms_status dms_stepper_inject_fault(dms_stepper* s, int fault) {
  if (!s || fault != DMS_FAULT_DROP_INPUT_SIGNAL) {
    set_last_error("null stepper or unknown fault %d", fault);
    return DMS_ERR_INVALID_ARG;
  }
  if (!s->wait_value) {
    set_last_error("the stepper runs on events (no stream memory operations): no signal to drop");
    return DMS_ERR_UNSUPPORTED;
  }
  s->drop_input_signal = true;
  return DMS_OK;
}

extern "C" dms_status dms_stepper_join(dms_stepper* s, cudaStream_t stream) {
  if (!s) {
    set_last_error("null stepper");
    return DMS_ERR_INVALID_ARG;
  }
  for (int j = 0; j < kStepperDepth && j < s->steps; ++j) {
    dms_status st = cuda_status(cudaStreamWaitEvent(stream, s->drained[j], 0), "stepper join");
    if (st != DMS_OK) return st;
  }
  return DMS_OK;
}

extern "C" dms_status dms_stepper_destroy(dms_stepper* s) {
  if (!s) return DMS_OK;
  dms_status st = cuda_status(cudaStreamSynchronize(s->h2d), "stepper sync");
  dms_status st2 = cuda_status(cudaStreamSynchronize(s->d2h), "stepper sync");
  stepper_release(s);
  return st != DMS_OK ? st : st2;
}
