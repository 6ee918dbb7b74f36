// iq_decode_attention_noalloc: decode attention whose split-K scratch lives in a fixed
// device array inside this library, for callers that cannot allocate device memory.
//
// Some callers are not allowed to call cudaMalloc: plugins whose host application owns every
// device allocation, and real-time or long-running services that must not allocate after
// start-up (an allocation can synchronise the device, and it can fail under memory pressure
// at the worst moment).  They can still pass their own inputs and outputs; this entry point
// takes care of the scratch space that iq_decode_attention otherwise asks the caller for.
//
// The scratch is one file-scope array of IQ_NOALLOC_SCRATCH_BYTES per device.  Every GPU that
// loads this library keeps it until the process exits.  Host code cannot use the array's name
// as a device address, so the device address is looked up with cudaGetSymbolAddress once per
// device, with that device current, on the first call made on it.
#include <cuda_runtime.h>

#include <mutex>

#include "iq_internal.h"

namespace {

// Split-K scratch of one call: per-group arrival counters (cleared by every call before its
// kernel runs), then the partial maxima, sums and value sums.
static __device__ __align__(256) unsigned char g_noalloc_scratch[IQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of this device's copy of the scratch array (looked up once per device).
cudaError_t scratch_for_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" iq_status iq_decode_attention_noalloc(const iq_cache* cache, int32_t layer, const void* q_dev,
                                                 iq_dtype q_dtype, int32_t batch, int32_t n_q_heads,
                                                 const int32_t* ctx_len_dev, int32_t max_ctx,
                                                 const float* params_dev, float* out_dev, iq_stream_t stream) {
  if (!cache || cache->n_kv_heads < 1 || batch < 0 || n_q_heads < 0 || max_ctx < 0) return IQ_ERR_INVALID_ARG;
  const size_t need = iq_decode_workspace_size(batch, n_q_heads, cache->n_kv_heads, max_ctx);
  if (need > (size_t)IQ_NOALLOC_SCRATCH_BYTES) return IQ_ERR_WORKSPACE;  // problem too large for the fixed scratch
  void* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) return IQ_ERR_CUDA;
  // the arrival counters must start at zero; a call cut short by an error may leave them set
  if (cudaMemsetAsync(scratch, 0, iq::decode_counter_bytes(batch, cache->n_kv_heads), (cudaStream_t)stream) !=
      cudaSuccess)
    return IQ_ERR_CUDA;
  return iq_decode_attention(cache, layer, q_dev, q_dtype, batch, n_q_heads, ctx_len_dev, max_ctx, params_dev,
                             out_dev, scratch, (size_t)IQ_NOALLOC_SCRATCH_BYTES, stream);
}
