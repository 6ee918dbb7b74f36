// Host side of decode attention: grid sizing, workspace layout and the dispatch to the kernel
// instantiation of the cache's (K, V) code widths (one translation unit per width pair,
// iq_decode_k*v*.cu, so that they compile in parallel).
#include <cuda_runtime.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

#include "iq_prefill_impl.cuh"

namespace iq {

static inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// CTAs of one launch that an SM holds at once: the occupancy calculator's figure for this
// kernel instantiation at the launch's dynamic shared memory (rounded up to 1 KB), cached per
// device.  The final merge waits for other CTAs of the same grid, so a grid must never exceed it.
int resident_per_sm(const void* fn, size_t smem, int threads) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const size_t bucket = (smem + 1023) & ~(size_t)1023;
  static std::mutex mu;
  static std::map<std::tuple<int, const void*, size_t>, int> memo;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_tuple(dev, fn, bucket);
  const auto it = memo.find(key);
  if (it != memo.end()) return it->second;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, bucket) != cudaSuccess) n = 0;
  memo[key] = n;
  return n;
}

// Two CTAs per SM when the problem is large (each warp gets >= 16 tiles) and two are resident;
// else one, which leaves the other half of every SM free for the next kernel's CTAs to start
// their loads early (programmatic dependent launch).  0 when not even one CTA fits.
int decode_ctas(int batch, int n_kv_heads, int max_ctx, int resident) {
  const int n_sm = sm_count();
  const long long tiles = (long long)batch * n_kv_heads * ((max_ctx + TT - 1) / TT);
  const bool big = tiles >= (long long)n_sm * 2 * DEC_WARPS * 16;
  return n_sm * std::min(resident, big ? 2 : 1);
}

// Partial slots: one per (CTA, group) pair a run can produce; CTA c's partial of group gid is
// slot c + gid (a CTA's run covers consecutive groups), so 2 * #SMs + groups slots suffice.
static size_t ws_slots(int batch, int n_kv_heads) { return (size_t)2 * sm_count() + (size_t)batch * n_kv_heads; }

int workspace_base_slots(int batch, int n_kv_heads) { return (int)ws_slots(batch, n_kv_heads); }

size_t decode_workspace_bytes(int batch, int n_q_heads, int n_kv_heads, int max_ctx, int extra_slots) {
  (void)n_q_heads;
  (void)max_ctx;
  const size_t groups = (size_t)batch * n_kv_heads, slots = ws_slots(batch, n_kv_heads) + (size_t)extra_slots;
  return align256(groups * 8) + align256(slots * HMAX * sizeof(float2)) + align256(slots * HMAX * D * sizeof(float));
}

size_t decode_counter_bytes(int batch, int n_kv_heads) { return align256((size_t)batch * n_kv_heads * 8); }

Workspace carve_workspace(void* ws, int batch, int n_kv_heads, int extra_slots) {
  const size_t groups = (size_t)batch * n_kv_heads, slots = ws_slots(batch, n_kv_heads) + (size_t)extra_slots;
  Workspace w;
  char* p = (char*)ws;
  w.counters = (uint32_t*)p;
  p += align256(groups * 8);
  w.part_ml = (float2*)p;
  p += align256(slots * HMAX * sizeof(float2));
  w.part_o = (float*)p;
  return w;
}

#define IQ_DECODE_WIDTHS(X) X(2, 2) X(3, 2) X(3, 3) X(4, 2) X(4, 3) X(4, 4)
#define IQ_DECL(KB, VB)                                                                                      \
  extern template int launch_decode_kv<KB, VB>(const LayerView&, const void*, int, int, int, const int32_t*, \
                                               int, const float*, float*, void*, const KernelConsts&, void*,  \
                                               const void*, const void*, const DeferredInfo*);
IQ_DECODE_WIDTHS(IQ_DECL)
#undef IQ_DECL
#define IQ_DECL(KB, VB)                                                                                         \
  extern template int launch_prefill_kv<KB, VB>(const LayerView&, const void*, int, int, int, int, const int32_t*, \
                                                int, const float*, float*, void*, const KernelConsts&, void*, int);
IQ_DECODE_WIDTHS(IQ_DECL)
#undef IQ_DECL

static int dispatch(const LayerView& v, const void* q, int q_f32, int batch, int n_q_heads, const int32_t* ctx_len,
                    int max_ctx, const float* params_layer, float* out, void* workspace, const KernelConsts& kc,
                    void* stream, const void* k_new, const void* v_new, const DeferredInfo* def = nullptr) {
#define IQ_CASE(KB, VB)                                                                                          \
  if (v.kb == KB && v.vb == VB)                                                                                 \
    return launch_decode_kv<KB, VB>(v, q, q_f32, batch, n_q_heads, ctx_len, max_ctx, params_layer, out, workspace, \
                                    kc, stream, k_new, v_new, def);
  IQ_DECODE_WIDTHS(IQ_CASE)
#undef IQ_CASE
  return (int)cudaErrorInvalidValue;
}

int launch_decode(const LayerView& v, const void* q, int q_f32, int batch, int n_q_heads, const int32_t* ctx_len,
                  int max_ctx, const float* params_layer, float* out, void* workspace, const KernelConsts& kc,
                  void* stream) {
  return dispatch(v, q, q_f32, batch, n_q_heads, ctx_len, max_ctx, params_layer, out, workspace, kc, stream, nullptr,
                  nullptr);
}

int launch_decode_step(const LayerView& v, const void* q, int q_f32, const void* k_new, const void* v_new, int batch,
                       int n_q_heads, const int32_t* ctx_len, int max_ctx, const float* params_layer, float* out,
                       void* workspace, const KernelConsts& kc, void* stream) {
  return dispatch(v, q, q_f32, batch, n_q_heads, ctx_len, max_ctx, params_layer, out, workspace, kc, stream, k_new,
                  v_new);
}

// Deferred quantisation: the fp16-prefix kernel writes its split partials into the extra slots,
// then the fused step (which waits for it) attends over the packed tail and merges both.
int launch_decode_deferred(const LayerView& v, const void* q, int q_f32, const void* k_new, const void* v_new,
                           int batch, int n_q_heads, const int32_t* ctx_len, int max_ctx, const float* params_layer,
                           float* out, void* workspace, const KernelConsts& kc, void* stream, const void* k16,
                           const void* v16, const int32_t* len, int max_len) {
  if (batch == 0 || n_q_heads == 0) return 0;
  const int splits = prefix_splits(batch, v.n_kv_heads, max_len, sm_count());
  int e = launch_prefix(v, k16, v16, len, max_len, ctx_len, max_ctx, q, q_f32, batch, n_q_heads, params_layer, kc,
                        workspace, splits, workspace_base_slots(batch, v.n_kv_heads), stream);
  if (e) return e;
  DeferredInfo def{len, splits};
  return dispatch(v, q, q_f32, batch, n_q_heads, ctx_len, max_ctx, params_layer, out, workspace, kc, stream, k_new,
                  v_new, &def);
}

// Prefill workspace: per (group, split, query row) one (m, l) pair and one 128-float O; the
// query rows of a group depend on the group size, which the size query does not know, so the
// largest over group sizes 1 .. 8.
size_t prefill_workspace_bytes(int batch, int n_tok, int n_kv_heads, int max_ctx) {
  size_t rows = 0;
  for (int g = 1; g <= HMAX; ++g) rows = std::max(rows, prefill_rows(batch, n_tok, n_kv_heads, max_ctx, g, sm_count(), nullptr));
  return align256(rows * sizeof(float2)) + align256(rows * D * sizeof(float));
}

int launch_prefill(const LayerView& v, const void* q, int q_f32, int batch, int n_tok, int n_q_heads,
                   const int32_t* start, int max_ctx, const float* params_layer, float* out, void* workspace,
                   const KernelConsts& kc, void* stream) {
#define IQ_CASE(KB, VB)                                                                                        \
  if (v.kb == KB && v.vb == VB)                                                                               \
    return launch_prefill_kv<KB, VB>(v, q, q_f32, batch, n_tok, n_q_heads, start, max_ctx, params_layer, out, \
                                     workspace, kc, stream, sm_count());
  IQ_DECODE_WIDTHS(IQ_CASE)
#undef IQ_CASE
  return (int)cudaErrorInvalidValue;
}

}  // namespace iq
