// extern "C" entry points of libiq: argument checks, layer views, kernel dispatch.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "iq_internal.h"

namespace iq {

// Centroids reach the tensor cores as int8 pairs: alpha8 * c_k ~ hi_k + lo_k / 254 with
// hi_k, lo_k integers in [-127, 127].  alpha8 is the scale (searched on a 1e-5 grid below the
// largest admissible value) that minimises the worst relative error over the codebook's
// positive levels; for the 2-, 3- and 4-bit N(0,1) codebooks it is far below the fp32 rounding
// of the products that follow (3 bits: under 3e-6).
static void int8_levels(const Codebook& cb, double& alpha8, int hi[16], int lo[16]) {
  const int n = 1 << cb.bits;
  const double cmax = cb.level[n - 1];
  double best = 1e30;
  alpha8 = 0.0;
  for (long i = 0;; ++i) {
    const double a = 127.49 / cmax - 1e-5 * (double)i;
    if (a < 0.5 * 127.49 / cmax) break;
    double err = 0.0;
    bool ok = true;
    for (int k = n / 2; k < n; ++k) {
      const double v = a * cb.level[k];
      const double h = std::nearbyint(v);
      const double l = std::nearbyint((v - h) * 254.0);
      if (std::fabs(h) > 127.0 || std::fabs(l) > 127.0) { ok = false; break; }
      err = std::fmax(err, std::fabs((h + l / 254.0) / a - cb.level[k]) / cb.level[k]);
      if (err >= best) { ok = false; break; }
    }
    if (ok && err < best) { best = err; alpha8 = a; }
  }
  for (int k = 0; k < n; ++k) {
    const double v = alpha8 * cb.level[k];
    hi[k] = (int)std::nearbyint(v);
    lo[k] = (int)std::nearbyint((v - hi[k]) * 254.0);
  }
}

static SideConsts make_side(int bits) {
  const Codebook cb = compute_codebook(bits);
  const int n = 1 << bits;
  SideConsts sc = {};
  sc.bits = bits;
  for (int j = 0; j < n / 2 - 1; ++j) sc.bound_pos[j] = (float)cb.bound[n / 2 + j];
  double alpha8;
  int hi[16], lo[16];
  int8_levels(cb, alpha8, hi, lo);
  for (int k = 0; k < n; ++k) {
    sc.lut_hi[k >> 2] |= (uint32_t)(uint8_t)(int8_t)hi[k] << (8 * (k & 3));
    sc.lut_lo[k >> 2] |= (uint32_t)(uint8_t)(int8_t)lo[k] << (8 * (k & 3));
  }
  sc.alpha8 = (float)alpha8;
  for (int k = 0; k < n; ++k) {
    const __half h = __float2half_rn((float)cb.level[k]);
    const __half l = __float2half_rn((float)(cb.level[k] - (double)__half2float(h)));
    const uint16_t bits16[2] = {__half_as_ushort(h), __half_as_ushort(l)};
    for (int t = 0; t < 2; ++t) {
      sc.f16_lb[t][k >> 2] |= (uint32_t)(bits16[t] & 0xFFu) << (8 * (k & 3));
      sc.f16_hb[t][k >> 2] |= (uint32_t)(bits16[t] >> 8) << (8 * (k & 3));
    }
  }
  return sc;
}

const KernelConsts& kernel_consts(int kb, int vb) {
  static std::once_flag once;
  static SideConsts side[5];
  static KernelConsts table[5][5];
  std::call_once(once, [] {
    for (int b = 2; b <= 4; ++b) side[b] = make_side(b);
    for (int k = 2; k <= 4; ++k)
      for (int v = 2; v <= 4; ++v) table[k][v] = KernelConsts{side[k], side[v]};
  });
  return table[kb][vb];
}

static bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

static int k_bits(const iq_cache* c) { return c->k_bits ? c->k_bits : 3; }
static int v_bits(const iq_cache* c) { return c->v_bits ? c->v_bits : 3; }

static iq_status check_cache(const iq_cache* c, int32_t layer) {
  if (!c) return IQ_ERR_INVALID_ARG;
  if (c->head_dim != D) return IQ_ERR_UNSUPPORTED;
  if (c->n_layers < 1 || c->n_kv_heads < 1 || c->page_size < TILE_TOKENS || c->page_size % TILE_TOKENS != 0 ||
      c->n_pages < 1)
    return IQ_ERR_INVALID_ARG;
  if (layer < 0 || layer >= c->n_layers) return IQ_ERR_INVALID_ARG;
  if (!c->pool) return IQ_ERR_INVALID_ARG;
  if (c->block_table_dev && c->max_pages_per_seq < 1) return IQ_ERR_INVALID_ARG;
  if (!supported_widths(k_bits(c), v_bits(c))) return IQ_ERR_UNSUPPORTED;
  if (c->rotation != IQ_ROT_ISO && c->rotation != IQ_ROT_QUAT && c->rotation != IQ_ROT_PLANAR) return IQ_ERR_UNSUPPORTED;
  if (!aligned(c->pool, 16)) return IQ_ERR_ALIGNMENT;
  return IQ_OK;
}

static size_t layer_pool_bytes(const iq_cache* c) {
  return (size_t)c->n_pages * c->n_kv_heads * (c->page_size / TILE_TOKENS) * tile_bytes(k_bits(c), v_bits(c));
}

static LayerView view(const iq_cache* c, int32_t layer) {
  LayerView v;
  v.pool = (uint8_t*)c->pool + layer_pool_bytes(c) * layer;
  v.block_table = c->block_table_dev;
  v.max_pages = c->block_table_dev ? c->max_pages_per_seq : 1;
  v.page_size = c->page_size;
  v.n_pages = c->n_pages;
  v.n_kv_heads = c->n_kv_heads;
  v.status = c->status_dev;
  v.kb = k_bits(c);
  v.vb = v_bits(c);
  v.rot = c->rotation;
  return v;
}

static const float* layer_params(const iq_cache* c, const float* params_dev, int32_t layer) {
  return params_dev + (size_t)layer * c->n_kv_heads * params_per_head(c->rotation);
}

static int64_t seq_capacity(const iq_cache* c) {
  return c->block_table_dev ? (int64_t)c->page_size * c->max_pages_per_seq : (int64_t)c->page_size;
}

}  // namespace iq

using namespace iq;

extern "C" {

const char* iq_version(void) { return "libiq 0.2 (sm_100a; packed 2/3/4-bit IsoQuant KV)"; }

const char* iq_status_string(iq_status s) {
  switch (s) {
    case IQ_OK: return "ok";
    case IQ_ERR_INVALID_ARG: return "invalid argument";
    case IQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case IQ_ERR_CAPACITY: return "size exceeds cache capacity";
    case IQ_ERR_WORKSPACE: return "workspace missing or too small";
    case IQ_ERR_ALIGNMENT: return "device pointer not aligned";
    case IQ_ERR_CUDA: return "CUDA launch or runtime error";
  }
  return "unknown status";
}

iq_status iq_cache_bytes(int32_t n_layers, int32_t n_kv_heads, int32_t page_size, int32_t n_pages, int32_t k_bits,
                         int32_t v_bits, size_t* pool_bytes_host) {
  if (n_layers < 1 || n_kv_heads < 1 || page_size < TILE_TOKENS || page_size % TILE_TOKENS != 0 || n_pages < 1)
    return IQ_ERR_INVALID_ARG;
  const int kb = k_bits ? k_bits : 3, vb = v_bits ? v_bits : 3;
  if (!supported_widths(kb, vb)) return IQ_ERR_UNSUPPORTED;
  if (pool_bytes_host)
    *pool_bytes_host = (size_t)n_layers * n_pages * n_kv_heads * (page_size / TILE_TOKENS) * tile_bytes(kb, vb);
  return IQ_OK;
}

iq_status iq_init_rotation(uint64_t seed, int32_t n_layers, int32_t n_kv_heads, float* params_host) {
  return iq_init_rotation_variant(seed, IQ_ROT_ISO, n_layers, n_kv_heads, params_host);
}

int32_t iq_rotation_params_per_head(int32_t rotation) {
  return (rotation == IQ_ROT_ISO || rotation == IQ_ROT_QUAT || rotation == IQ_ROT_PLANAR) ? params_per_head(rotation)
                                                                                         : 0;
}

iq_status iq_init_rotation_variant(uint64_t seed, int32_t rotation, int32_t n_layers, int32_t n_kv_heads,
                                   float* params_host) {
  if (!params_host || n_layers < 1 || n_kv_heads < 1) return IQ_ERR_INVALID_ARG;
  if (iq_rotation_params_per_head(rotation) == 0) return IQ_ERR_UNSUPPORTED;
  init_rotation_params(seed, rotation, n_layers, n_kv_heads, params_host);
  return IQ_OK;
}

iq_status iq_encode_append(const iq_cache* cache, int32_t layer, const void* k_dev, const void* v_dev,
                           int32_t batch, int32_t n_new, const int32_t* start_pos_dev,
                           const float* params_dev, iq_stream_t stream) {
  iq_status st = check_cache(cache, layer);
  if (st != IQ_OK) return st;
  if (batch < 0 || n_new < 0 || !start_pos_dev || !params_dev) return IQ_ERR_INVALID_ARG;
  if (!k_dev && !v_dev) return IQ_ERR_INVALID_ARG;
  if (!cache->block_table_dev && batch > cache->n_pages) return IQ_ERR_CAPACITY;
  if ((int64_t)n_new > seq_capacity(cache)) return IQ_ERR_CAPACITY;
  if ((k_dev && !aligned(k_dev, 16)) || (v_dev && !aligned(v_dev, 16)) || !aligned(params_dev, 16) ||
      !aligned(start_pos_dev, 4))
    return IQ_ERR_ALIGNMENT;
  const LayerView v = view(cache, layer);
  const int e = launch_encode(v, k_dev, v_dev, batch, n_new, start_pos_dev, layer_params(cache, params_dev, layer),
                              kernel_consts(v.kb, v.vb), stream);
  return e ? IQ_ERR_CUDA : IQ_OK;
}

size_t iq_decode_workspace_size(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int32_t max_ctx) {
  if (batch < 0 || n_q_heads < 0 || n_kv_heads < 1 || max_ctx < 0) return 0;
  return decode_workspace_bytes(batch, n_q_heads, n_kv_heads, max_ctx);
}

iq_status iq_decode_attention(const iq_cache* cache, int32_t layer, const void* q_dev, iq_dtype q_dtype,
                              int32_t batch, int32_t n_q_heads, const int32_t* ctx_len_dev, int32_t max_ctx,
                              const float* params_dev, float* out_dev, void* workspace_dev,
                              size_t workspace_bytes, iq_stream_t stream) {
  iq_status st = check_cache(cache, layer);
  if (st != IQ_OK) return st;
  if (batch < 0 || n_q_heads < 1 || max_ctx < 0 || !q_dev || !ctx_len_dev || !params_dev || !out_dev)
    return IQ_ERR_INVALID_ARG;
  if (q_dtype != IQ_F16 && q_dtype != IQ_F32) return IQ_ERR_UNSUPPORTED;
  if (batch > DECODE_MAX_BATCH) return IQ_ERR_UNSUPPORTED;
  if (n_q_heads % cache->n_kv_heads != 0) return IQ_ERR_INVALID_ARG;
  const int G = n_q_heads / cache->n_kv_heads;
  if (G < 1 || G > 8) return IQ_ERR_UNSUPPORTED;  // at most 8 query heads per kv head (one mma row block)
  if (!cache->block_table_dev && batch > cache->n_pages) return IQ_ERR_CAPACITY;
  if ((int64_t)max_ctx > seq_capacity(cache)) return IQ_ERR_CAPACITY;
  if (!aligned(q_dev, 16) || !aligned(out_dev, 16) || !aligned(params_dev, 16) || !aligned(ctx_len_dev, 4))
    return IQ_ERR_ALIGNMENT;
  const size_t need = decode_workspace_bytes(batch, n_q_heads, cache->n_kv_heads, max_ctx);
  if (!workspace_dev || workspace_bytes < need) return IQ_ERR_WORKSPACE;
  if (!aligned(workspace_dev, 256)) return IQ_ERR_ALIGNMENT;
  const LayerView v = view(cache, layer);
  const int e = launch_decode(v, q_dev, q_dtype == IQ_F32, batch, n_q_heads, ctx_len_dev, max_ctx,
                              layer_params(cache, params_dev, layer), out_dev, workspace_dev,
                              kernel_consts(v.kb, v.vb), stream);
  return e ? IQ_ERR_CUDA : IQ_OK;
}

iq_status iq_decode_step(const iq_cache* cache, int32_t layer, const void* q_dev, iq_dtype q_dtype,
                         const void* k_new_dev, const void* v_new_dev, int32_t batch, int32_t n_q_heads,
                         const int32_t* ctx_len_dev, int32_t max_ctx, const float* params_dev, float* out_dev,
                         void* workspace_dev, size_t workspace_bytes, iq_stream_t stream) {
  iq_status st = check_cache(cache, layer);
  if (st != IQ_OK) return st;
  if (batch < 0 || n_q_heads < 1 || max_ctx < 1 || !q_dev || !ctx_len_dev || !params_dev || !out_dev || !k_new_dev ||
      !v_new_dev)
    return IQ_ERR_INVALID_ARG;
  if (q_dtype != IQ_F16 && q_dtype != IQ_F32) return IQ_ERR_UNSUPPORTED;
  if (batch > DECODE_MAX_BATCH) return IQ_ERR_UNSUPPORTED;
  if (n_q_heads % cache->n_kv_heads != 0) return IQ_ERR_INVALID_ARG;
  const int G = n_q_heads / cache->n_kv_heads;
  if (G < 1 || G > 8) return IQ_ERR_UNSUPPORTED;  // at most 8 query heads per kv head (one mma row block)
  if (!cache->block_table_dev && batch > cache->n_pages) return IQ_ERR_CAPACITY;
  if ((int64_t)max_ctx > seq_capacity(cache)) return IQ_ERR_CAPACITY;
  if (!aligned(q_dev, 16) || !aligned(out_dev, 16) || !aligned(params_dev, 16) || !aligned(ctx_len_dev, 4) ||
      !aligned(k_new_dev, 16) || !aligned(v_new_dev, 16))
    return IQ_ERR_ALIGNMENT;
  const size_t need = decode_workspace_bytes(batch, n_q_heads, cache->n_kv_heads, max_ctx);
  if (!workspace_dev || workspace_bytes < need) return IQ_ERR_WORKSPACE;
  if (!aligned(workspace_dev, 256)) return IQ_ERR_ALIGNMENT;
  const LayerView v = view(cache, layer);
  const int e = launch_decode_step(v, q_dev, q_dtype == IQ_F32, k_new_dev, v_new_dev, batch, n_q_heads, ctx_len_dev,
                                   max_ctx, layer_params(cache, params_dev, layer), out_dev, workspace_dev,
                                   kernel_consts(v.kb, v.vb), stream);
  return e ? IQ_ERR_CUDA : IQ_OK;
}

size_t iq_decode_deferred_workspace_size(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int32_t max_ctx,
                                         int32_t max_len) {
  if (batch < 0 || n_q_heads < 0 || n_kv_heads < 1 || max_ctx < 0 || max_len < 0) return 0;
  const int extra = batch * n_kv_heads * prefix_splits(batch, n_kv_heads, max_len, sm_count());
  return decode_workspace_bytes(batch, n_q_heads, n_kv_heads, max_ctx, extra);
}

iq_status iq_decode_step_deferred(const iq_cache* cache, int32_t layer, const iq_fp16_prefix* prefix, const void* q_dev,
                                  iq_dtype q_dtype, const void* k_new_dev, const void* v_new_dev, int32_t batch,
                                  int32_t n_q_heads, const int32_t* ctx_len_dev, int32_t max_ctx,
                                  const float* params_dev, float* out_dev, void* workspace_dev, size_t workspace_bytes,
                                  iq_stream_t stream) {
  iq_status st = check_cache(cache, layer);
  if (st != IQ_OK) return st;
  if (!prefix || !prefix->k_dev || !prefix->v_dev || !prefix->len_dev || prefix->max_len < 0) return IQ_ERR_INVALID_ARG;
  if (batch < 0 || n_q_heads < 1 || max_ctx < 1 || !q_dev || !ctx_len_dev || !params_dev || !out_dev || !k_new_dev ||
      !v_new_dev)
    return IQ_ERR_INVALID_ARG;
  if (q_dtype != IQ_F16 && q_dtype != IQ_F32) return IQ_ERR_UNSUPPORTED;
  if (batch > DECODE_MAX_BATCH) return IQ_ERR_UNSUPPORTED;
  if (n_q_heads % cache->n_kv_heads != 0) return IQ_ERR_INVALID_ARG;
  const int G = n_q_heads / cache->n_kv_heads;
  if (G < 1 || G > 8) return IQ_ERR_UNSUPPORTED;  // at most 8 query heads per kv head (one mma row block)
  if (!cache->block_table_dev && batch > cache->n_pages) return IQ_ERR_CAPACITY;
  if ((int64_t)max_ctx > seq_capacity(cache)) return IQ_ERR_CAPACITY;
  if (!aligned(q_dev, 16) || !aligned(out_dev, 16) || !aligned(params_dev, 16) || !aligned(ctx_len_dev, 4) ||
      !aligned(k_new_dev, 16) || !aligned(v_new_dev, 16) || !aligned(prefix->k_dev, 16) ||
      !aligned(prefix->v_dev, 16) || !aligned(prefix->len_dev, 4))
    return IQ_ERR_ALIGNMENT;
  const size_t need = iq_decode_deferred_workspace_size(batch, n_q_heads, cache->n_kv_heads, max_ctx, prefix->max_len);
  if (!workspace_dev || workspace_bytes < need) return IQ_ERR_WORKSPACE;
  if (!aligned(workspace_dev, 256)) return IQ_ERR_ALIGNMENT;
  const LayerView v = view(cache, layer);
  const int e = launch_decode_deferred(v, q_dev, q_dtype == IQ_F32, k_new_dev, v_new_dev, batch, n_q_heads, ctx_len_dev,
                                       max_ctx, layer_params(cache, params_dev, layer), out_dev, workspace_dev,
                                       kernel_consts(v.kb, v.vb), stream, prefix->k_dev, prefix->v_dev,
                                       prefix->len_dev, prefix->max_len);
  return e ? IQ_ERR_CUDA : IQ_OK;
}

size_t iq_prefill_workspace_size(int32_t batch, int32_t n_tokens, int32_t n_kv_heads, int32_t max_ctx) {
  if (batch < 0 || n_tokens < 0 || n_kv_heads < 1 || max_ctx < 0) return 0;
  return prefill_workspace_bytes(batch, n_tokens, n_kv_heads, max_ctx);
}

iq_status iq_prefill_attention(const iq_cache* cache, int32_t layer, const void* q_dev, iq_dtype q_dtype, int32_t batch,
                               int32_t n_tokens, int32_t n_q_heads, const int32_t* start_pos_dev, int32_t max_ctx,
                               const float* params_dev, float* out_dev, void* workspace_dev, size_t workspace_bytes,
                               iq_stream_t stream) {
  iq_status st = check_cache(cache, layer);
  if (st != IQ_OK) return st;
  if (batch < 0 || n_tokens < 0 || n_q_heads < 1 || max_ctx < n_tokens || !q_dev || !start_pos_dev || !params_dev ||
      !out_dev)
    return IQ_ERR_INVALID_ARG;
  if (q_dtype != IQ_F16 && q_dtype != IQ_F32) return IQ_ERR_UNSUPPORTED;
  if (n_q_heads % cache->n_kv_heads != 0) return IQ_ERR_INVALID_ARG;
  const int G = n_q_heads / cache->n_kv_heads;
  if (G < 1 || G > 8) return IQ_ERR_UNSUPPORTED;  // at most 8 query heads per kv head (one mma row block)
  if (!cache->block_table_dev && batch > cache->n_pages) return IQ_ERR_CAPACITY;
  if ((int64_t)max_ctx > seq_capacity(cache)) return IQ_ERR_CAPACITY;
  if ((int64_t)batch * cache->n_kv_heads * ((n_tokens + 7) / 8) > (int64_t)1 << 24) return IQ_ERR_UNSUPPORTED;
  if (!aligned(q_dev, 16) || !aligned(out_dev, 16) || !aligned(params_dev, 16) || !aligned(start_pos_dev, 4))
    return IQ_ERR_ALIGNMENT;
  const size_t need = prefill_workspace_bytes(batch, n_tokens, cache->n_kv_heads, max_ctx);
  if (batch > 0 && n_tokens > 0 && (!workspace_dev || workspace_bytes < need)) return IQ_ERR_WORKSPACE;
  if (workspace_dev && !aligned(workspace_dev, 256)) return IQ_ERR_ALIGNMENT;
  const LayerView v = view(cache, layer);
  const int e = launch_prefill(v, q_dev, q_dtype == IQ_F32, batch, n_tokens, n_q_heads, start_pos_dev, max_ctx,
                               layer_params(cache, params_dev, layer), out_dev, workspace_dev,
                               kernel_consts(v.kb, v.vb), stream);
  return e ? IQ_ERR_CUDA : IQ_OK;
}

iq_status iq_export_codes(const iq_cache* cache, int32_t layer, int32_t kv, int32_t seq, int32_t t0, int32_t n,
                          uint8_t* codes_dev, uint16_t* norms_dev, iq_stream_t stream) {
  iq_status st = check_cache(cache, layer);
  if (st != IQ_OK) return st;
  if ((kv != 0 && kv != 1) || seq < 0 || t0 < 0 || n < 0 || !codes_dev) return IQ_ERR_INVALID_ARG;
  if (!cache->block_table_dev && seq >= cache->n_pages) return IQ_ERR_CAPACITY;
  if ((int64_t)t0 + n > seq_capacity(cache)) return IQ_ERR_CAPACITY;
  const LayerView v = view(cache, layer);
  const int e = launch_export(v, kv, seq, t0, n, codes_dev, norms_dev, stream);
  return e ? IQ_ERR_CUDA : IQ_OK;
}

}  // extern "C"
