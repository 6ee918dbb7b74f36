// Deferred quantisation: decode attention over a cache whose first tokens are still fp16.
//
// "RotorQuant" (sd114.wiki), section "2. 延迟量化策略", and "压缩与速度的博弈" (zhichai.net), section
// "延迟量化（Deferred Quantization）": during prompt processing the K/V cache stays fp16 (no
// rotation, no quantisation); tokens generated during decoding are quantised when they are
// inserted.  So a decode step attends over an fp16 prefix (positions 0 .. len-1 of each sequence,
// unrotated, as the model produced them) and the packed tail (positions len .. ctx-1, the new
// token appended and quantised by the same step).
//
// Two kernels per call.  prefix_kernel computes, on CUDA cores in fp32, the attention of every
// query head of a kv head over a split of the fp16 prefix, exactly (fp16 inputs, fp32 products
// and sums): online softmax over 32-token tiles in shared memory, then the value sum rotated
// forward (R) and scaled to the packed kernel's units, written as extra split partials.  The
// fused decode step (decode_kernel) then appends the new token, attends over the packed tiles
// from the prefix's tile onward (positions below len masked) and merges its own partials with
// the extra ones before the single inverse rotation.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <algorithm>
#include <mutex>

#include "iq_decode_impl.cuh"

namespace iq {

constexpr int PX_THREADS = 256;
constexpr int PX_ROW = D + 8;  // halves per token row in shared memory (16-byte rows, staggered banks)

struct PrefixArgs {
  const __half* k;  // [batch][Hkv][max_len][128]
  const __half* v;
  const int32_t* len;      // [batch]
  const int32_t* ctx_len;  // [batch]
  int max_len, max_ctx;
  const void* q;
  int q_f32, batch, n_q_heads, g_real, n_kv_heads, splits, rot;
  const float* params_layer;
  float alpha_v;
  float2* part_ml;
  float* part_o;
  int extra_base;
  uint32_t* status;
};

__global__ void __launch_bounds__(PX_THREADS) prefix_kernel(PrefixArgs a) {
  // wait before letting the decode kernel start, so that the kernel before this one is the only
  // one the decode kernel's early reads can overlap
  pdl_wait();
  pdl_launch_dependents();
  constexpr int R_MAX = 8;
  __shared__ __align__(16) float sq[HMAX][D];
  __shared__ float sml[R_MAX][HMAX][2];
  __shared__ float sprm[256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.g_real, R = HMAX / G;  // warp w: head w % G, replica w / G
  // dynamic: R K tiles then R V tiles, [R][32][PX_ROW] halves each
  extern __shared__ __align__(16) uint8_t px_smem[];
  __half(*sk)[TT][PX_ROW] = reinterpret_cast<__half(*)[TT][PX_ROW]>(px_smem);
  __half(*sv)[TT][PX_ROW] = reinterpret_cast<__half(*)[TT][PX_ROW]>(px_smem + (size_t)R * TT * PX_ROW * 2);
  const int gid = blockIdx.x / a.splits, split = blockIdx.x % a.splits;
  const int b = gid / a.n_kv_heads, kvh = gid % a.n_kv_heads;
  // prefix length, clamped as the decode kernel clamps it (0 <= len < ctx)
  int c = a.ctx_len[b];
  c = c < 0 ? 0 : (c > a.max_ctx ? a.max_ctx : c);
  int p = a.len[b];
  p = p < 0 ? 0 : ((c > 0 && p >= c) ? max(c - 1, 0) : p);
  if (p > a.max_len) {
    if (a.status && split == 0 && kvh == 0 && threadIdx.x == 0) atomicOr(a.status, IQ_DEVERR_CTX);
    p = a.max_len;
  }
  const int ntiles = (p + TT - 1) / TT;
  const int t_lo = (int)((long long)split * ntiles / a.splits), t_hi = (int)((long long)(split + 1) * ntiles / a.splits);

  // queries of the group, scaled so that q.k gives scores in log2 units: log2(e) / sqrt(128)
  const float qs = kLog2e * 0.08838834764831845f;
  for (int i = threadIdx.x; i < HMAX * D; i += PX_THREADS) {
    const int h = i / D, x = i % D;
    float val = 0.f;
    if (h < G) {
      const size_t row = ((size_t)b * a.n_q_heads + (size_t)kvh * G + h) * D + x;
      val = a.q_f32 ? ((const float*)a.q)[row] : __half2float(((const __half*)a.q)[row]);
    }
    sq[h][x] = val * qs;
  }
  if (threadIdx.x < params_per_head(a.rot) / 4)
    reinterpret_cast<float4*>(sprm)[threadIdx.x] =
        reinterpret_cast<const float4*>(a.params_layer + (size_t)kvh * params_per_head(a.rot))[threadIdx.x];

  const int h = warp % G, r = warp / G;
  float m = -CUDART_INF_F, l = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
  const size_t seq_base = ((size_t)b * a.n_kv_heads + kvh) * a.max_len;
  for (int base = t_lo; base < t_hi; base += R) {
    __syncthreads();  // the previous tiles are consumed (and sq, sprm written, on the first pass)
    // the R tiles base .. base+R-1: rows of 16-byte pieces, all threads
    for (int i = threadIdx.x; i < R * TT * (D / 8); i += PX_THREADS) {
      const int rr = i / (TT * (D / 8)), t = (i / (D / 8)) % TT, piece = i % (D / 8);
      const int pos = TT * (base + rr) + t;
      uint4 kk = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
      if (base + rr < t_hi && pos < p) {
        kk = reinterpret_cast<const uint4*>(a.k + (seq_base + pos) * D)[piece];
        vv = reinterpret_cast<const uint4*>(a.v + (seq_base + pos) * D)[piece];
      }
      *reinterpret_cast<uint4*>(&sk[rr][t][8 * piece]) = kk;
      *reinterpret_cast<uint4*>(&sv[rr][t][8 * piece]) = vv;
    }
    __syncthreads();
    const int tile = base + r;
    if (tile < t_hi) {
      // score of token `lane`: coordinates visited from a lane-dependent start (no bank conflicts)
      float s = 0.f;
#pragma unroll 8
      for (int c2 = 0; c2 < D / 2; ++c2) {
        const int x = 2 * ((c2 + lane) & (D / 2 - 1));
        const float2 kf = __half22float2(*reinterpret_cast<const __half2*>(&sk[r][lane][x]));
        s = fmaf(sq[h][x], kf.x, s);
        s = fmaf(sq[h][x + 1], kf.y, s);
      }
      const int pos = TT * tile + lane;
      if (pos >= p) s = -CUDART_INF_F;
      float mx = s;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_new = fmaxf(m, mx);
      const float sc = (m == -CUDART_INF_F) ? 0.f : exp2f(m - m_new);
      const float pw = (s == -CUDART_INF_F) ? 0.f : exp2f(s - m_new);
      float ps = pw;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
      l = l * sc + ps;
      m = m_new;
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] *= sc;
      // values: lane holds coordinates 4 lane .. 4 lane + 3
#pragma unroll 4
      for (int t = 0; t < TT; ++t) {
        const float pt = __shfl_sync(0xffffffffu, pw, t);
        const uint2 raw = *reinterpret_cast<const uint2*>(&sv[r][t][4 * lane]);
        const float2 v0 = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
        const float2 v1 = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
        acc[0] = fmaf(pt, v0.x, acc[0]);
        acc[1] = fmaf(pt, v0.y, acc[1]);
        acc[2] = fmaf(pt, v1.x, acc[2]);
        acc[3] = fmaf(pt, v1.y, acc[3]);
      }
    }
  }
  // merge the replicas of each head (shared memory), then R, scale and write the partial
  __syncthreads();
  float* so = reinterpret_cast<float*>(&sk[0][0][0]);  // [R][G][128] floats, reused
  if (lane == 0) {
    sml[r][h][0] = m;
    sml[r][h][1] = l;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) so[(r * G + h) * D + 4 * lane + i] = acc[i];
  __syncthreads();
  if (r == 0) {
    float M = -CUDART_INF_F;
    for (int rr = 0; rr < R; ++rr) M = fmaxf(M, sml[rr][h][0]);
    float L = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
    for (int rr = 0; rr < R; ++rr) {
      const float mr = sml[rr][h][0];
      if (mr == -CUDART_INF_F) continue;
      const float w = exp2f(mr - M);
      L = fmaf(sml[rr][h][1], w, L);
#pragma unroll
      for (int i = 0; i < 4; ++i) o[i] = fmaf(so[(rr * G + h) * D + 4 * lane + i], w, o[i]);
    }
    // into the packed kernel's basis and units: R o, times alpha_v sqrt(128)
    float Mp[4][4];
    variant_block_matrix(a.rot, sprm + lane * params_per_block(a.rot), Mp);
    warp_rotate_forward(o, Mp, a.rot == ROT_ISO);
    const float unit = a.alpha_v * 11.313708498984761f;  // alpha_v * sqrt(128)
    const size_t slot = (size_t)a.extra_base + (size_t)gid * a.splits + split;
    reinterpret_cast<float4*>(a.part_o + (slot * HMAX + h) * D)[lane] =
        make_float4(o[0] * unit, o[1] * unit, o[2] * unit, o[3] * unit);
    if (lane == 0) a.part_ml[slot * HMAX + h] = make_float2(M, L);
  }
}

int prefix_splits(int batch, int n_kv_heads, int max_len, int n_sm) {
  const int groups = std::max(1, batch * n_kv_heads);
  int s = (2 * n_sm + groups - 1) / groups;
  s = std::min(s, std::max(1, (max_len + TT - 1) / TT / 2));
  return std::max(1, std::min(s, 64));
}

int launch_prefix(const LayerView& v, const void* k16, const void* v16, const int32_t* len, int max_len,
                  const int32_t* ctx_len, int max_ctx, const void* q, int q_f32, int batch, int n_q_heads,
                  const float* params_layer, const KernelConsts& kc, void* workspace, int splits, int extra_base,
                  void* stream) {
  if (batch == 0) return 0;
  PrefixArgs a;
  a.k = (const __half*)k16;
  a.v = (const __half*)v16;
  a.len = len;
  a.ctx_len = ctx_len;
  a.max_len = max_len;
  a.max_ctx = max_ctx;
  a.q = q;
  a.q_f32 = q_f32;
  a.batch = batch;
  a.n_q_heads = n_q_heads;
  a.g_real = n_q_heads / v.n_kv_heads;
  a.n_kv_heads = v.n_kv_heads;
  a.splits = splits;
  a.rot = v.rot;
  a.params_layer = params_layer;
  a.alpha_v = kc.v.alpha8;
  const Workspace w = carve_workspace(workspace, batch, v.n_kv_heads, batch * v.n_kv_heads * splits);
  a.part_ml = w.part_ml;
  a.part_o = w.part_o;
  a.extra_base = extra_base;
  a.status = v.status;
  const size_t smem = (size_t)(HMAX / a.g_real) * 2 * TT * PX_ROW * sizeof(__half);
  static std::once_flag once;
  std::call_once(once, [] {
    cudaFuncSetAttribute(prefix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, HMAX * 2 * TT * PX_ROW * 2);
  });
  return (int)launch_pdl(prefix_kernel, dim3(batch * v.n_kv_heads * splits), dim3(PX_THREADS), smem,
                         (cudaStream_t)stream, a);
}

}  // namespace iq
