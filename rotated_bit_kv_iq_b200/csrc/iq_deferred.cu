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
// and sums): 32-token K and V tiles stream into shared memory by bulk copies, two rounds in
// flight, each warp keeping the online softmax of one head over one stream of tiles; the value
// sum is rotated forward (R) and scaled to the packed kernel's units, and written as extra split
// partials.  The
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
constexpr int PX_NB = 2;       // rounds of tiles in flight
constexpr int PX_RMAX = 4;     // replicas (tile streams) per CTA
constexpr int PX_TILE = TT * D * 2;  // bytes of one fp16 tile (32 tokens x 128)

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

// Replicas: tile streams per CTA; warp w works on head w % G of stream w / G.
__host__ __device__ inline int px_replicas(int G) { return (HMAX / G) < PX_RMAX ? (HMAX / G) : PX_RMAX; }

__global__ void __launch_bounds__(PX_THREADS) prefix_kernel(PrefixArgs a) {
  // Wait before letting the decode kernel start: it reads q and the new token (through L2)
  // before its own wait, relying on the kernel before this one having completed by then.
  pdl_wait();
  pdl_launch_dependents();
  __shared__ __align__(16) float sq[HMAX][D];
  __shared__ float sml[PX_RMAX][HMAX][2];
  __shared__ float sprm[256];
  __shared__ __align__(8) uint64_t bars[PX_NB][PX_RMAX];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.g_real, R = px_replicas(G);
  const int h = warp % G, r = warp / G;  // r >= R: idle warp (group size 1 only)
  // dynamic: [PX_NB][R] K tiles, then [PX_NB][R] V tiles, each [32][128] halves as stored
  extern __shared__ __align__(128) uint8_t px_smem[];
  auto ktile = [&](int buf, int rr) { return reinterpret_cast<__half*>(px_smem + (size_t)(buf * R + rr) * PX_TILE); };
  auto vtile = [&](int buf, int rr) {
    return reinterpret_cast<__half*>(px_smem + (size_t)(PX_NB * R + buf * R + rr) * PX_TILE);
  };
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
  const int n_rounds = (t_hi - t_lo + R - 1) / R;
  const size_t seq_base = ((size_t)b * a.n_kv_heads + kvh) * a.max_len;

  if (threadIdx.x == 0) {
    for (int i = 0; i < PX_NB; ++i)
      for (int rr = 0; rr < R; ++rr) mbar_init(&bars[i][rr], 1);
    mbar_fence_init();
  }
  __syncthreads();
  // round rd: tiles t_lo + rd R + rr, rr < R; each K and V tile is one bulk copy of its valid rows
  auto issue_round = [&](int rd) {
    const int buf = rd % PX_NB;
    for (int rr = 0; rr < R; ++rr) {
      const int tile = t_lo + rd * R + rr;
      const int rows = tile < t_hi ? min(TT, p - TT * tile) : 0;
      mbar_arrive_expect_tx(&bars[buf][rr], 2u * rows * D * 2);
      if (rows > 0) {
        bulk_g2s(ktile(buf, rr), a.k + (seq_base + (size_t)TT * tile) * D, rows * D * 2, &bars[buf][rr]);
        bulk_g2s(vtile(buf, rr), a.v + (seq_base + (size_t)TT * tile) * D, rows * D * 2, &bars[buf][rr]);
      }
    }
  };
  if (threadIdx.x == 0)
    for (int rd = 0; rd < min(PX_NB, n_rounds); ++rd) issue_round(rd);

  // queries of the group, scaled so that q.k gives scores in log2 units: log2(e) / sqrt(128)
  const float qs = kLog2e * 0.08838834764831845f;
  for (int i = threadIdx.x; i < HMAX * D; i += PX_THREADS) {
    const int hh = i / D, x = i % D;
    float val = 0.f;
    if (hh < G) {
      const size_t row = ((size_t)b * a.n_q_heads + (size_t)kvh * G + hh) * D + x;
      val = a.q_f32 ? ((const float*)a.q)[row] : __half2float(((const __half*)a.q)[row]);
    }
    sq[hh][x] = val * qs;
  }
  if (threadIdx.x < params_per_head(a.rot) / 4)
    reinterpret_cast<float4*>(sprm)[threadIdx.x] =
        reinterpret_cast<const float4*>(a.params_layer + (size_t)kvh * params_per_head(a.rot))[threadIdx.x];
  __syncthreads();

  float m = -CUDART_INF_F, l = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
  bool ok = true;
  for (int rd = 0; rd < n_rounds; ++rd) {
    const int buf = rd % PX_NB, tile = t_lo + rd * R + r;
    if (r < R && tile < t_hi) {
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[buf][r], (rd / PX_NB) & 1, a.status));
      const int n_valid = min(TT, p - TT * tile);  // rows of this tile in the prefix
      const __half* kt = ktile(buf, r);
      const __half* vt = vtile(buf, r);
      if (ok) {
        // score of token `lane`: coordinates visited from a lane-dependent start, so the 32 lanes
        // read 32 different banks of their 256-byte rows
        float s = 0.f;
#pragma unroll 8
        for (int c2 = 0; c2 < D / 2; ++c2) {
          const int x = 2 * ((c2 + lane) & (D / 2 - 1));
          const float2 kf = __half22float2(*reinterpret_cast<const __half2*>(kt + lane * D + x));
          const float2 qv = *reinterpret_cast<const float2*>(&sq[h][x]);
          s = fmaf(qv.x, kf.x, s);
          s = fmaf(qv.y, kf.y, s);
        }
        if (lane >= n_valid) s = -CUDART_INF_F;  // rows past the prefix were not copied
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
        // values: lane holds coordinates 4 lane .. 4 lane + 3; only the copied rows are read
        for (int t = 0; t < n_valid; ++t) {
          const float pt = __shfl_sync(0xffffffffu, pw, t);
          const uint2 raw = *reinterpret_cast<const uint2*>(vt + t * D + 4 * lane);
          const float2 v0 = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
          const float2 v1 = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
          acc[0] = fmaf(pt, v0.x, acc[0]);
          acc[1] = fmaf(pt, v0.y, acc[1]);
          acc[2] = fmaf(pt, v1.x, acc[2]);
          acc[3] = fmaf(pt, v1.y, acc[3]);
        }
      }
    }
    __syncthreads();  // every stream is done with buffer buf
    if (threadIdx.x == 0 && rd + PX_NB < n_rounds) issue_round(rd + PX_NB);
  }
  // leave no bulk copy in flight (only after a timed-out wait can one be pending)
  if (!__syncthreads_and(ok) && threadIdx.x == 0)
    for (int rd = 0; rd < n_rounds; ++rd)
      for (int rr = 0; rr < R; ++rr)
        if (t_lo + rd * R + rr < t_hi) mbar_wait(&bars[rd % PX_NB][rr], (rd / PX_NB) & 1, nullptr);
  // merge the streams of each head (shared memory), then R, scale and write the partial
  __syncthreads();
  float* so = reinterpret_cast<float*>(px_smem);  // [R][G][128] floats, over the tile buffers
  if (r < R) {
    if (lane == 0) {
      sml[r][h][0] = m;
      sml[r][h][1] = l;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) so[(r * G + h) * D + 4 * lane + i] = acc[i];
  }
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
  const size_t smem = (size_t)2 * PX_NB * px_replicas(a.g_real) * PX_TILE;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaFuncSetAttribute(prefix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 2 * PX_NB * PX_RMAX * PX_TILE);
  });
  return (int)launch_pdl(prefix_kernel, dim3(batch * v.n_kv_heads * splits), dim3(PX_THREADS), smem,
                         (cudaStream_t)stream, a);
}

}  // namespace iq
