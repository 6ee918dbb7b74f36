// Decode attention directly on the packed 3-bit cache.
//
// "RotaryQuant" (rebasdaily.com, section "妙处不只是压缩，而是不再展开") and its abstract
// (arXiv 2608.08081): queries are matched against packed keys, softmax is taken, values are
// accumulated from the packed values, and the inverse rotation is applied at the end;
// full-precision K/V are never built.  "RotorQuant" (sd114.wiki, "3. V 缓存的逆旋转修复"):
// the value sum must be mapped back with the inverse rotation.
//
// Kernel 1 (split): grid (split, kv head, sequence).  Each CTA rotates the G = Hq/Hkv
// queries of its kv head once (WHT + SO(4), one warp per query), then its warps walk
// 16-token tiles of the CTA's context range.  Per tile one warp:
//   * loads 48-byte K records of 16 tokens and 96-byte V records of 8 token pairs,
//   * turns codes into binary16 centroid values with byte-permute table lookups
//     (levels are stored scaled by alpha so that all eight are within 2e-5 of a binary16),
//   * scores all G heads at once on the tensor cores: mma.m16n8k16 with the 16 tokens as
//     M, the 128 rotated coordinates as K and (head, hi/lo half of q) as N,
//   * runs the online softmax (running max, rescale on increase) with warp shuffles,
//   * accumulates sum_t p_t n_v,t c[codes] with a second mma (coordinates as M, tokens as
//     K, heads as N); P reaches the B-operand layout through movmatrix.
// Warps merge (m, l, acc) in shared memory; the CTA writes one partial per query head.
// Kernel 2 (combine): merges the splits, divides by l, rescales and applies R^T.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "iq_device.cuh"

namespace iq {

constexpr int DEC_WARPS = 8;
constexpr float kLog2e = 1.4426950408889634f;

struct Workspace {
  float* part_o;   // [batch][Hq][n_split][128]
  float2* part_ml; // [batch][Hq][n_split] (max in log2 units, sum of exp2)
};

static inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

SplitPlan plan_splits(int batch, int n_kv_heads, int max_ctx) {
  SplitPlan p;
  const int groups = batch * n_kv_heads;
  const int target_ctas = 2 * 148;
  int want = (target_ctas + groups - 1) / groups;
  if (want < 1) want = 1;
  int chunk = (max_ctx + want - 1) / want;
  chunk = (chunk + 15) / 16 * 16;
  if (chunk < 16 * DEC_WARPS * 2) chunk = 16 * DEC_WARPS * 2;
  p.chunk = chunk;
  p.n_split = max_ctx > 0 ? (max_ctx + chunk - 1) / chunk : 1;
  return p;
}

size_t decode_workspace_bytes(int batch, int n_q_heads, int n_kv_heads, int max_ctx) {
  SplitPlan p = plan_splits(batch, n_kv_heads, max_ctx);
  const size_t rows = (size_t)batch * n_q_heads * p.n_split;
  return align256(rows * D * sizeof(float)) + align256(rows * sizeof(float2));
}

static Workspace carve(void* ws, int batch, int n_q_heads, int n_split) {
  Workspace w;
  const size_t rows = (size_t)batch * n_q_heads * n_split;
  w.part_o = (float*)ws;
  w.part_ml = (float2*)((char*)ws + align256(rows * D * sizeof(float)));
  return w;
}

__device__ __forceinline__ int clamp_ctx(int c, int max_ctx, uint32_t* status) {
  if (c < 0 || c > max_ctx) {
    if (status && threadIdx.x == 0) atomicOr(status, IQ_DEVERR_CTX);
    c = c < 0 ? 0 : max_ctx;
  }
  return c;
}

// G: kernel layout width (4 or 8 query heads per kv head); g_real <= G query heads exist
// (group sizes 1 and 2 run on the 4-wide layout with the unused columns zero).
template <int G>
__global__ void __launch_bounds__(DEC_WARPS * 32)
decode_split_kernel(LayerView v, const void* __restrict__ q, int q_f32, int n_q_heads, int g_real,
                    const int32_t* __restrict__ ctx_len, int max_ctx, int chunk, int n_split,
                    const float* __restrict__ params_layer, Workspace ws, KernelConsts kc) {
  constexpr int NT = G / 4;  // score n-tiles
  __shared__ float sq[G][D];
  __shared__ float so[DEC_WARPS][G][D];
  __shared__ float sm[DEC_WARPS][G];
  __shared__ float sl[DEC_WARPS][G];

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;
  const int ctx = clamp_ctx(ctx_len[b], max_ctx, v.status);
  const int t_begin = split * chunk;
  if (t_begin >= ctx) return;  // uniform over the CTA
  const int t_end = min(t_begin + chunk, ctx);

  // ---- rotate the G queries of this kv head (one warp per query) and scale them so that
  // score_log2 = n_k * <q', alpha*c[codes]>:  q' = R q * log2(e) / (128 * alpha).
  {
    float Mp[4][4];
    fused_block_matrix(params_layer + ((size_t)kvh * NBLK + lane) * 8, Mp);
    for (int h = warp; h < G; h += DEC_WARPS) {
      const size_t row = ((size_t)b * n_q_heads + (size_t)kvh * g_real + h) * D + 4 * lane;
      float x[4] = {0.f, 0.f, 0.f, 0.f};
      if (h >= g_real) {
        // no such query head: zero column
      } else if (q_f32) {
        const float4 f = *reinterpret_cast<const float4*>((const float*)q + row);
        x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
      } else {
        const uint2 u = *reinterpret_cast<const uint2*>((const __half*)q + row);
        const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
        const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
        x[0] = f0.x; x[1] = f0.y; x[2] = f1.x; x[3] = f1.y;
      }
      warp_rotate_forward(x, Mp);
      const float s = kLog2e * kc.inv_alpha * (1.0f / 128.0f);
#pragma unroll
      for (int i = 0; i < 4; ++i) sq[h][4 * lane + i] = x[i] * s;
    }
  }
  __syncthreads();

  // ---- query B-fragments (k16 x n8 per k-chunk c): MMA k index 2tq+e <-> coordinate
  // 32tq+4c+e, k index 2tq+8+e <-> 32tq+4c+2+e.  Columns: G=4 -> (head n/2, hi|lo = n%2);
  // G=8 -> tile 0 = hi halves of heads 0..7, tile 1 = lo halves.
  uint32_t qb[NT][8][2];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int head = (G == 4) ? (g >> 1) : g;
      const bool lo_part = (G == 4) ? (g & 1) : (nt == 1);
      float vals[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x = sq[head][32 * tq + 4 * c + e];
        const float hi = __half2float(__float2half_rn(x));
        vals[e] = lo_part ? (x - hi) : x;
      }
      qb[nt][c][0] = pack_half2(vals[0], vals[1]);
      qb[nt][c][1] = pack_half2(vals[2], vals[3]);
    }
  }

  constexpr int HS = G / 4;  // head slots per thread: G=4 -> head tq; G=8 -> heads 2tq, 2tq+1
  float m_run[HS], l_run[HS];
  float acc[8][4];
#pragma unroll
  for (int s = 0; s < HS; ++s) { m_run[s] = -CUDART_INF_F; l_run[s] = 0.f; }
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[j][i] = 0.f;

  const uint32_t lut_lo[2] = {kc.lut_lo[0], kc.lut_lo[1]};
  const uint32_t lut_hi[2] = {kc.lut_hi[0], kc.lut_hi[1]};

  for (int t0 = t_begin + 16 * warp; t0 < t_end; t0 += 16 * DEC_WARPS) {
    // ---- locate the tile (16 tokens, one page)
    int page = resolve_page(v, b, t0);
    if (page < 0) continue;
    const int s0 = t0 % v.page_size;
    const size_t hs = (size_t)page * v.n_kv_heads + kvh;
    const uint8_t* kp = v.k_codes + (hs * v.page_size + s0) * K_REC;
    const uint8_t* vp = v.v_codes + (hs * (v.page_size / 2) + s0 / 2) * V_REC;
    const uint16_t* knp = v.k_norms + hs * v.page_size + s0;
    const uint16_t* vnp = v.v_norms + hs * v.page_size + s0;

    const uint32_t* kA = reinterpret_cast<const uint32_t*>(kp + g * K_REC + tq * 12);
    const uint32_t* kB = reinterpret_cast<const uint32_t*>(kp + (g + 8) * K_REC + tq * 12);
    const uint32_t* vA = reinterpret_cast<const uint32_t*>(vp + tq * V_REC + g * 12);
    const uint32_t* vB = reinterpret_cast<const uint32_t*>(vp + (4 + tq) * V_REC + g * 12);
    const uint32_t ka0 = __ldg(kA), ka1 = __ldg(kA + 1), ka2 = __ldg(kA + 2);
    const uint32_t kb0 = __ldg(kB), kb1 = __ldg(kB + 1), kb2 = __ldg(kB + 2);
    const uint32_t va0 = __ldg(vA), va1 = __ldg(vA + 1), va2 = __ldg(vA + 2);
    const uint32_t vb0 = __ldg(vB), vb1 = __ldg(vB + 1), vb2 = __ldg(vB + 2);
    const bool okA = t0 + g < t_end, okB = t0 + g + 8 < t_end;
    const float nkA = half_bits_to_float(__ldg(knp + g)), nkB = half_bits_to_float(__ldg(knp + g + 8));
    const float nvA = half_bits_to_float(__ldg(vnp + g)), nvB = half_bits_to_float(__ldg(vnp + g + 8));

    // ---- scores: S[token][col] over 8 k-chunks
    float sc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) sc[nt][i] = 0.f;
    {
      uint32_t selA[4], selB[4];
      chunk_selectors(ka0, ka1, ka2, selA);
      chunk_selectors(kb0, kb1, kb2, selB);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t sA = (c & 1) ? (selA[c >> 1] >> 16) : selA[c >> 1];
        const uint32_t sB = (c & 1) ? (selB[c >> 1] >> 16) : selB[c >> 1];
        uint32_t lA, hA, lB, hB;
        lut4(sA, lut_lo, lut_hi, lA, hA);
        lut4(sB, lut_lo, lut_hi, lB, hB);
        const uint32_t a0 = pair01(lA, hA), a2 = pair23(lA, hA);
        const uint32_t a1 = pair01(lB, hB), a3 = pair23(lB, hB);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma16816(sc[nt], a0, a1, a2, a3, qb[nt][c][0], qb[nt][c][1]);
      }
    }

    // ---- online softmax per head slot; s[slot][0] = token g, s[slot][1] = token g+8
    float s[HS][2];
    if (G == 4) {
      s[0][0] = sc[0][0] + sc[0][1];
      s[0][1] = sc[0][2] + sc[0][3];
    } else {
      s[0][0] = sc[0][0] + sc[NT - 1][0];
      s[0][1] = sc[0][2] + sc[NT - 1][2];
      s[HS - 1][0] = sc[0][1] + sc[NT - 1][1];
      s[HS - 1][1] = sc[0][3] + sc[NT - 1][3];
    }
    float p[HS][2];
#pragma unroll
    for (int hsl = 0; hsl < HS; ++hsl) {
      const float sa = okA ? s[hsl][0] * nkA : -CUDART_INF_F;
      const float sb = okB ? s[hsl][1] * nkB : -CUDART_INF_F;
      float mx = fmaxf(sa, sb);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      const float m_new = fmaxf(m_run[hsl], mx);
      if (m_new > m_run[hsl]) {
        const float r = fast_exp2(m_run[hsl] - m_new);
        l_run[hsl] *= r;
        if (G == 4) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[j][i] *= r;
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            acc[j][hsl] *= r;
            acc[j][hsl + 2] *= r;
          }
        }
        m_run[hsl] = m_new;
      }
      const float pa = fast_exp2(sa - m_new), pb = fast_exp2(sb - m_new);
      l_run[hsl] += pa + pb;
      p[hsl][0] = okA ? pa * nvA : 0.f;
      p[hsl][1] = okB ? pb * nvB : 0.f;
    }

    // ---- P in the S layout (row = token, cols 2tq, 2tq+1) -> B operand via movmatrix
    uint32_t rowA, rowB;
    if (G == 4) {
      const float hiA = __half2float(__float2half_rn(p[0][0]));
      const float hiB = __half2float(__float2half_rn(p[0][1]));
      rowA = pack_half2(hiA, p[0][0] - hiA);
      rowB = pack_half2(hiB, p[0][1] - hiB);
    } else {
      rowA = pack_half2(p[0][0], p[HS - 1][0]);
      rowB = pack_half2(p[0][1], p[HS - 1][1]);
    }
    const uint32_t bp0 = movmatrix_trans(rowA), bp1 = movmatrix_trans(rowB);

    // ---- values: O^T[coord][col] += V^T[coord][token] P^T[token][col]
    {
      uint32_t selA[4], selB[4];
      chunk_selectors(va0, va1, va2, selA);
      chunk_selectors(vb0, vb1, vb2, selB);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t sA = (j & 1) ? (selA[j >> 1] >> 16) : selA[j >> 1];
        const uint32_t sB = (j & 1) ? (selB[j >> 1] >> 16) : selB[j >> 1];
        uint32_t lA, hA, lB, hB;
        lut4(sA, lut_lo, lut_hi, lA, hA);
        lut4(sB, lut_lo, lut_hi, lB, hB);
        const uint32_t a0 = pair02(lA, hA), a1 = pair13(lA, hA);
        const uint32_t a2 = pair02(lB, hB), a3 = pair13(lB, hB);
        mma16816(acc[j], a0, a1, a2, a3, bp0, bp1);
      }
    }
  }

  // ---- warp partials -> shared memory.  Thread (g, tq) holds coordinates 16g..16g+15:
  // acc[j][0|1] at 16g+2j, acc[j][2|3] at 16g+2j+1.
#pragma unroll
  for (int hsl = 0; hsl < HS; ++hsl) {
    float l = l_run[hsl];
    l += __shfl_xor_sync(0xffffffffu, l, 4);
    l += __shfl_xor_sync(0xffffffffu, l, 8);
    l += __shfl_xor_sync(0xffffffffu, l, 16);
    const int head = (G == 4) ? tq : 2 * tq + hsl;
    if (g == 0) {
      sm[warp][head] = m_run[hsl];
      sl[warp][head] = l;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float o0, o1;
      if (G == 4) {
        o0 = acc[j][0] + acc[j][1];
        o1 = acc[j][2] + acc[j][3];
      } else {
        o0 = acc[j][hsl];
        o1 = acc[j][hsl + 2];
      }
      so[warp][head][16 * g + 2 * j] = o0;
      so[warp][head][16 * g + 2 * j + 1] = o1;
    }
  }
  __syncthreads();

  // ---- merge warps, write this split's partial for each of the G query heads
  for (int idx = threadIdx.x; idx < G * D; idx += DEC_WARPS * 32) {
    const int h = idx / D, coord = idx % D;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < DEC_WARPS; ++w) M = fmaxf(M, sm[w][h]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < DEC_WARPS; ++w) {
      const float mw = sm[w][h];
      const float f = (mw == -CUDART_INF_F) ? 0.f : fast_exp2(mw - M);
      L = fmaf(sl[w][h], f, L);
      O = fmaf(so[w][h][coord], f, O);
    }
    if (h >= g_real) continue;
    const size_t row = ((size_t)b * n_q_heads + (size_t)kvh * g_real + h) * n_split + split;
    ws.part_o[row * D + coord] = O;
    if (coord == 0) ws.part_ml[row] = make_float2(M, L);
  }
}

// One warp per (sequence, query head): merge splits, normalise, undo the alpha and
// 1/sqrt(128) centroid scales, rotate back with R^T = H_hat S^T.
__global__ void __launch_bounds__(128)
decode_combine_kernel(int batch, int n_q_heads, int G, const int32_t* __restrict__ ctx_len, int max_ctx,
                      int chunk, int n_split, const float* __restrict__ params_layer, Workspace ws,
                      float* __restrict__ out, uint32_t* status, KernelConsts kc) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (row >= batch * n_q_heads) return;
  const int b = row / n_q_heads, hq = row % n_q_heads;
  int ctx = ctx_len[b];
  if (ctx < 0) ctx = 0;
  if (ctx > max_ctx) ctx = max_ctx;
  const int ns = (ctx + chunk - 1) / chunk;
  float4* dst = reinterpret_cast<float4*>(out + (size_t)row * D) + lane;
  if (ns == 0) {
    *dst = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  const size_t base = (size_t)row * n_split;
  float M = -CUDART_INF_F;
  for (int s = 0; s < ns; ++s) M = fmaxf(M, ws.part_ml[base + s].x);
  float L = 0.f;
  float o[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < ns; ++s) {
    const float2 ml = ws.part_ml[base + s];
    const float f = (ml.x == -CUDART_INF_F) ? 0.f : fast_exp2(ml.x - M);
    L = fmaf(ml.y, f, L);
    const float4 po = *(reinterpret_cast<const float4*>(ws.part_o + (base + s) * D) + lane);
    o[0] = fmaf(po.x, f, o[0]);
    o[1] = fmaf(po.y, f, o[1]);
    o[2] = fmaf(po.z, f, o[2]);
    o[3] = fmaf(po.w, f, o[3]);
  }
  if (!(L > 0.f)) {  // only when every tile of the context sat on an invalid page
    *dst = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  const float scale = kc.inv_alpha * 0.08838834764831845f / L;
#pragma unroll
  for (int i = 0; i < 4; ++i) o[i] *= scale;
  float Mp[4][4];
  fused_block_matrix(params_layer + ((size_t)(hq / G) * NBLK + lane) * 8, Mp);
  warp_rotate_inverse(o, Mp);
  *dst = make_float4(o[0], o[1], o[2], o[3]);
}

int launch_decode(const LayerView& v, const void* q, int q_f32, int batch, int n_q_heads, const int32_t* ctx_len,
                  int max_ctx, const float* params_layer, float* out, void* workspace, const KernelConsts& kc,
                  void* stream) {
  if (batch == 0 || n_q_heads == 0) return 0;
  const int G = n_q_heads / v.n_kv_heads;
  SplitPlan p = plan_splits(batch, v.n_kv_heads, max_ctx);
  Workspace ws = carve(workspace, batch, n_q_heads, p.n_split);
  cudaStream_t st = (cudaStream_t)stream;
  if (max_ctx > 0) {
    dim3 grid(p.n_split, v.n_kv_heads, batch);
    if (G <= 4)
      decode_split_kernel<4><<<grid, DEC_WARPS * 32, 0, st>>>(v, q, q_f32, n_q_heads, G, ctx_len, max_ctx, p.chunk,
                                                              p.n_split, params_layer, ws, kc);
    else
      decode_split_kernel<8><<<grid, DEC_WARPS * 32, 0, st>>>(v, q, q_f32, n_q_heads, G, ctx_len, max_ctx, p.chunk,
                                                              p.n_split, params_layer, ws, kc);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return (int)e;
  }
  const int rows = batch * n_q_heads;
  decode_combine_kernel<<<(rows + 3) / 4, 128, 0, st>>>(batch, n_q_heads, G, ctx_len, max_ctx, p.chunk, p.n_split,
                                                         params_layer, ws, out, v.status, kc);
  return (int)cudaGetLastError();
}

}  // namespace iq
