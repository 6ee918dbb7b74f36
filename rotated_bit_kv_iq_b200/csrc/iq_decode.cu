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

#include <mutex>

#include "iq_device.cuh"

namespace iq {

constexpr int DEC_WARPS = 8;                    // every warp consumes; lane 0 of warp 0 also produces
constexpr int DEC_THREADS = DEC_WARPS * 32;
constexpr int STAGE_TOKENS = DEC_WARPS * TILE;  // 128 tokens: one 16-token tile per consumer warp
constexpr int TILE_K = TILE * K_REC;            // 768 B of K records per tile
constexpr int TILE_V = TILE / 2 * V_REC;        // 768 B of V records per tile
constexpr int TILE_N = TILE * 2;                // 32 B of norms per tile
constexpr int STAGE_K = 0;
constexpr int STAGE_V = STAGE_K + DEC_WARPS * TILE_K;
constexpr int STAGE_KN = STAGE_V + DEC_WARPS * TILE_V;
constexpr int STAGE_VN = STAGE_KN + DEC_WARPS * TILE_N;
constexpr int STAGE_BYTES = STAGE_VN + DEC_WARPS * TILE_N;  // 12800 B
constexpr int NSTAGE = 6;
constexpr float kLog2e = 1.4426950408889634f;

template <int G>
struct DecSmem {
  // Row strides chosen for conflict-free shared-memory access (see the uses):
  static constexpr int SQ_STRIDE = 132;                      // floats per rotated-query row
  static constexpr int SO_STRIDE = (G == 4) ? 132 : 134;     // floats per (warp, head) partial row (>= 131)
  static constexpr int sq = NSTAGE * STAGE_BYTES;            // float [G][SQ_STRIDE] rotated queries
  static constexpr int sm = sq + G * SQ_STRIDE * 4;          // float [DEC_WARPS][G] warp maxima
  static constexpr int sl = sm + DEC_WARPS * G * 4;          // float [DEC_WARPS][G] warp sums
  static constexpr int valid = sl + DEC_WARPS * G * 4;       // uint8 [NSTAGE] tile masks
  static constexpr int abort_flag = valid + 16;              // int
  static constexpr int bars = (abort_flag + 4 + 7) / 8 * 8;  // uint64 full[NSTAGE], empty[NSTAGE]
  static constexpr int bytes = bars + 2 * NSTAGE * 8;
  static_assert(DEC_WARPS * G * SO_STRIDE * 4 <= NSTAGE * STAGE_BYTES, "merge buffer reuses the stages");
  static_assert(SO_STRIDE >= D + D / 32 - 1 + 1, "skewed row fits its stride");
};

struct Workspace {
  float* part_o;   // [batch][Hq][n_split][128]
  float2* part_ml; // [batch][Hq][n_split] (max in log2 units, sum of exp2)
};

static inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

SplitPlan plan_splits(int batch, int n_kv_heads, int max_ctx) {
  SplitPlan p;
  const int groups = batch * n_kv_heads;
  const int target_ctas = 2 * 148;  // two resident CTAs per SM
  int want = (target_ctas + groups - 1) / groups;
  if (want < 1) want = 1;
  int chunk = (max_ctx + want - 1) / want;
  chunk = (chunk + STAGE_TOKENS - 1) / STAGE_TOKENS * STAGE_TOKENS;
  if (chunk < STAGE_TOKENS) chunk = STAGE_TOKENS;
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

// Producer side: stream stage i (up to 8 tiles of 16 tokens) of this CTA's range into ring
// slot s with bulk copies; runs of tiles on the same page with consecutive slots share one
// copy per component.  Tiles past the context or on invalid pages are left out of the mask.
__device__ __forceinline__ void issue_stage(const LayerView& v, int b, int kvh, int t_stage, int t_end,
                                            uint8_t* stage, uint8_t* valid_mask, uint64_t* full_bar) {
  int pages[DEC_WARPS], slots[DEC_WARPS];
  uint32_t bytes = 0, mask = 0;
#pragma unroll
  for (int j = 0; j < DEC_WARPS; ++j) {
    const int t = t_stage + TILE * j;
    pages[j] = -1;
    slots[j] = 0;
    if (t < t_end) {
      pages[j] = resolve_page(v, b, t);
      slots[j] = t % v.page_size;
      if (pages[j] >= 0) {
        mask |= 1u << j;
        bytes += TILE_K + TILE_V + 2 * TILE_N;
      }
    }
  }
  *valid_mask = (uint8_t)mask;
  mbar_arrive_expect_tx(full_bar, bytes);
  int j = 0;
  while (j < DEC_WARPS) {
    if (pages[j] < 0) { ++j; continue; }
    int k = j + 1;
    while (k < DEC_WARPS && pages[k] == pages[j] && slots[k] == slots[j] + TILE * (k - j)) ++k;
    const int n = k - j;
    const size_t hs = (size_t)pages[j] * v.n_kv_heads + kvh;
    bulk_g2s(stage + STAGE_K + j * TILE_K, v.k_codes + (hs * v.page_size + slots[j]) * K_REC, n * TILE_K, full_bar);
    bulk_g2s(stage + STAGE_V + j * TILE_V, v.v_codes + (hs * (v.page_size / 2) + slots[j] / 2) * V_REC, n * TILE_V,
             full_bar);
    bulk_g2s(stage + STAGE_KN + j * TILE_N, v.k_norms + hs * v.page_size + slots[j], n * TILE_N, full_bar);
    bulk_g2s(stage + STAGE_VN + j * TILE_N, v.v_norms + hs * v.page_size + slots[j], n * TILE_N, full_bar);
    j = k;
  }
}

// G: kernel layout width (4 or 8 query heads per kv head); g_real <= G query heads exist
// (group sizes 1 and 2 run on the 4-wide layout with the unused columns zero).
// FUSED: decode step -- the new token of each sequence (position ctx-1; fp16 K/V in
// k_new/v_new, [batch][Hkv][128]) is encoded into the cache by the CTA whose range holds it
// before that tile is loaded.  The cache stages not holding it are requested before waiting
// for the previous kernel in the stream (their contents do not depend on it), so layer l+1's
// loads overlap layer l's tail.
template <int G, bool FUSED>
__global__ void __launch_bounds__(DEC_THREADS, 2)
decode_split_kernel(LayerView v, const void* __restrict__ q, int q_f32, int n_q_heads, int g_real,
                    const int32_t* __restrict__ ctx_len, int max_ctx, int chunk, int n_split,
                    const float* __restrict__ params_layer, Workspace ws, KernelConsts kc,
                    const __half* __restrict__ k_new, const __half* __restrict__ v_new) {
  pdl_launch_dependents();
  if (!FUSED) pdl_wait();  // a plain call may read anything the previous kernel wrote
  using L = DecSmem<G>;
  extern __shared__ __align__(128) uint8_t smem[];
  float(*sq)[L::SQ_STRIDE] = reinterpret_cast<float(*)[L::SQ_STRIDE]>(smem + L::sq);
  float(*sm)[G] = reinterpret_cast<float(*)[G]>(smem + L::sm);
  float(*sl)[G] = reinterpret_cast<float(*)[G]>(smem + L::sl);
  uint8_t* valid = smem + L::valid;
  int* abort_flag = reinterpret_cast<int*>(smem + L::abort_flag);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::bars);
  uint64_t* empty = full + NSTAGE;

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;
  const int ctx = clamp_ctx(ctx_len[b], max_ctx, v.status);
  const int t_begin = split * chunk;
  if (t_begin >= ctx) return;  // uniform over the CTA
  const int t_end = min(t_begin + chunk, ctx);
  const int n_stage = (t_end - t_begin + STAGE_TOKENS - 1) / STAGE_TOKENS;
  const int p_new = ctx - 1;  // FUSED: position of the token appended by this call
  const bool owner = FUSED && p_new >= t_begin && p_new < t_end;
  const int s_new = owner ? (p_new - t_begin) / STAGE_TOKENS : -1;  // stage holding it

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], DEC_WARPS);
    }
    *abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  const bool producer = (threadIdx.x == 0);
  if (producer) {
    // Fill the ring: stages 0 .. NSTAGE-1 go out before any compute (the one holding a token
    // appended by this call only once that token is written).
    for (int i = 0; i < n_stage && i < NSTAGE; ++i)
      if (i != s_new)
        issue_stage(v, b, kvh, t_begin + i * STAGE_TOKENS, t_end, smem + i * STAGE_BYTES, &valid[i], &full[i]);
  }
  if (FUSED) pdl_wait();

  // Rotate the G queries of this kv head (one warp per query) while the first stages land,
  // scaled so that score_log2 = n_k * <q', alpha*c[codes]>: q' = R q log2(e) / (128 alpha).
  {
    float Mp[4][4];
    fused_block_matrix(params_layer + ((size_t)kvh * NBLK + lane) * 8, Mp);
    if (owner && warp < 2) {
      // FUSED: warp 0 appends the new K vector, warp 1 the new V vector, of this kv head.
      const int page = resolve_page(v, b, p_new);
      if (page >= 0)
        warp_encode_vector(v, (warp == 0 ? k_new : v_new) + ((size_t)b * v.n_kv_heads + kvh) * D, kvh, warp, page,
                           p_new % v.page_size, Mp, kc);
    }
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
      const float sc = kLog2e * kc.inv_alpha * (1.0f / 128.0f);
      *reinterpret_cast<float4*>(&sq[h][4 * lane]) = make_float4(x[0] * sc, x[1] * sc, x[2] * sc, x[3] * sc);
    }
  }
  __syncthreads();
  if (owner && producer) {
    // The appended token's record is in global memory (visible CTA-wide after the barrier);
    // order it before the bulk-copy reads of its stage (now or in a later refill).
    fence_proxy_async_global();
    if (s_new < NSTAGE)
      issue_stage(v, b, kvh, t_begin + s_new * STAGE_TOKENS, t_end, smem + s_new * STAGE_BYTES, &valid[s_new],
                  &full[s_new]);
  }

  {
    // Query B-fragments (k16 x n8 per k-chunk c): MMA k index 2tq+e <-> coordinate
    // 32tq+4c+e, k index 2tq+8+e <-> 32tq+4c+2+e.  Columns: G=4 -> (head n/2, hi|lo = n%2);
    // G=8 -> tile 0 = hi halves of heads 0..7, tile 1 = lo halves.
    constexpr int NT = G / 4;
    uint32_t qb[NT][8][2];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int head = (G == 4) ? (g >> 1) : g;
        const bool lo_part = (G == 4) ? (g & 1) : (nt == 1);
        // float4 reads: with a 132-float row the 8 lanes of each wavefront hit distinct banks
        const float4 x4 = *reinterpret_cast<const float4*>(&sq[head][32 * tq + 4 * c]);
        const float xs[4] = {x4.x, x4.y, x4.z, x4.w};
        float vals[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float hi = __half2float(__float2half_rn(xs[e]));
          vals[e] = lo_part ? (xs[e] - hi) : xs[e];
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

    for (int i = 0; i < n_stage; ++i) {
      // Refill: the slot of stage i-2 takes stage i-2+NSTAGE once every warp has left it.
      if (producer && i >= 2 && i - 2 + NSTAGE < n_stage) {
        const int j = i - 2, sj = j % NSTAGE;
        if (mbar_wait(&empty[sj], (j / NSTAGE) & 1, v.status))
          issue_stage(v, b, kvh, t_begin + (j + NSTAGE) * STAGE_TOKENS, t_end, smem + sj * STAGE_BYTES, &valid[sj],
                      &full[sj]);
        else
          *abort_flag = 1;
      }
      const int s = i % NSTAGE;
      // every lane polls; the verdict is made warp-uniform before any warp-wide instruction
      const bool landed = __all_sync(0xffffffffu, mbar_wait(&full[s], (i / NSTAGE) & 1, v.status));
      if (!landed) {
        if (lane == 0) *abort_flag = 1;
        break;
      }
      const int t0 = t_begin + i * STAGE_TOKENS + TILE * warp;
      if (t0 < t_end && ((valid[s] >> warp) & 1)) {
        const uint8_t* st = smem + s * STAGE_BYTES;
        const uint32_t* kA = reinterpret_cast<const uint32_t*>(st + STAGE_K + warp * TILE_K + g * K_REC + tq * 12);
        const uint32_t* kB = kA + 8 * K_REC / 4;
        const uint32_t* vA = reinterpret_cast<const uint32_t*>(st + STAGE_V + warp * TILE_V + tq * V_REC + g * 12);
        const uint32_t* vB = vA + 4 * V_REC / 4;
        const uint16_t* knp = reinterpret_cast<const uint16_t*>(st + STAGE_KN + warp * TILE_N);
        const uint16_t* vnp = reinterpret_cast<const uint16_t*>(st + STAGE_VN + warp * TILE_N);
        const bool okA = t0 + g < t_end, okB = t0 + g + 8 < t_end;
        const float nkA = half_bits_to_float(knp[g]), nkB = half_bits_to_float(knp[g + 8]);
        const float nvA = half_bits_to_float(vnp[g]), nvB = half_bits_to_float(vnp[g + 8]);

        // ---- scores: S[token][col] over 8 k-chunks
        // two independent accumulation chains (even / odd k-chunks) halve the mma latency chain
        float sc[NT][4], sc2[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[nt][e] = sc2[nt][e] = 0.f;
        {
          uint32_t selA[4], selB[4];
          chunk_selectors(kA[0], kA[1], kA[2], selA);
          chunk_selectors(kB[0], kB[1], kB[2], selB);
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
            for (int nt = 0; nt < NT; ++nt)
              mma16816((c & 1) ? sc2[nt] : sc[nt], a0, a1, a2, a3, qb[nt][c][0], qb[nt][c][1]);
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[nt][e] += sc2[nt][e];
        }

        // ---- online softmax per head slot; sv[slot][0] = token g, sv[slot][1] = token g+8
        float sv[HS][2];
        if (G == 4) {
          sv[0][0] = sc[0][0] + sc[0][1];
          sv[0][1] = sc[0][2] + sc[0][3];
        } else {
          sv[0][0] = sc[0][0] + sc[NT - 1][0];
          sv[0][1] = sc[0][2] + sc[NT - 1][2];
          sv[HS - 1][0] = sc[0][1] + sc[NT - 1][1];
          sv[HS - 1][1] = sc[0][3] + sc[NT - 1][3];
        }
        float p[HS][2];
#pragma unroll
        for (int hsl = 0; hsl < HS; ++hsl) {
          const float sa = okA ? sv[hsl][0] * nkA : -CUDART_INF_F;
          const float sb = okB ? sv[hsl][1] * nkB : -CUDART_INF_F;
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
                for (int e = 0; e < 4; ++e) acc[j][e] *= r;
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
          chunk_selectors(vA[0], vA[1], vA[2], selA);
          chunk_selectors(vB[0], vB[1], vB[2], selB);
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
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }

    // ---- warp partials.  Thread (g, tq) holds coordinates 16g..16g+15: acc[j][0|1] at
    // 16g+2j, acc[j][2|3] at 16g+2j+1.  Every consumer warp has left the ring before any
    // of them overwrites it with the merge buffer.
    __syncthreads();
    // Partial row of (warp, head): coordinate c at c + c/32 (a one-word skew per 32), rows
    // SO_STRIDE floats apart; with these the strided stores below and the merge reads are
    // free of bank conflicts.
    float(*so)[G][L::SO_STRIDE] = reinterpret_cast<float(*)[G][L::SO_STRIDE]>(smem);
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
        const int c0 = 16 * g + 2 * j;
        so[warp][head][c0 + (c0 >> 5)] = o0;
        so[warp][head][c0 + 1 + (c0 >> 5)] = o1;
      }
    }
  }
  __syncthreads();
  if (*abort_flag) return;

  // ---- merge warps, write this split's partial for each of the G query heads
  const float(*so)[G][L::SO_STRIDE] = reinterpret_cast<const float(*)[G][L::SO_STRIDE]>(smem);
  for (int idx = threadIdx.x; idx < G * D; idx += DEC_THREADS) {
    const int h = idx / D, coord = idx % D;
    if (h >= g_real) continue;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < DEC_WARPS; ++w) M = fmaxf(M, sm[w][h]);
    float Lsum = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < DEC_WARPS; ++w) {
      const float mw = sm[w][h];
      const float f = (mw == -CUDART_INF_F) ? 0.f : fast_exp2(mw - M);
      Lsum = fmaf(sl[w][h], f, Lsum);
      O = fmaf(so[w][h][coord + (coord >> 5)], f, O);
    }
    const size_t row = ((size_t)b * n_q_heads + (size_t)kvh * g_real + h) * n_split + split;
    ws.part_o[row * D + coord] = O;
    if (coord == 0) ws.part_ml[row] = make_float2(M, Lsum);
  }
}

// One CTA (8 warps) per (sequence, query head).  Phase 1: the global max M and sum L over
// the splits (one split per thread, block reductions).  Phase 2: warp w sums splits w, w+8, ...
// weighted by exp2(m_s - M) with independent loads; the 8 warp sums meet in shared memory and
// warp 0 normalises, undoes the alpha and 1/sqrt(128) centroid scales and rotates back with
// R^T = H_hat S^T.
constexpr int CMB_WARPS = 8;
__global__ void __launch_bounds__(CMB_WARPS * 32)
decode_combine_kernel(int batch, int n_q_heads, int G, const int32_t* __restrict__ ctx_len, int max_ctx,
                      int chunk, int n_split, const float* __restrict__ params_layer, Workspace ws,
                      float* __restrict__ out, uint32_t* status, KernelConsts kc) {
  __shared__ float4 so[CMB_WARPS][32];
  __shared__ float red[CMB_WARPS];
  __shared__ float sM, sL;
  pdl_launch_dependents();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x;
  const int b = row / n_q_heads, hq = row % n_q_heads;
  int ctx = ctx_len[b];
  if (ctx < 0) ctx = 0;
  if (ctx > max_ctx) ctx = max_ctx;
  const int ns = (ctx + chunk - 1) / chunk;
  const size_t base = (size_t)row * n_split;

  float m = -CUDART_INF_F;
  for (int s = threadIdx.x; s < ns; s += CMB_WARPS * 32) m = fmaxf(m, ws.part_ml[base + s].x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float M = -CUDART_INF_F;
    for (int w = 0; w < CMB_WARPS; ++w) M = fmaxf(M, red[w]);
    sM = M;
  }
  __syncthreads();
  const float M = sM;
  float l = 0.f;
  for (int s = threadIdx.x; s < ns; s += CMB_WARPS * 32) {
    const float2 ml = ws.part_ml[base + s];
    if (ml.x != -CUDART_INF_F) l = fmaf(ml.y, fast_exp2(ml.x - M), l);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  __syncthreads();
  if (lane == 0) red[warp] = l;

  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int s = warp; s < ns; s += CMB_WARPS) {
    const float2 ml = ws.part_ml[base + s];
    const float4 po = *(reinterpret_cast<const float4*>(ws.part_o + (base + s) * D) + lane);
    const float f = (ml.x == -CUDART_INF_F) ? 0.f : fast_exp2(ml.x - M);
    acc.x = fmaf(po.x, f, acc.x); acc.y = fmaf(po.y, f, acc.y); acc.z = fmaf(po.z, f, acc.z); acc.w = fmaf(po.w, f, acc.w);
  }
  so[warp][lane] = acc;
  __syncthreads();
  if (warp != 0) return;
  float L = 0.f, r[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int w = 0; w < CMB_WARPS; ++w) {
    L += red[w];
    const float4 x = so[w][lane];
    r[0] += x.x; r[1] += x.y; r[2] += x.z; r[3] += x.w;
  }
  float4* dst = reinterpret_cast<float4*>(out + (size_t)row * D) + lane;
  if (!(L > 0.f)) {  // empty context, or every tile on an invalid page
    *dst = make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  const float scale = kc.inv_alpha * 0.08838834764831845f / L;
#pragma unroll
  for (int i = 0; i < 4; ++i) r[i] *= scale;
  float Mp[4][4];
  fused_block_matrix(params_layer + ((size_t)(hq / G) * NBLK + lane) * 8, Mp);
  warp_rotate_inverse(r, Mp);
  *dst = make_float4(r[0], r[1], r[2], r[3]);
}

template <bool FUSED>
static int launch_decode_impl(const LayerView& v, const void* q, int q_f32, int batch, int n_q_heads,
                              const int32_t* ctx_len, int max_ctx, const float* params_layer, float* out,
                              void* workspace, const KernelConsts& kc, void* stream, const __half* k_new,
                              const __half* v_new) {
  if (batch == 0 || n_q_heads == 0) return 0;
  const int G = n_q_heads / v.n_kv_heads;
  SplitPlan p = plan_splits(batch, v.n_kv_heads, max_ctx);
  Workspace ws = carve(workspace, batch, n_q_heads, p.n_split);
  cudaStream_t st = (cudaStream_t)stream;
  static std::once_flag attr_once;
  std::call_once(attr_once, [] {
    cudaFuncSetAttribute(decode_split_kernel<4, FUSED>, cudaFuncAttributeMaxDynamicSharedMemorySize, DecSmem<4>::bytes);
    cudaFuncSetAttribute(decode_split_kernel<8, FUSED>, cudaFuncAttributeMaxDynamicSharedMemorySize, DecSmem<8>::bytes);
    cudaFuncSetAttribute(decode_split_kernel<4, FUSED>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    cudaFuncSetAttribute(decode_split_kernel<8, FUSED>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  });
  if (max_ctx > 0) {
    const dim3 grid(p.n_split, v.n_kv_heads, batch);
    cudaError_t e;
    if (G <= 4)
      e = launch_pdl(decode_split_kernel<4, FUSED>, grid, dim3(DEC_THREADS), DecSmem<4>::bytes, st, v, q, q_f32,
                     n_q_heads, G, ctx_len, max_ctx, p.chunk, p.n_split, params_layer, ws, kc, k_new, v_new);
    else
      e = launch_pdl(decode_split_kernel<8, FUSED>, grid, dim3(DEC_THREADS), DecSmem<8>::bytes, st, v, q, q_f32,
                     n_q_heads, G, ctx_len, max_ctx, p.chunk, p.n_split, params_layer, ws, kc, k_new, v_new);
    if (e != cudaSuccess) return (int)e;
  }
  const int rows = batch * n_q_heads;
  return (int)launch_pdl(decode_combine_kernel, dim3(rows), dim3(CMB_WARPS * 32), 0, st, batch, n_q_heads, G, ctx_len,
                         max_ctx, p.chunk, p.n_split, params_layer, ws, out, v.status, kc);
}

int launch_decode(const LayerView& v, const void* q, int q_f32, int batch, int n_q_heads, const int32_t* ctx_len,
                  int max_ctx, const float* params_layer, float* out, void* workspace, const KernelConsts& kc,
                  void* stream) {
  return launch_decode_impl<false>(v, q, q_f32, batch, n_q_heads, ctx_len, max_ctx, params_layer, out, workspace, kc,
                                   stream, nullptr, nullptr);
}

int launch_decode_step(const LayerView& v, const void* q, int q_f32, const void* k_new, const void* v_new, int batch,
                       int n_q_heads, const int32_t* ctx_len, int max_ctx, const float* params_layer, float* out,
                       void* workspace, const KernelConsts& kc, void* stream) {
  return launch_decode_impl<true>(v, q, q_f32, batch, n_q_heads, ctx_len, max_ctx, params_layer, out, workspace, kc,
                                  stream, (const __half*)k_new, (const __half*)v_new);
}

}  // namespace iq
