// Chunked-prefill attention directly on the packed cache: many query tokens per KV tile.
//
// The packed pipeline of "RotaryQuant" (rebasdaily.com, section "妙处不只是压缩，而是不再展开"),
// applied to a chunk of new prompt tokens instead of one decode token ("RotorQuant",
// sd114.wiki, section "性能基准" and "压缩与速度的博弈" section "宣称的数字" report prefill speed for
// these caches).  The chunk's own K/V have been appended to the cache first; query token i of
// sequence b sits at position start[b] + i and attends causally to positions 0 .. start[b] + i.
//
// Work: groups (sequence, kv head, block of QB = 8 query tokens), each split over `splits` CTAs
// along the KV tiles 0 .. ceil(kv_end / 32) - 1 (kv_end = the block's last position + 1).  The CTA
// streams its tiles through a ring in shared memory with bulk copies; every tile is used by all
// eight warps, warp w being query token w of the block (its rotated query in its own fragment
// buffer, its own causal limit, its own online softmax), so the packed K/V are read once per
// eight query tokens and expanded by each warp on the tensor cores exactly as in decode.  Each
// warp writes one partial (m, l, O) per head; a second kernel merges the splits, normalises and
// applies the inverse rotation.
#pragma once
#include <algorithm>

#include "iq_decode_impl.cuh"

namespace iq {

constexpr int PF_QB = 8;      // query tokens per block (one per warp)
constexpr int PF_NSLOT = 4;   // tiles in flight per CTA

struct PreArgs {
  LayerView v;
  const void* q;                 // [batch][n_tok][Hq][128]
  int q_f32, batch, n_tok, n_q_heads, g_real, n_qblk, splits, max_ctx;
  const int32_t* start;          // [batch] position of each sequence's first chunk token
  const float* params_layer;
  float2* part_ml;               // [group][split][QB][HMAX]
  float* part_o;                 // [group][split][QB][HMAX][128]
  float* out;                    // [batch][n_tok][Hq][128]
  KernelConsts kc;
};

template <int KB, int VB>
struct PreSmem {
  static constexpr int SLOT_BYTES = tile_bytes(KB, VB);
  static constexpr int ring = 0;                                        // [slot] tile records
  static constexpr int qfrag = ring + PF_NSLOT * SLOT_BYTES;            // uint32 [QB][32][QF_WORDS]
  static constexpr int kappa = qfrag + PF_QB * 32 * QF_WORDS * 4;       // float [QB][HMAX]
  static constexpr int sparams = kappa + PF_QB * HMAX * 4;              // float [256]
  static constexpr int valid = sparams + 256 * 4;                       // uint32 [slot] token masks
  static constexpr int bars = valid + PF_NSLOT * 4;                     // uint64 [slot]
  static constexpr int bytes = bars + PF_NSLOT * 8;
};

template <bool P4, int KB, int VB>
__global__ void __launch_bounds__(DEC_THREADS, 2) prefill_kernel(PreArgs a) {
  using SM = PreSmem<KB, VB>;
  constexpr int SLOT = SM::SLOT_BYTES;
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ring = smem + SM::ring;
  uint32_t* qfrag = reinterpret_cast<uint32_t*>(smem + SM::qfrag);
  float* kappa = reinterpret_cast<float*>(smem + SM::kappa);
  float* sprm = reinterpret_cast<float*>(smem + SM::sparams);
  uint32_t* valid = reinterpret_cast<uint32_t*>(smem + SM::valid);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::bars);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Hkv = a.v.n_kv_heads;

  const int group = blockIdx.x / a.splits, split = blockIdx.x % a.splits;
  const int qb = group % a.n_qblk, kvh = (group / a.n_qblk) % Hkv, b = group / (a.n_qblk * Hkv);
  const int tok0 = qb * PF_QB;
  const int n_live = min(PF_QB, a.n_tok - tok0);
  int sp = a.start[b];
  if (sp < 0 || sp > a.max_ctx - a.n_tok) {  // outside [0, max_ctx - n_tok]: clamped and flagged
    if (a.v.status && split == 0 && qb == 0 && kvh == 0 && threadIdx.x == 0) atomicOr(a.v.status, IQ_DEVERR_CTX);
    sp = sp < 0 ? 0 : a.max_ctx - a.n_tok;
  }
  const int p0 = sp + tok0;               // position of the block's first query token
  const int kv_end = p0 + n_live;         // positions 0 .. kv_end - 1 are read
  const int ntiles = (kv_end + TT - 1) / TT;
  const int t_lo = (int)((long long)split * ntiles / a.splits), t_hi = (int)((long long)(split + 1) * ntiles / a.splits);

  if (threadIdx.x == 0) {
    for (int s = 0; s < PF_NSLOT; ++s) mbar_init(&bars[s], 1);
    mbar_fence_init();
  }
  if (threadIdx.x < params_per_head(a.v.rot) / 4)
    reinterpret_cast<float4*>(sprm)[threadIdx.x] =
        reinterpret_cast<const float4*>(a.params_layer + (size_t)kvh * params_per_head(a.v.rot))[threadIdx.x];
  __syncthreads();

  // first tiles of the range in flight while the queries are rotated
  auto issue = [&](int i) {
    const int t = TT * i;
    int pg = b;
    if (a.v.block_table) {
      const int idx = t / a.v.page_size;
      pg = idx < a.v.max_pages ? a.v.block_table[(size_t)b * a.v.max_pages + idx] : -1;
    }
    const int sl = (i - t_lo) % PF_NSLOT;
    issue_tile(a.v, b, kvh, i, kv_end, 0, pg, ring + sl * SLOT, &valid[sl], &bars[sl], SLOT);
  };
  if (threadIdx.x == 0)
    for (int i = t_lo; i < min(t_hi, t_lo + PF_NSLOT); ++i) issue(i);

  // rotated queries: (token j, head h) pairs spread over the warps; P4 fills rows h and h + 4
  constexpr int HQ = P4 ? 4 : HMAX;
  for (int idx = warp; idx < PF_QB * HQ; idx += DEC_WARPS) {
    const int j = idx / HQ, h = idx % HQ;
    const bool live = j < n_live && h < a.g_real;
    const size_t row = (((size_t)b * a.n_tok + tok0 + j) * a.n_q_heads + (size_t)kvh * a.g_real + h) * D;
    rotate_query_row<P4>(a.q, a.q_f32, row, live, a.v.rot, a.kc.k.alpha8, h, sprm, qfrag + j * 32 * QF_WORDS,
                         kappa + j * HMAX);
    if (P4 && lane == 0) kappa[j * HMAX + h + 4] = 0.f;  // rows of lo terms: their lanes' scores are unused
  }
  __syncthreads();

  const int my_pos = p0 + warp;  // this warp's query position (live when warp < n_live)
  const bool live = warp < n_live;
  const float kap = kappa[warp * HMAX + (lane >> 2)];
  const uint32_t* qf = qfrag + warp * 32 * QF_WORDS + lane * QF_WORDS;
  WarpState st;
  st.m = -CUDART_INF_F;
  st.l = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) st.acc[j][e] = 0.f;

  bool ok = true;
  for (int i = t_lo; i < t_hi; ++i) {
    const int k = i - t_lo, sl = k % PF_NSLOT;
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[sl], (k / PF_NSLOT) & 1, a.v.status));
    const int tok_end = my_pos + 1 - TT * i;  // causal limit inside this tile
    if (ok && live && tok_end > 0)
      process_tile<P4, KB, VB>(ring + sl * SLOT, valid[sl] & token_range_mask(0, tok_end), qf, kap, a.kc, st);
    __syncthreads();  // every warp is done with slot sl
    if (threadIdx.x == 0 && i + PF_NSLOT < t_hi) issue(i + PF_NSLOT);
  }
  // leave no bulk copy in flight (only after a timed-out wait can one be pending)
  if (!ok && threadIdx.x == 0)
    for (int i = t_lo; i < t_hi; ++i) mbar_wait(&bars[(i - t_lo) % PF_NSLOT], ((i - t_lo) / PF_NSLOT) & 1, nullptr);

  // ---- this warp's partial: (m, l) per head and O in the rotated basis
  if (P4) {  // add the lo columns (lanes t >= 2) into the hi columns of the same heads
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) st.acc[j][e] += __shfl_xor_sync(0xffffffffu, st.acc[j][e], 2);
  }
  float lq = st.l;
  lq += __shfl_xor_sync(0xffffffffu, lq, 1);
  lq += __shfl_xor_sync(0xffffffffu, lq, 2);
  const size_t prow = ((size_t)group * a.splits + split) * PF_QB + warp;
  const int g = lane >> 2, t = lane & 3;
  if ((lane & 3) == 0) a.part_ml[prow * HMAX + g] = make_float2(live ? st.m : -CUDART_INF_F, live ? lq : 0.f);
  float* po = a.part_o + prow * HMAX * D;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    po[(2 * t) * D + 16 * j + g] = st.acc[j][0];
    po[(2 * t + 1) * D + 16 * j + g] = st.acc[j][1];
    po[(2 * t) * D + 16 * j + g + 8] = st.acc[j][2];
    po[(2 * t + 1) * D + 16 * j + g + 8] = st.acc[j][3];
  }
}

// Merge of the splits of every group: warp per (token, head); normalise; inverse rotation.
static __global__ void __launch_bounds__(DEC_THREADS) prefill_merge_kernel(PreArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float sprm[256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Hkv = a.v.n_kv_heads;
  const int group = blockIdx.x;
  const int qb = group % a.n_qblk, kvh = (group / a.n_qblk) % Hkv, b = group / (a.n_qblk * Hkv);
  const int tok0 = qb * PF_QB, n_live = min(PF_QB, a.n_tok - tok0);
  if (threadIdx.x < params_per_head(a.v.rot) / 4)
    reinterpret_cast<float4*>(sprm)[threadIdx.x] =
        reinterpret_cast<const float4*>(a.params_layer + (size_t)kvh * params_per_head(a.v.rot))[threadIdx.x];
  __syncthreads();
  float Mp[4][4];
  variant_block_matrix(a.v.rot, sprm + lane * params_per_block(a.v.rot), Mp);
  for (int idx = warp; idx < n_live * a.g_real; idx += DEC_WARPS) {
    const int j = idx / a.g_real, h = idx % a.g_real;
    float M = -CUDART_INF_F;
    for (int s = 0; s < a.splits; ++s)
      M = fmaxf(M, a.part_ml[(((size_t)group * a.splits + s) * PF_QB + j) * HMAX + h].x);
    float L = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < a.splits; ++s) {
      const size_t prow = ((size_t)group * a.splits + s) * PF_QB + j;
      const float2 ml = a.part_ml[prow * HMAX + h];
      if (ml.x == -CUDART_INF_F) continue;
      const float w = fast_exp2(ml.x - M);
      L = fmaf(ml.y, w, L);
      const float4 v = reinterpret_cast<const float4*>(a.part_o + (prow * HMAX + h) * D)[lane];
      o[0] = fmaf(v.x, w, o[0]); o[1] = fmaf(v.y, w, o[1]); o[2] = fmaf(v.z, w, o[2]); o[3] = fmaf(v.w, w, o[3]);
    }
    const float sc = L > 0.f ? 0.08838834764831845f / (a.kc.v.alpha8 * L) : 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] *= sc;
    warp_rotate_inverse(o, Mp, a.v.rot == ROT_ISO);
    reinterpret_cast<float4*>(a.out + (((size_t)b * a.n_tok + tok0 + j) * a.n_q_heads + (size_t)kvh * a.g_real + h) *
                                          D)[lane] = make_float4(o[0], o[1], o[2], o[3]);
  }
}

// Splits per group: enough CTAs for two per SM, each with at least two tiles.
inline int prefill_splits(int groups, int max_tiles, int n_sm) {
  int s = (2 * n_sm + groups - 1) / groups;
  s = std::min(s, std::max(1, max_tiles / 2));
  return std::max(1, std::min(s, 64));
}

template <int KB, int VB>
int launch_prefill_kv(const LayerView& v, const void* q, int q_f32, int batch, int n_tok, int n_q_heads,
                      const int32_t* start, int max_ctx, const float* params_layer, float* out, void* workspace,
                      const KernelConsts& kc, void* stream, int n_sm) {
  if (batch == 0 || n_tok == 0 || n_q_heads == 0) return 0;
  PreArgs a;
  a.v = v;
  a.q = q;
  a.q_f32 = q_f32;
  a.batch = batch;
  a.n_tok = n_tok;
  a.n_q_heads = n_q_heads;
  a.g_real = n_q_heads / v.n_kv_heads;
  a.n_qblk = (n_tok + PF_QB - 1) / PF_QB;
  const int groups = batch * v.n_kv_heads * a.n_qblk;
  a.splits = prefill_splits(groups, (max_ctx + TT - 1) / TT, n_sm);
  a.max_ctx = max_ctx;
  a.start = start;
  a.params_layer = params_layer;
  const size_t rows = (size_t)groups * a.splits * PF_QB * HMAX;
  a.part_ml = (float2*)workspace;
  a.part_o = (float*)((char*)workspace + ((rows * sizeof(float2) + 255) & ~(size_t)255));
  a.out = out;
  a.kc = kc;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaFuncSetAttribute(prefill_kernel<false, KB, VB>, cudaFuncAttributeMaxDynamicSharedMemorySize, PreSmem<KB, VB>::bytes);
    cudaFuncSetAttribute(prefill_kernel<true, KB, VB>, cudaFuncAttributeMaxDynamicSharedMemorySize, PreSmem<KB, VB>::bytes);
  });
  auto kern = a.g_real <= 4 ? prefill_kernel<true, KB, VB> : prefill_kernel<false, KB, VB>;
  int e = (int)launch_pdl(kern, dim3(groups * a.splits), dim3(DEC_THREADS), PreSmem<KB, VB>::bytes,
                          (cudaStream_t)stream, a);
  if (e) return e;
  return (int)launch_pdl(prefill_merge_kernel, dim3(groups), dim3(DEC_THREADS), 0, (cudaStream_t)stream, a);
}

}  // namespace iq
