// Chunked-prefill attention directly on the packed cache, on the 5th-generation tensor cores.
//
// The packed pipeline of "RotaryQuant" (rebasdaily.com, section "妙处不只是压缩，而是不再展开"),
// applied to a chunk of new prompt tokens instead of one decode token ("RotorQuant",
// sd114.wiki, section "性能基准" and "压缩与速度的博弈" section "宣称的数字" report prefill speed for
// these caches).  The chunk's own K/V have been appended to the cache first; query token i of
// sequence b sits at position start[b] + i and attends causally to positions 0 .. start[b] + i.
//
// Many query tokens share every key, so the contractions are dense: one CTA takes 128 query
// rows (TQ = 128 / G tokens x the G query heads of one kv head) and streams the keys in steps
// of 64 (two tile records), with the math on tcgen05 MMAs (M = 128) and fp32 accumulators in
// tensor memory:
//   * the rotated queries, scaled per row by a power of two to |q| <= 1, are split into binary16
//     hi + lo terms once; the step's K codes become binary16 centroid terms c_hi + c_lo in
//     shared memory (byte-permute table lookups), and S = Q K^T is the sum of the three
//     products hi.hi, lo.hi and hi.lo (K = 128 coordinates);
//   * the online softmax runs one thread per row on S read back from tensor memory; the
//     probabilities times the V norms, P' = 2^(s - m) n_v, are written to shared memory as
//     binary16 hi + lo terms;
//   * the V codes become the centroid terms of V^T (coordinates as rows), and O^T = V^T P'^T
//     (M = 128 coordinates, N = 128 rows, K = 64 keys; products V_hi P_hi, V_lo P_hi and
//     V_hi P_lo) lands in tensor memory; one thread per coordinate folds each step's tile into
//     its registers with the rows' rescale factors.  (The output sums terms of both signs, so a
//     single binary16 term of P' would cost far more relative accuracy than its 2^-11.)
// Roles (warp-specialised, double-buffered, synchronised by mbarriers): warps 8-11 expand the
// codes of step i + 1 while warps 0-7 take the softmax of step i (two warps per row quarter of
// tensor memory: one per half of the keys, and per half of the rows when folding the output)
// and the tensor cores compute S of step i + 1 and O of step i; one thread of warp 12 issues
// the score MMAs as soon as a step's K is expanded, one of warp 14 the output MMAs as soon as
// its P' is written, and one of warp 13 stages the tile records with bulk copies.  Splits of the key
// range leave (m, l, O) partials that a second kernel merges, normalises and rotates back (R^T).
#pragma once
#include <algorithm>

#include "iq_decode_impl.cuh"
#include "iq_tcgen05.cuh"

namespace iq {

constexpr int PF_ROWS = 128;     // query rows (token, head) per CTA: the MMA's M
constexpr int PF_BN = 64;        // keys per step (two tile records)
constexpr int PF_THREADS = 480;  // warps 0-7 softmax and output, 8-11 code expansion, 12 and 14 MMA issue, 13 loads
constexpr int PF_TMEM_COLS = 512;
constexpr int PF_S_COL = 0;      // scores of buffer b: columns [64 b, 64 b + 64)
constexpr int PF_O_COL = 128;    // output tile of buffer b: columns [128 + 128 b, 256 + 128 b)

// query tokens per CTA for G heads per kv head
IQ_HD constexpr int pf_tokens(int g) { return PF_ROWS / g; }

struct PreArgs {
  LayerView v;
  const void* q;                 // [batch][n_tok][Hq][128]
  int q_f32, batch, n_tok, n_q_heads, g_real, n_qblk, splits, max_ctx;
  const int32_t* start;          // [batch] position of each sequence's first chunk token
  const float* params_layer;
  float2* part_ml;               // [group][split][row]: (max in log2 units, sum of 2^(s - max))
  float* part_o;                 // [group][split][row][128]: sum of 2^(s - max) n_v c (rotated basis)
  float* out;                    // [batch][n_tok][Hq][128]
  KernelConsts kc;
};

// Shared memory (bytes, from a 1024-byte aligned base).  Operand tiles use the 128-byte swizzled
// K-major layout of iq_tcgen05.cuh.
template <int KB, int VB>
struct PfSmem {
  static constexpr int TB = tile_bytes(KB, VB);
  static constexpr int q_hi = 0, q_lo = 32768;  // 128 rows x 128 coordinates
  static constexpr int k0 = 65536;              // hi, lo: 64 keys x 128 coordinates
  static constexpr int vt0 = 98304;             // [buf] hi, lo: 128 coordinates x 64 keys (32 KB per buf)
  static constexpr int p = 163840;              // hi, lo: 128 rows x 64 keys (before the steps: parameters, row scales)
  static constexpr int rec = 196608;            // [buf][2] tile records
  static constexpr int nk = rec + 4 * TB;       // float [buf][64] K norms of the step's keys
  static constexpr int nv = nk + 2 * 64 * 4;    // float [buf][64] V norms
  static constexpr int mrec = nv + 2 * 64 * 4;  // uint32 [buf][2] token masks of the staged records
  static constexpr int mkv = mrec + 16;         // uint32 [buf][2] token masks of the expanded step
  static constexpr int alpha = mkv + 16;        // float [128] rows' rescale factors of the last step
  static constexpr int red = alpha + 128 * 4;   // float [2][128] per key half: row maxima, at the end sums
  static constexpr int bars = red + 256 * 4;    // uint64 [PB_COUNT]
  static constexpr int misc = bars + 24 * 8;    // uint32 tensor-memory base, int abort flag
  static constexpr int bytes = misc + 16 + 1024;  // + the alignment of the base
  static_assert(bytes <= 232448, "one CTA's shared memory on sm_100");
};

// mbarriers, by step parity [buf] where marked: records staged [buf]; K, K norms and masks
// expanded [buf]; V^T and V norms expanded [buf]; V^T free again [buf]; scores ready [buf];
// scores read [buf]; output tile ready [buf]; output tile read [buf]; P' written; K read
// (single buffer); the score MMAs done; the output MMAs done; records read [buf].
enum { PB_REC = 0, PB_KFULL = 2, PB_VFULL = 4, PB_VFREE = 6, PB_SFULL = 8, PB_SFREE = 10, PB_OFULL = 12,
       PB_OFREE = 14, PB_PFULL = 16, PB_KFREE = 17, PB_DRAIN_S = 18, PB_DRAIN_O = 19, PB_RECFREE = 20,
       PB_COUNT = 22 };
static_assert(PB_COUNT <= 24, "mbarrier slots of PfSmem");

// Bounded wait on an mbarrier phase that also gives up once another thread has given up (the
// abort flag); a timeout flags IQ_DEVERR_TIMEOUT.
__device__ __forceinline__ bool pf_wait(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort) return false;
    if (global_timer_ns() - t0 > 1000000000ull) {
      if (status) atomicOr(status, IQ_DEVERR_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
  return true;
}

// AND of `ok` over the `count` threads of named barrier `id` (a barrier for them as well).
__device__ __forceinline__ bool wg_all(bool ok, int id, int count) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred pi, po;\n setp.ne.u32 pi, %1, 0;\n bar.red.and.pred po, %2, %3, pi;\n selp.u32 %0, 1, 0, po;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)ok), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// Four codes (nibbles 0..3 of s) -> their binary16 centroid terms from the byte tables lb / hb.
template <int BITS>
__device__ __forceinline__ uint2 lut_f16x4(const uint32_t* lb, const uint32_t* hb, uint32_t s) {
  const uint32_t l = lut4<BITS>(lb, s), h = lut4<BITS>(hb, s);
  return make_uint2(prmt(l, h, 0x5140u), prmt(l, h, 0x7362u));
}

// Stage the two tile records of step `step` (positions 64 step .. 64 step + 63 of group (b, kvh))
// into dst with bulk copies completing on `bar` (two arrivals); their token masks go to `mask`.
__device__ __forceinline__ void pf_stage(const PreArgs& a, int b, int kvh, int step, int kv_end, uint8_t* dst,
                                         uint32_t* mask, uint64_t* bar, uint32_t tbytes) {
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int i = 2 * step + t, pos = TT * i;
    int pg = b;
    if (a.v.block_table && pos < kv_end) {
      const int idx = pos / a.v.page_size;
      pg = idx < a.v.max_pages ? a.v.block_table[(size_t)b * a.v.max_pages + idx] : -1;
    }
    issue_tile(a.v, b, kvh, i, kv_end, 0, pg, dst + t * tbytes, &mask[t], bar, tbytes);
  }
}

template <int KB, int VB>
__global__ void __launch_bounds__(PF_THREADS, 1) prefill_kernel(PreArgs a) {
  using SM = PfSmem<KB, VB>;
  constexpr int TB = SM::TB;
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* const smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::misc);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + SM::misc + 4);
  float* s_nk = reinterpret_cast<float*>(smem + SM::nk);
  float* s_nv = reinterpret_cast<float*>(smem + SM::nv);
  uint32_t* s_mrec = reinterpret_cast<uint32_t*>(smem + SM::mrec);
  uint32_t* s_mkv = reinterpret_cast<uint32_t*>(smem + SM::mkv);
  float* s_alpha = reinterpret_cast<float*>(smem + SM::alpha);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hkv = a.v.n_kv_heads, G = a.g_real, TQ = pf_tokens(G);

  const int group = blockIdx.x / a.splits, split = blockIdx.x % a.splits;
  const int qb = group % a.n_qblk, kvh = (group / a.n_qblk) % Hkv, b = group / (a.n_qblk * Hkv);
  const int tok0 = qb * TQ;
  const int n_live = min(TQ, a.n_tok - tok0);
  int sp = a.start[b];
  if (sp < 0 || sp > a.max_ctx - a.n_tok) {  // outside [0, max_ctx - n_tok]: clamped and flagged
    if (a.v.status && split == 0 && qb == 0 && kvh == 0 && tid == 0) atomicOr(a.v.status, IQ_DEVERR_CTX);
    sp = sp < 0 ? 0 : a.max_ctx - a.n_tok;
  }
  const int p0 = sp + tok0;        // position of the CTA's first query token
  const int kv_end = p0 + n_live;  // positions 0 .. kv_end - 1 are read
  const int steps = (kv_end + PF_BN - 1) / PF_BN;
  const int s_lo = (int)((long long)split * steps / a.splits), s_hi = (int)((long long)(split + 1) * steps / a.splits);
  const int n = s_hi - s_lo;
  const size_t prow0 = ((size_t)group * a.splits + split) * PF_ROWS;
  if (n <= 0) {  // an empty split: neutral partials (the merge skips them)
    if (tid < PF_ROWS) a.part_ml[prow0 + tid] = make_float2(-CUDART_INF_F, 0.f);
    return;
  }

  if (tid == 0) {
    for (int i = 0; i < PB_COUNT; ++i) {
      const bool by_expansion = (i >= PB_KFULL && i < PB_VFULL + 2) || (i >= PB_RECFREE && i < PB_RECFREE + 2);
      const bool by_softmax = (i >= PB_SFREE && i < PB_SFREE + 2) || (i >= PB_OFREE && i < PB_OFREE + 2) || i == PB_PFULL;
      mbar_init(&bars[i], i < PB_REC + 2 ? 2 : by_softmax ? 256 : by_expansion ? 128 : 1);
    }
    mbar_fence_init();
    *abort = 0;
  }
  if (warp == 0) tmem_alloc(tmem_slot, PF_TMEM_COLS);
  float* sprm = reinterpret_cast<float*>(smem + SM::p);  // this kv head's rotation parameters
  float* sqs = sprm + 256;                               // rows' score scales
  if (tid < params_per_head(a.v.rot) / 4)
    reinterpret_cast<float4*>(sprm)[tid] =
        reinterpret_cast<const float4*>(a.params_layer + (size_t)kvh * params_per_head(a.v.rot))[tid];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (tid == 416)  // the first two steps' records, in flight while the queries are rotated
    for (int i = 0; i < 2 && i < n; ++i)
      pf_stage(a, b, kvh, s_lo + i, kv_end, smem + SM::rec + i * 2 * TB, s_mrec + 2 * i, &bars[PB_REC + i], TB);

  // ---- queries: row r = (token r / G, head r % G), rotated, scaled by the power of two that
  // brings max |q'| into [1/2, 1), split into binary16 hi + lo (K-major rows of 128)
  for (int r = warp; r < PF_ROWS; r += PF_THREADS / 32) {
    const int tok = r / G, h = r % G;
    const bool live = r < TQ * G && tok < n_live;
    float x[4] = {0.f, 0.f, 0.f, 0.f};
    if (live) {
      const size_t row = (((size_t)b * a.n_tok + tok0 + tok) * a.n_q_heads + (size_t)kvh * G + h) * D + 4 * lane;
      if (a.q_f32) {
        const float4 f = __ldg(reinterpret_cast<const float4*>((const float*)a.q + row));
        x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
      } else {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>((const __half*)a.q + row));
        const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
        const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
        x[0] = f0.x; x[1] = f0.y; x[2] = f1.x; x[3] = f1.y;
      }
      float Mp[4][4];
      variant_block_matrix(a.v.rot, sprm + lane * params_per_block(a.v.rot), Mp);
      warp_rotate_forward(x, Mp, a.v.rot == ROT_ISO);
    }
    float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    int ex = 0;
    if (amax > 0.f) frexpf(amax, &ex);
    const float sig = ldexpf(1.f, -ex);  // exact: a power of two
    uint32_t hw[2], lw[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float y0 = x[2 * i] * sig, y1 = x[2 * i + 1] * sig;
      const __half2 hi = __floats2half2_rn(y0, y1);
      const float2 hf = __half22float2(hi);
      const __half2 lo = __floats2half2_rn(y0 - hf.x, y1 - hf.y);
      hw[i] = *reinterpret_cast<const uint32_t*>(&hi);
      lw[i] = *reinterpret_cast<const uint32_t*>(&lo);
    }
    const int off = umma_sw128_off(r, 4 * (lane & ~1), PF_ROWS) + (lane & 1) * 8;  // coordinates 4 lane ..
    *reinterpret_cast<uint2*>(smem + SM::q_hi + off) = make_uint2(hw[0], hw[1]);
    *reinterpret_cast<uint2*>(smem + SM::q_lo + off) = make_uint2(lw[0], lw[1]);
    // log2-domain score of a key = S n_k log2(e) / (128 sigma): q' c / sqrt(128) is the rotated
    // dot product with the unit key, n_k / sqrt(128) the key's norm and softmax scale
    if (lane == 0) sqs[r] = live ? kLog2e / (128.f * sig) : 0.f;
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the query tiles before the MMAs read them
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp < 8) {
    // ==== softmax and output.  Warp w reads tensor-memory lanes 32 (w % 4) ..: thread = score
    // row r of those lanes for keys 32 kh .. 32 kh + 31 (kh = w / 4), and output coordinate r for
    // rows 64 kh .. 64 kh + 63.
    const int kh = warp >> 2;
    const int r = 32 * (warp & 3) + lane;
    float* s_red = reinterpret_cast<float*>(smem + SM::red);
    const int tok = r / G;
    const bool live = r < TQ * G && tok < n_live;
    const int qpos = p0 + tok;
    const float qs = sqs[r];
    const uint32_t tlane = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    float O[PF_ROWS / 2];  // coordinate r of rows 64 kh ..
#pragma unroll
    for (int j = 0; j < PF_ROWS / 2; ++j) O[j] = 0.f;
    float m = -CUDART_INF_F, l = 0.f;  // l: this key half's share of the row's sum
    bool ok = true;
    auto fold_output = [&](int i) {  // O += the output tile of step i (rows rescaled first)
      const uint32_t tcol = tlane + PF_O_COL + 128 * (i & 1) + 64 * kh;
#pragma unroll
      for (int c = 0; c < PF_ROWS / 64; ++c) {
        uint32_t v[16], u[16];
        tmem_ld16(tcol + 32 * c, v);
        tmem_ld16(tcol + 32 * c + 16, u);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          O[32 * c + j] = fmaf(O[32 * c + j], s_alpha[64 * kh + 32 * c + j], __uint_as_float(v[j]));
          O[32 * c + 16 + j] = fmaf(O[32 * c + 16 + j], s_alpha[64 * kh + 32 * c + 16 + j], __uint_as_float(u[j]));
        }
      }
    };
    for (int i = 0; i < n; ++i) {
      const int buf = i & 1;
      // the step's scores, and its norms and masks (written by the expansion warps: their own
      // barrier orders them before these reads; it has completed before the scores can)
      ok = pf_wait(&bars[PB_SFULL + buf], (i >> 1) & 1, abort, a.v.status);
      ok = wg_all(ok && pf_wait(&bars[PB_KFULL + buf], (i >> 1) & 1, abort, a.v.status), 2, 256);
      if (!ok) break;
      tc_fence_after();
      const int kb = PF_BN * (s_lo + i) + 32 * kh;  // position of this thread's first key
      uint32_t vmask = live ? s_mkv[2 * buf + kh] : 0u;
      if (qpos - kb < 31) vmask &= qpos < kb ? 0u : (2u << (qpos - kb)) - 1u;  // causal: keys <= qpos
      const float* nkb = s_nk + 64 * buf + 32 * kh;
      const float* nvb = s_nv + 64 * buf + 32 * kh;
      const bool full = __all_sync(0xffffffffu, vmask == 0xFFFFFFFFu);
      float sv[32];
      float mx = -CUDART_INF_F;
      {
        uint32_t v[32];
        tmem_ld16(tlane + PF_S_COL + 64 * buf + 32 * kh, *reinterpret_cast<uint32_t(*)[16]>(v));
        tmem_ld16(tlane + PF_S_COL + 64 * buf + 32 * kh + 16, *reinterpret_cast<uint32_t(*)[16]>(v + 16));
        tmem_wait_ld();
        if (full) {  // every key of the half valid for every row of the warp (below the diagonal)
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            sv[k] = __uint_as_float(v[k]) * nkb[k] * qs;
            mx = fmaxf(mx, sv[k]);
          }
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            sv[k] = ((vmask >> k) & 1u) ? __uint_as_float(v[k]) * nkb[k] * qs : -CUDART_INF_F;
            mx = fmaxf(mx, sv[k]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars[PB_SFREE + buf]);  // the scores of this buffer are read
      s_red[128 * kh + r] = mx;
      // the P buffer is free once the previous step's P.V is done; the V norms are in once V^T is
      // (this barrier also publishes s_red)
      ok = i == 0 || pf_wait(&bars[PB_OFULL + ((i - 1) & 1)], ((i - 1) >> 1) & 1, abort, a.v.status);
      ok = wg_all(ok && pf_wait(&bars[PB_VFULL + buf], (i >> 1) & 1, abort, a.v.status), 2, 256);
      if (!ok) break;
      const float m_new = fmaxf(m, fmaxf(s_red[r], s_red[128 + r]));
      const float alpha = (m == -CUDART_INF_F) ? 0.f : fast_exp2(m - m_new);
      float lsum = 0.f;
      uint8_t* prow = smem + SM::p;  // row r, keys 32 kh .. 32 kh + 31
#pragma unroll
      for (int c = 0; c < 4; ++c) {  // keys 8 c .. 8 c + 7 of this half: one 16-byte row of a core matrix
        uint32_t ph[4], pl[4];
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
          float pp[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int k = 8 * c + j + e;
            const bool kv = full || ((vmask >> k) & 1u);
            const float p = kv ? fast_exp2(sv[k] - m_new) : 0.f;
            lsum += p;
            pp[e] = kv ? p * nvb[k] : 0.f;
          }
          const __half2 h2 = __floats2half2_rn(pp[0], pp[1]);
          const float2 hf = __half22float2(h2);
          const __half2 l2 = __floats2half2_rn(pp[0] - hf.x, pp[1] - hf.y);
          ph[j >> 1] = *reinterpret_cast<const uint32_t*>(&h2);
          pl[j >> 1] = *reinterpret_cast<const uint32_t*>(&l2);
        }
        const int off = umma_sw128_off(r, 32 * kh + 8 * c, PF_ROWS);
        *reinterpret_cast<uint4*>(prow + off) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
        *reinterpret_cast<uint4*>(prow + 16384 + off) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&bars[PB_PFULL]);
      l = l * alpha + lsum;
      m = m_new;
      if (i >= 1) {  // every row's factor of step i - 1 is in s_alpha (published by the barriers above)
        fold_output(i - 1);
        tc_fence_before();
        mbar_arrive(&bars[PB_OFREE + ((i - 1) & 1)]);
      }
      named_barrier_sync(2, 256);  // s_alpha and s_red are read
      if (kh == 0) s_alpha[r] = alpha;
    }
    if (ok) {
      ok = wg_all(pf_wait(&bars[PB_OFULL + ((n - 1) & 1)], ((n - 1) >> 1) & 1, abort, a.v.status), 2, 256);
      if (ok) {
        tc_fence_after();
        fold_output(n - 1);
      }
    }
    // partials: (m, l) of row r (the two key halves' sums), and coordinate r of rows 64 kh ..
    named_barrier_sync(2, 256);
    s_red[128 * kh + r] = l;
    named_barrier_sync(2, 256);
    if (kh == 0)
      a.part_ml[prow0 + r] = make_float2(live && ok ? m : -CUDART_INF_F, live && ok ? l + s_red[128 + r] : 0.f);
    float* po = a.part_o + (prow0 + 64 * kh) * D + r;
#pragma unroll
    for (int j = 0; j < PF_ROWS / 2; ++j) po[(size_t)j * D] = O[j];
  } else if (warp < 12) {
    // ==== code expansion: K as 64 keys x 128 coordinates, V^T as 128 coordinates x 64 keys
    const int e = tid - 256;
    const int key = e & 63, half = e >> 6;  // K: key and half of its coordinates
    const int d = e, g = d & 7, hh = (d >> 3) & 1, e2 = (d >> 4) & 1, w = d >> 5;  // V: coordinate d
    uint32_t kl0[4], kh0[4], kl1[4], kh1[4], vl0[4], vh0[4], vl1[4], vh1[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      kl0[t] = a.kc.k.f16_lb[0][t]; kh0[t] = a.kc.k.f16_hb[0][t];
      kl1[t] = a.kc.k.f16_lb[1][t]; kh1[t] = a.kc.k.f16_hb[1][t];
      vl0[t] = a.kc.v.f16_lb[0][t]; vh0[t] = a.kc.v.f16_hb[0][t];
      vl1[t] = a.kc.v.f16_lb[1][t]; vh1[t] = a.kc.v.f16_hb[1][t];
    }
    for (int i = 0; i < n; ++i) {
      const int buf = i & 1;
      // K (single buffer: the score MMAs of step i - 1 are done), its norms and masks (their
      // buffer: the softmax of step i - 2 has read them)
      bool ok = pf_wait(&bars[PB_REC + buf], (i >> 1) & 1, abort, a.v.status);
      ok = ok && (i == 0 || pf_wait(&bars[PB_KFREE], (i - 1) & 1, abort, a.v.status));
      ok = ok && pf_wait(&bars[PB_SFREE + buf], ((i >> 1) & 1) ^ 1, abort, a.v.status);
      if (!wg_all(ok, 1, 128)) break;
      const uint8_t* recb = smem + SM::rec + buf * 2 * TB;
      {  // K: coordinates 64 half .. 64 half + 63 of key `key`, eight per 16-byte core-matrix row
        const uint8_t* kr = recb + (key >> 5) * TB + (key & 31) * k_rec_bytes(KB);
        uint8_t* khi = smem + SM::k0;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int c = 2 * half + cc;
          uint32_t wd[KB], sel[4];
#pragma unroll
          for (int t = 0; t < KB; ++t) wd[t] = reinterpret_cast<const uint32_t*>(kr + c * chunk_bytes(KB))[t];
          chunk_selectors<KB>(wd, sel);
#pragma unroll
          for (int wq = 0; wq < 4; ++wq) {
            const uint2 a0 = lut_f16x4<KB>(kl0, kh0, sel[wq]), a1 = lut_f16x4<KB>(kl0, kh0, sel[wq] >> 16);
            const uint2 b0 = lut_f16x4<KB>(kl1, kh1, sel[wq]), b1 = lut_f16x4<KB>(kl1, kh1, sel[wq] >> 16);
            const int off = umma_sw128_off(key, 8 * (4 * c + wq), PF_BN);
            *reinterpret_cast<uint4*>(khi + off) = make_uint4(a0.x, a0.y, a1.x, a1.y);
            *reinterpret_cast<uint4*>(khi + 16384 + off) = make_uint4(b0.x, b0.y, b1.x, b1.y);
          }
        }
      }
      if (e < 64) {  // the step's K norms and token masks
        s_nk[64 * buf + e] = __half2float(reinterpret_cast<const __half*>(recb + (e >> 5) * TB + tr_kn(KB, VB))[e & 31]);
      } else if (e < 66) {
        s_mkv[2 * buf + (e - 64)] = s_mrec[2 * buf + (e - 64)];
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&bars[PB_KFULL + buf]);
      // V^T and the V norms (buffer buf: the output MMAs of step i - 2 are done)
      if (!wg_all(pf_wait(&bars[PB_VFREE + buf], ((i >> 1) & 1) ^ 1, abort, a.v.status), 1, 128)) break;
      {  // V^T: coordinate d of the 64 keys.  Coordinate d = 32 w + 16 e2 + 8 hh + g of the
         // block's tokens u sits in chunk (g, tq = (u mod 8) / 2, hh), selector word w, nibble
         // m + 4 e2 (m = 2 (u / 8) + u mod 2): byte 2 e2 of that word holds tokens 2 tq, 2 tq + 1,
         // byte 2 e2 + 1 tokens 2 tq + 8, 2 tq + 9.
        uint8_t* vhi = smem + SM::vt0 + buf * 32768;
        const uint32_t b0 = 2 * e2, b1 = 2 * e2 + 1;
        const uint32_t sl0 = b0 | ((4 + b0) << 4), sl1 = b1 | ((4 + b1) << 4);
#pragma unroll
        for (int v16 = 0; v16 < 4; ++v16) {  // the step's four 16-token V blocks
          const uint8_t* vb = recb + (v16 >> 1) * TB + tr_v(KB) + (v16 & 1) * v_blk_bytes(VB);
          uint32_t s[4];
#pragma unroll
          for (int tq = 0; tq < 4; ++tq)
            s[tq] = chunk_selector<VB>(
                reinterpret_cast<const uint32_t*>(vb + 2 * chunk_bytes(VB) * (4 * g + tq) + hh * chunk_bytes(VB)), w);
          const uint32_t sA = prmt(s[0], s[1], sl0), sB = prmt(s[2], s[3], sl0);  // tokens 0-3, 4-7
          const uint32_t sC = prmt(s[0], s[1], sl1), sD = prmt(s[2], s[3], sl1);  // tokens 8-11, 12-15
          const int off0 = umma_sw128_off(d, 16 * v16, 128), off1 = umma_sw128_off(d, 16 * v16 + 8, 128);
          const uint2 hA = lut_f16x4<VB>(vl0, vh0, sA), hB = lut_f16x4<VB>(vl0, vh0, sB);
          const uint2 hC = lut_f16x4<VB>(vl0, vh0, sC), hD = lut_f16x4<VB>(vl0, vh0, sD);
          *reinterpret_cast<uint4*>(vhi + off0) = make_uint4(hA.x, hA.y, hB.x, hB.y);
          *reinterpret_cast<uint4*>(vhi + off1) = make_uint4(hC.x, hC.y, hD.x, hD.y);
          const uint2 lA = lut_f16x4<VB>(vl1, vh1, sA), lB = lut_f16x4<VB>(vl1, vh1, sB);
          const uint2 lC = lut_f16x4<VB>(vl1, vh1, sC), lD = lut_f16x4<VB>(vl1, vh1, sD);
          *reinterpret_cast<uint4*>(vhi + 16384 + off0) = make_uint4(lA.x, lA.y, lB.x, lB.y);
          *reinterpret_cast<uint4*>(vhi + 16384 + off1) = make_uint4(lC.x, lC.y, lD.x, lD.y);
        }
      }
      if (e < 64)
        s_nv[64 * buf + e] = __half2float(reinterpret_cast<const __half*>(recb + (e >> 5) * TB + tr_vn(KB, VB))[e & 31]);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the tiles, and the record reads, before the async proxy
      mbar_arrive(&bars[PB_VFULL + buf]);
      mbar_arrive(&bars[PB_RECFREE + buf]);
    }
  } else if (warp == 13) {
    // ==== loads: the records of step i go into buffer i % 2 once the expansion warps have read
    // the records of step i - 2 (steps 0 and 1 were staged before the query rotation)
    if (lane == 0) {
      int i = 2;
      for (; i < n; ++i) {
        const int buf = i & 1;
        if (!pf_wait(&bars[PB_RECFREE + buf], ((i >> 1) & 1) ^ 1, abort, a.v.status)) break;
        pf_stage(a, b, kvh, s_lo + i, kv_end, smem + SM::rec + buf * 2 * TB, s_mrec + 2 * buf, &bars[PB_REC + buf], TB);
      }
      // leave no bulk copy in flight (only after a timed-out wait can one be pending)
      for (int j = max(0, i - 2); j < i && j < n; ++j) mbar_wait(&bars[PB_REC + (j & 1)], (j >> 1) & 1, nullptr);
    }
  } else if (warp == 12 && lane == 0) {
    // ==== score MMAs: S_i = Q K_i^T (hi.hi, lo.hi, hi.lo) once K_i is expanded and buffer i % 2 read
    const uint32_t idS = umma_idesc_f16(128, PF_BN);
    const uint32_t qh = smem_addr(smem + SM::q_hi), ql = smem_addr(smem + SM::q_lo);
    const uint32_t kh = smem_addr(smem + SM::k0), kl = kh + 16384;
    for (int i = 0; i < n; ++i) {
      const int buf = i & 1;
      if (!pf_wait(&bars[PB_KFULL + buf], (i >> 1) & 1, abort, a.v.status)) break;
      if (!pf_wait(&bars[PB_SFREE + buf], ((i >> 1) & 1) ^ 1, abort, a.v.status)) break;
      tc_fence_after();
      const uint32_t dst = tmem + PF_S_COL + 64 * buf;
      // k-step ks: K block ks / 4, 32 bytes per step inside it (128 query rows, 64 keys)
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_f16(dst, umma_sdesc_sw128(qh + (ks >> 2) * 16384 + (ks & 3) * 32),
                 umma_sdesc_sw128(kh + (ks >> 2) * 8192 + (ks & 3) * 32), idS, ks > 0);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_f16(dst, umma_sdesc_sw128(ql + (ks >> 2) * 16384 + (ks & 3) * 32),
                 umma_sdesc_sw128(kh + (ks >> 2) * 8192 + (ks & 3) * 32), idS, 1);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        umma_f16(dst, umma_sdesc_sw128(qh + (ks >> 2) * 16384 + (ks & 3) * 32),
                 umma_sdesc_sw128(kl + (ks >> 2) * 8192 + (ks & 3) * 32), idS, 1);
      umma_commit(&bars[PB_SFULL + buf]);
      umma_commit(&bars[PB_KFREE]);
    }
    umma_commit(&bars[PB_DRAIN_S]);  // every MMA issued is complete before tensor memory is released
    mbar_wait(&bars[PB_DRAIN_S], 0, nullptr);
  } else if (warp == 14 && lane == 0) {
    // ==== output MMAs: O_i^T = V_i^T P_i'^T (V hi.P hi, V lo.P hi, V hi.P lo) once P_i' is written
    const uint32_t idO = umma_idesc_f16(128, 128);
    const uint32_t pa = smem_addr(smem + SM::p);
    for (int i = 0; i < n; ++i) {
      const int buf = i & 1;
      if (!pf_wait(&bars[PB_VFULL + buf], (i >> 1) & 1, abort, a.v.status)) break;
      if (!pf_wait(&bars[PB_PFULL], i & 1, abort, a.v.status)) break;
      if (!pf_wait(&bars[PB_OFREE + buf], ((i >> 1) & 1) ^ 1, abort, a.v.status)) break;
      tc_fence_after();
      const uint32_t vh = smem_addr(smem + SM::vt0 + buf * 32768), vl = vh + 16384;
      const uint32_t dst = tmem + PF_O_COL + 128 * buf;
      // k-step ks: 32 bytes per step in the single K block (64 keys)
#pragma unroll
      for (int ks = 0; ks < PF_BN / 16; ++ks)
        umma_f16(dst, umma_sdesc_sw128(vh + 32 * ks), umma_sdesc_sw128(pa + 32 * ks), idO, ks > 0);
#pragma unroll
      for (int ks = 0; ks < PF_BN / 16; ++ks)
        umma_f16(dst, umma_sdesc_sw128(vl + 32 * ks), umma_sdesc_sw128(pa + 32 * ks), idO, 1);
#pragma unroll
      for (int ks = 0; ks < PF_BN / 16; ++ks)
        umma_f16(dst, umma_sdesc_sw128(vh + 32 * ks), umma_sdesc_sw128(pa + 16384 + 32 * ks), idO, 1);
      umma_commit(&bars[PB_OFULL + buf]);
      umma_commit(&bars[PB_VFREE + buf]);
    }
    umma_commit(&bars[PB_DRAIN_O]);
    mbar_wait(&bars[PB_DRAIN_O], 0, nullptr);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_free(tmem, PF_TMEM_COLS);
}

// Merge of the splits of every group: CTA (group, block of 8 rows), warp per row, one pass over
// the splits (online rescaling); normalise; inverse rotation.
static __global__ void __launch_bounds__(DEC_THREADS) prefill_merge_kernel(PreArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float sprm[256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Hkv = a.v.n_kv_heads, G = a.g_real, TQ = pf_tokens(G);
  const int group = blockIdx.x;
  const int qb = group % a.n_qblk, kvh = (group / a.n_qblk) % Hkv, b = group / (a.n_qblk * Hkv);
  const int tok0 = qb * TQ, n_live = min(TQ, a.n_tok - tok0);
  if (threadIdx.x < params_per_head(a.v.rot) / 4)
    reinterpret_cast<float4*>(sprm)[threadIdx.x] =
        reinterpret_cast<const float4*>(a.params_layer + (size_t)kvh * params_per_head(a.v.rot))[threadIdx.x];
  __syncthreads();
  const int r = DEC_WARPS * blockIdx.y + warp;
  const int tok = r / G, h = r % G;
  if (r >= TQ * G || tok >= n_live) return;
  float M = -CUDART_INF_F, L = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < a.splits; ++s) {
    const size_t prow = ((size_t)group * a.splits + s) * PF_ROWS + r;
    const float2 ml = a.part_ml[prow];
    const float4 v = reinterpret_cast<const float4*>(a.part_o + prow * D)[lane];
    if (ml.x == -CUDART_INF_F) continue;
    const float Mn = fmaxf(M, ml.x);
    const float fo = (M == -CUDART_INF_F) ? 0.f : fast_exp2(M - Mn), wgt = fast_exp2(ml.x - Mn);
    L = L * fo + ml.y * wgt;
    o[0] = fmaf(v.x, wgt, o[0] * fo); o[1] = fmaf(v.y, wgt, o[1] * fo);
    o[2] = fmaf(v.z, wgt, o[2] * fo); o[3] = fmaf(v.w, wgt, o[3] * fo);
    M = Mn;
  }
  const float sc = L > 0.f ? 0.08838834764831845f / L : 0.f;  // V = n_v c / sqrt(128)
#pragma unroll
  for (int i = 0; i < 4; ++i) o[i] *= sc;
  float Mp[4][4];
  variant_block_matrix(a.v.rot, sprm + lane * params_per_block(a.v.rot), Mp);
  warp_rotate_inverse(o, Mp, a.v.rot == ROT_ISO);
  reinterpret_cast<float4*>(a.out + (((size_t)b * a.n_tok + tok0 + tok) * a.n_q_heads + (size_t)kvh * G + h) * D)[lane] =
      make_float4(o[0], o[1], o[2], o[3]);
}

// Splits per group: at most one CTA per SM in all, each with at least four steps.
inline int prefill_splits(int groups, int max_steps, int n_sm) {
  int s = std::max(1, n_sm / std::max(groups, 1));
  s = std::min(s, std::max(1, max_steps / 4));
  return std::max(1, std::min(s, 64));
}

// Workspace rows (partials) of one call, for the group size g.
inline size_t prefill_rows(int batch, int n_tok, int n_kv_heads, int max_ctx, int g, int n_sm, int* splits_out) {
  const int n_qblk = (n_tok + pf_tokens(g) - 1) / pf_tokens(g);
  const int groups = batch * n_kv_heads * n_qblk;
  const int splits = prefill_splits(groups, (max_ctx + PF_BN - 1) / PF_BN, n_sm);
  if (splits_out) *splits_out = splits;
  return (size_t)groups * splits * PF_ROWS;
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
  a.n_qblk = (n_tok + pf_tokens(a.g_real) - 1) / pf_tokens(a.g_real);
  const int groups = batch * v.n_kv_heads * a.n_qblk;
  const size_t rows = prefill_rows(batch, n_tok, v.n_kv_heads, max_ctx, a.g_real, n_sm, &a.splits);
  a.max_ctx = max_ctx;
  a.start = start;
  a.params_layer = params_layer;
  a.part_ml = (float2*)workspace;
  a.part_o = (float*)((char*)workspace + ((rows * sizeof(float2) + 255) & ~(size_t)255));
  a.out = out;
  a.kc = kc;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaFuncSetAttribute(prefill_kernel<KB, VB>, cudaFuncAttributeMaxDynamicSharedMemorySize, PfSmem<KB, VB>::bytes);
  });
  int e = (int)launch_pdl(prefill_kernel<KB, VB>, dim3(groups * a.splits), dim3(PF_THREADS), PfSmem<KB, VB>::bytes,
                          (cudaStream_t)stream, a);
  if (e) return e;
  return (int)launch_pdl(prefill_merge_kernel, dim3(groups, PF_ROWS / DEC_WARPS), dim3(DEC_THREADS), 0,
                         (cudaStream_t)stream, a);
}

}  // namespace iq
