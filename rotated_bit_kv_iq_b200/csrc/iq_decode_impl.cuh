// Decode attention directly on the packed 3-bit cache.
//
// "RotaryQuant" (rebasdaily.com, section "妙处不只是压缩，而是不再展开") and its abstract
// (arXiv 2608.08081): queries are matched against packed keys, softmax is taken, values are
// accumulated from the packed values, and the inverse rotation is applied at the end;
// full-precision K/V are never built.  "RotorQuant" (sd114.wiki, "3. V 缓存的逆旋转修复"):
// the value sum must be mapped back with the inverse rotation.
//
// One kernel per call.  The work is the list of 32-token tiles of every (sequence, kv head)
// group, group after group; CTA c takes the contiguous run [cT/N, (c+1)T/N) of the T tiles,
// so every CTA gets the same number of tiles whatever the context lengths.  The run is cut
// into segments at group boundaries.  In a segment the 8 warps take the tiles round robin;
// each warp streams its tiles through its own ring of shared-memory slots with bulk copies
// (one mbarrier per slot) and, per tile, on the tensor cores (mma.sync int8, m16n8k32):
//   * scores: S^T = Q' K^T with the 8 query heads' int8 hi/lo rows as M (16 rows; a third
//     int8 term of q is a second A operand), the 32 tokens as four n-tiles and the 128
//     rotated coordinates as K; the K codes become
//     int8 centroid values hi_k, lo_k (alpha8 c_k = hi_k + lo_k/254) by byte-permute table
//     lookups, two per four codes;
//   * online softmax per head on the lane that holds the head's scores; the V norm joins the
//     probability (P' = 2^(s - m) n_v), which is quantised to int8 hi/lo with a scale per
//     tile and head (127 / max P'), undone when the tile's value sums are accumulated;
//   * values: O^T += V^T P' with the 128 coordinates as eight m-tiles, the 32 tokens as K and
//     the heads as N; V blocks are laid out so that every A register is one table lookup.
// s32 accumulators start at a magic constant so one float subtraction converts them.  With
// at most four query heads per kv head the lower terms of q and P' ride in the mma rows and
// columns the group leaves free (template P4), so a tile takes 48 mma instead of 72.
// At a segment end the warps' (m, l, O) are merged in shared memory and written as one
// partial per (CTA, group), announced by a release-ordered count.  After its run, the k-th
// CTA of a group (k < heads per kv head) waits for the group's count, merges head k (and
// k + n, ... for n CTAs) over all partials, normalises and applies R^T: no second kernel.
#pragma once
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <mutex>

#include "iq_device.cuh"

namespace iq {

constexpr int DEC_WARPS = 8;
constexpr int DEC_THREADS = DEC_WARPS * 32;
constexpr int TT = 32;  // tokens per tile
static_assert(TT == TILE_TOKENS, "a tile is one tile record");
constexpr int HMAX = 8;                     // query heads per kv head (layout width)
constexpr int SO_STRIDE = 132;              // floats per (warp, head) row of the merge buffer
constexpr int QF_WORDS = 28;  // query fragment words per lane: 16 (hi, lo) + 8 (lo2) + 4 (bank skew)
constexpr float kLog2e = 1.4426950408889634f;

// Tiles in flight per warp by default: three while a tile record is at most 3200 bytes.
IQ_HD constexpr int dec_nslot(int kb, int vb) { return tile_bytes(kb, vb) <= 3200 ? 3 : 2; }

// Shared memory of one decode CTA for code widths (KB, VB).  A ring slot holds one tile record as
// stored (one bulk copy); each warp has NS of them.
template <int KB, int VB, int NS = dec_nslot(KB, VB)>
struct DecSmem {
  static constexpr int SLOT_BYTES = tile_bytes(KB, VB);
  static constexpr int NSLOT = NS;                                        // tiles in flight per warp
  static constexpr int SL_K = 0, SL_V = tr_v(KB), SL_KN = tr_kn(KB, VB), SL_VN = tr_vn(KB, VB);
  static constexpr int ring = 0;                                          // [warp][slot] tiles
  static constexpr int so = ring + DEC_WARPS * NSLOT * SLOT_BYTES;        // float [warp-4][head][SO_STRIDE]
  static constexpr int sm = so + (DEC_WARPS - 4) * HMAX * SO_STRIDE * 4;  // float [warp][head] maxima
  static constexpr int sl = sm + DEC_WARPS * HMAX * 4;                    // float [warp][head] sums
  static constexpr int qfrag = sl + DEC_WARPS * HMAX * 4;                 // uint32 [lane][QF_WORDS] query fragments
  static constexpr int kappa = qfrag + 32 * QF_WORDS * 4;                 // float [head] score scales
  static constexpr int sparams = kappa + HMAX * 4;                        // float [256] one head's parameters
  static constexpr int appbar = sparams + 256 * 4;                        // uint64: new token appended
  static constexpr int valid = appbar + 16;                               // uint32 [warp][slot] token masks
  static constexpr int bars = valid + DEC_WARPS * NSLOT * 4;              // uint64 [warp][slot]
  static constexpr int cursors = bars + DEC_WARPS * NSLOT * 8;           // Cursor [warp]
  static constexpr int plan = cursors + DEC_WARPS * 48;  // int [batch+1] tile prefix, [batch] ctx, [batch] fp16 prefix
  static size_t bytes(int batch) { return (size_t)plan + 4 * (size_t)(3 * batch + 1); }
  static_assert(appbar % 8 == 0 && bars % 8 == 0, "mbarriers are 8-byte aligned");
};

struct Workspace {
  uint32_t* counters;  // [2][groups]: partials written, merges finished; zero between calls
  float2* part_ml;     // [slots][HMAX] (max in log2 units, sum of 2^(s-max))
  float* part_o;       // [slots][HMAX][128]
};
Workspace carve_workspace(void* ws, int batch, int n_kv_heads, int extra_slots = 0);
int workspace_base_slots(int batch, int n_kv_heads);  // partial slots of the CTAs; extra slots follow

struct DecArgs {
  LayerView v;
  const void* q;
  int q_f32, n_q_heads, g_real, batch, max_ctx;
  const int32_t* ctx_len;
  const float* params_layer;
  float* out;
  Workspace ws;
  const __half* k_new;
  const __half* v_new;
  KernelConsts kc;
  // deferred quantisation: positions 0 .. pre_len[b]-1 of sequence b are held in fp16 outside the
  // packed cache (NULL: none); their attention arrives as n_extra partials per group, at partial
  // slots extra_base + gid * n_extra + s, written by the preceding kernel
  const int32_t* pre_len;
  int n_extra, extra_base;
};

// ------------------------------------------------------------------ work plan
// pre[b] = tiles of sequences 0..b-1 (per kv head) and pre[B + 1 + b] = the clamped context
// length of sequence b; every CTA builds the same table.
static // Clamped context length and fp16 prefix length of sequence b (flags out-of-range values once).
__device__ __forceinline__ void seq_lengths(const DecArgs& a, int b, int& c, int& p) {
  c = a.ctx_len[b];
  if (c < 0 || c > a.max_ctx) {
    if (a.v.status && blockIdx.x == 0) atomicOr(a.v.status, IQ_DEVERR_CTX);
    c = c < 0 ? 0 : a.max_ctx;
  }
  p = 0;
  if (a.pre_len) {  // 0 <= prefix < ctx: the step's new token is always packed
    p = a.pre_len[b];
    if (p < 0 || (c > 0 && p >= c)) {
      if (a.v.status && blockIdx.x == 0) atomicOr(a.v.status, IQ_DEVERR_CTX);
      p = p < 0 ? 0 : max(c - 1, 0);
    }
  }
}
// Packed tiles of a sequence: absolute tiles p/32 .. ceil(c/32)-1.
__device__ __forceinline__ int seq_tiles(int c, int p) { return c > 0 ? (c + TT - 1) / TT - p / TT : 0; }

static __device__ void build_plan(const DecArgs& a, int* pre) {
  const int B = a.batch;
  const int per = (B + DEC_THREADS - 1) / DEC_THREADS;
  const int lo = threadIdx.x * per, hi = min(B, lo + per);
  int sum = 0;
  for (int b = lo; b < hi; ++b) {
    int c, p;
    seq_lengths(a, b, c, p);
    sum += seq_tiles(c, p);
  }
  // block-wide exclusive scan of the per-thread sums
  __shared__ int warp_tot[DEC_WARPS];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int base = 0;
  for (int w = 0; w < warp; ++w) base += warp_tot[w];
  int run = base + incl - sum;
  for (int b = lo; b < hi; ++b) {
    pre[b] = run;
    int c = a.ctx_len[b], p = a.pre_len ? a.pre_len[b] : 0;
    c = c < 0 ? 0 : (c > a.max_ctx ? a.max_ctx : c);
    p = p < 0 ? 0 : ((c > 0 && p >= c) ? max(c - 1, 0) : p);
    pre[B + 1 + b] = c;
    pre[2 * B + 1 + b] = p;
    run += seq_tiles(c, p);
  }
  if (threadIdx.x == DEC_THREADS - 1) pre[B] = run;
  __syncthreads();
}

// Group holding global tile x (x < T): sequence b, kv head, first global tile of the group.
struct Seg {
  int b, kvh, ntiles, lo, hi;  // tiles [lo, hi) of the group's ntiles lie in this CTA
  int ctx;                     // context length of sequence b (clamped)
  int plo, first;              // fp16 prefix length (packed positions start there) and its tile
  long long gstart;
};
__device__ __forceinline__ Seg segment_at(const DecArgs& a, const int* pre, int B, int Hkv, long long x, long long c1) {
  int lo = 0, hi = B - 1;  // largest b with Hkv * pre[b] <= x
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((long long)Hkv * pre[mid] <= x) lo = mid; else hi = mid - 1;
  }
  // the largest such b has tiles (an empty b would share its prefix with b + 1, and x < T)
  Seg s;
  s.b = lo;
  s.ntiles = pre[lo + 1] - pre[lo];
  const long long off = x - (long long)Hkv * pre[s.b];
  s.kvh = (int)(off / s.ntiles);
  s.gstart = (long long)Hkv * pre[s.b] + (long long)s.kvh * s.ntiles;
  s.lo = (int)(x - s.gstart);
  s.hi = (int)min((long long)s.ntiles, c1 - s.gstart);
  s.ctx = pre[B + 1 + s.b];
  s.plo = pre[2 * B + 1 + s.b];
  s.first = s.plo / TT;
  return s;
}

__device__ __forceinline__ long long cta_begin(int c, long long T, int n) { return (long long)c * T / n; }
__device__ __forceinline__ int cta_of(long long x, long long T, int n) { return (int)(((x + 1) * n - 1) / T); }

// ------------------------------------------------------------------ tile loads
// Per-warp fetch cursor over the warp's tiles (round robin inside each segment of the
// CTA's run).  All fields are warp-uniform.  It lives in shared memory between refills: it
// is used once per tile, and registers held across the tile loop would be spilled to local
// memory, whose reloads miss the small L1 left next to a full shared-memory carve-out.
struct Cursor {
  Seg s;
  int i;     // next local tile of segment s for this warp
  int done;
};

static_assert(sizeof(Cursor) <= 48, "one cursor slot per warp");

// Lane 0 reads the block-table entry of the cursor's tile early, so that the load is in
// flight while the warp computes (the entry is checked when the copy is issued).
__device__ __forceinline__ int cursor_page(const Cursor& c, const LayerView& v) {
  if (c.done || (threadIdx.x & 31) != 0) return -1;
  const int t = TT * (c.s.first + c.i);
  int pg = c.s.b;
  if (v.block_table && t < c.s.ctx) {
    const int idx = t / v.page_size;
    pg = idx < v.max_pages ? __ldg(v.block_table + (size_t)c.s.b * v.max_pages + idx) : -1;
  }
  return pg;
}

__device__ __forceinline__ void cursor_normalise(Cursor& c, const DecArgs& a, const int* pre, int B, int Hkv, long long c1,
                                                 int warp) {
  while (!c.done && c.i >= c.s.hi) {
    const long long nx = c.s.gstart + c.s.hi;
    if (nx >= c1) { c.done = true; break; }
    c.s = segment_at(a, pre, B, Hkv, nx, c1);
    c.i = c.s.lo + warp;
  }
}

template <bool FUSED>
__device__ __forceinline__ bool is_new_token_tile(const Seg& s, int i) {
  return FUSED && i == s.ntiles - 1;
}

// Copy tile i (absolute: positions 32i .. 32i+31) of group (b, kvh) -- one tile record -- into slot
// `st` with one bulk copy (lane 0).  raw_pg is the tile's block-table entry (or b without a table),
// validated here; the token mask has bit u set when position 32i + u lies in [lo, ctx) on a valid
// page (lo > 0: the positions below are not in the packed cache).
__device__ __forceinline__ uint32_t token_range_mask(int a, int e) {  // bits [max(a,0), min(e,32))
  a = max(a, 0);
  e = min(e, 32);
  if (e <= a) return 0u;
  return (e == 32 ? 0xFFFFFFFFu : ((1u << e) - 1u)) & ~((1u << a) - 1u);
}
__device__ __forceinline__ void issue_tile(const LayerView& v, int b, int kvh, int i, int ctx, int lo, int raw_pg,
                                           uint8_t* st, uint32_t* valid, uint64_t* bar, uint32_t tbytes) {
  const int t = TT * i;
  int page = -1;
  if (t < ctx) {
    page = raw_pg;
    if (!v.block_table && t >= v.page_size) page = -1;
    if (page < 0 || page >= v.n_pages) {
      if (v.status)
        atomicOr(v.status, page < 0 && (v.block_table ? t / v.page_size >= v.max_pages : true) ? IQ_DEVERR_POSITION
                                                                                              : IQ_DEVERR_PAGE);
      page = -1;
    }
  }
  const uint32_t mask = page < 0 ? 0u : token_range_mask(lo - t, ctx - t);
  *valid = mask;
  mbar_arrive_expect_tx(bar, mask ? tbytes : 0);
  if (mask) bulk_g2s(st, tile_record(v, page, kvh, t % v.page_size), tbytes, bar);
}

// The new token of sequence b (position ctx-1): encode K and V into the cache (whole warp).
// Inlined: as an out-of-line call its register saves cost more than the encoding itself.
template <int KB, int VB>
// One side (0: K, 1: V) of the new token, by one warp; prm: the kv head's rotation parameters
// (shared memory).  The vector and the block-table entry are requested together, the vector
// through L2: the kernel may have started before the one that wrote k_new and v_new finished
// (see decode_kernel).
__device__ __forceinline__ void append_new_token(const DecArgs& a, int b, int kvh, int ctx, const float* prm,
                                                 int side) {
  const int p = ctx - 1;
  const int lane = threadIdx.x & 31;
  const size_t off = ((size_t)b * a.v.n_kv_heads + kvh) * D + 4 * lane;
  const uint2 raw = __ldcg(reinterpret_cast<const uint2*>((side ? a.v_new : a.k_new) + off));
  const int page = resolve_page(a.v, b, p);
  float Mp[4][4];
  variant_block_matrix(a.v.rot, prm + lane * params_per_block(a.v.rot), Mp);
  if (page < 0) return;
  if (side == 0)
    warp_encode_loaded<KB>(a.v, raw, kvh, 0, page, p % a.v.page_size, Mp, a.kc.k);
  else
    warp_encode_loaded<VB>(a.v, raw, kvh, 1, page, p % a.v.page_size, Mp, a.kc.v);
}

// ------------------------------------------------------------------ per-tile compute
struct WarpState {
  float m, l;          // head g: running max of the scores s, sum of 2^(s - m)
  float acc[8][4];     // coordinates 16j+g (+8) x heads 2t, 2t+1 (see the mma D layout)
};

__device__ __forceinline__ uint32_t pack4(uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3) {
  return prmt(prmt(x0, x1, 0x0040u), prmt(x2, x3, 0x0040u), 0x5410u);
}

// P4 (at most four query heads per kv head): the mma rows and columns left free by the
// small group carry the query's and the probabilities' lower terms, so the third score mma
// and the third value mma disappear.  Score rows: g < 4 = q hi of head g with q lo2 at row
// g + 8; g >= 4 = q lo of head g - 4 (rows 12..15 zero).  Value columns: n < 4 = P' hi of
// head n, n >= 4 = P' lo of head n - 4; lanes t < 2 accumulate the hi columns, t >= 2 the
// lo columns of the same heads (added together at the segment end).
template <bool P4, int KB, int VB>
__device__ __forceinline__ void process_tile(const uint8_t* __restrict__ st, uint32_t tmask,
                                             const uint32_t* __restrict__ qf, float kappa,
                                             const KernelConsts& kc, WarpState& ws) {
  using SM = DecSmem<KB, VB>;
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  uint32_t KH[4], KL[4], VH[4], VL[4];  // int8 centroid tables (entries beyond 2^bits unused)
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    KH[i] = kc.k.lut_hi[i];
    KL[i] = kc.k.lut_lo[i];
    VH[i] = kc.v.lut_hi[i];
    VL[i] = kc.v.lut_lo[i];
  }
  // ---- scores (head g; tokens 8nt + 2t + e as entry 2nt + e).  Rows of A: q hi (g), q lo
  // (g + 8); a third product adds the q lo2 row against the centroid hi bytes.
  float s[8];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
    const uint32_t* kw =
        reinterpret_cast<const uint32_t*>(st + SM::SL_K + (8 * nt + g) * k_rec_bytes(KB) + chunk_bytes(KB) * t);
    uint32_t kwr[KB];
    if constexpr (KB == 4) {
      const uint4 x = *reinterpret_cast<const uint4*>(kw);
      kwr[0] = x.x; kwr[1] = x.y; kwr[2] = x.z; kwr[3] = x.w;
    } else if constexpr (KB == 2) {
      const uint2 x = *reinterpret_cast<const uint2*>(kw);
      kwr[0] = x.x; kwr[1] = x.y;
    } else {
#pragma unroll
      for (int i = 0; i < KB; ++i) kwr[i] = kw[i];
    }
    uint32_t sel[4];
    chunk_selectors<KB>(kwr, sel);
    int a1[4] = {kMagicI, kMagicI, kMagicI, kMagicI}, a2[4] = {kMagicI, kMagicI, kMagicI, kMagicI};
    int a3[4] = {kMagicI, kMagicI, kMagicI, kMagicI};
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const uint32_t s0 = sel[cc], s1 = sel[cc] >> 16;
      const uint32_t bh0 = lut4<KB>(KH, s0), bh1 = lut4<KB>(KH, s1);
      const uint4 qv = reinterpret_cast<const uint4*>(qf)[cc];
      imma16832(a1, qv.x, qv.y, qv.z, qv.w, bh0, bh1, a1[0], a1[1], a1[2], a1[3]);
      imma16832(a2, qv.x, qv.y, qv.z, qv.w, lut4<KB>(KL, s0), lut4<KB>(KL, s1), a2[0], a2[1], a2[2], a2[3]);
      if (!P4) {
        const uint2 qw = reinterpret_cast<const uint2*>(qf + 16)[cc];
        imma16832(a3, qw.x, 0u, qw.y, 0u, bh0, bh1, a3[0], a3[1], a3[2], a3[3]);
      }
    }
    if (P4) {
      // rows g >= 4 hold lo.c_hi (a1) and lo.c_lo (a2) of head g - 4: scaled here and added by
      // lane g - 4 (lane - 16); rows g + 8 of lanes g < 4 hold lo2.c_hi
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float w = fmaf(magic_to_float(a2[e]), 1.0f / (254.0f * 254.0f), magic_to_float(a1[e]) * (1.0f / 254.0f));
        const float w_lo = __shfl_xor_sync(0xffffffffu, w, 16);
        s[2 * nt + e] = fmaf(magic_to_float(a1[2 + e]), 1.0f / (254.0f * 254.0f),
                             fmaf(magic_to_float(a2[e]), 1.0f / 254.0f, magic_to_float(a1[e]))) + w_lo;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        // hh + (lo.c_hi + hi.c_lo)/254 + (lo.c_lo + lo2.c_hi)/254^2; each pair of raw
        // accumulators sums to 2 * 1.5 * 2^23 + x, so one subtraction removes both offsets
        const float x1 = (__int_as_float(a1[2 + e]) + __int_as_float(a2[e])) - 2.f * kMagicF;
        const float x2 = (__int_as_float(a2[2 + e]) + __int_as_float(a3[e])) - 2.f * kMagicF;
        s[2 * nt + e] = fmaf(fmaf(x2, 1.0f / 254.0f, x1), 1.0f / 254.0f, magic_to_float(a1[e]));
      }
    }
  }
  // ---- norms, masks, online softmax (head g)
  float nv[8], mx = -CUDART_INF_F;
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
    const int tok = 8 * nt + 2 * t;
    const float2 nk = __half22float2(*reinterpret_cast<const __half2*>(st + SM::SL_KN + 2 * tok));
    const float2 nvv = __half22float2(*reinterpret_cast<const __half2*>(st + SM::SL_VN + 2 * tok));
    s[2 * nt] *= nk.x * kappa;
    s[2 * nt + 1] *= nk.y * kappa;
    nv[2 * nt] = nvv.x;
    nv[2 * nt + 1] = nvv.y;
  }
  if (tmask != 0xFFFFFFFFu) {  // a partial tile: tokens outside the context or on bad pages
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int tok = 8 * (i >> 1) + 2 * t + (i & 1);
      if (!((tmask >> tok) & 1u)) {
        s[i] = -CUDART_INF_F;
        nv[i] = 0.f;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) mx = fmaxf(mx, s[i]);
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  const float m_new = fmaxf(ws.m, mx);
  if (__any_sync(0xffffffffu, m_new > ws.m)) {
    const float r = (m_new > ws.m) ? fast_exp2(ws.m - m_new) : 1.f;
    ws.l *= r;
    const int hl = P4 ? 8 * (t & 1) : 8 * t;  // lane of the head of columns 2t, 2t+1
    const float r0 = __shfl_sync(0xffffffffu, r, hl), r1 = __shfl_sync(0xffffffffu, r, hl + 4);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      ws.acc[j][0] *= r0;
      ws.acc[j][2] *= r0;
      ws.acc[j][1] *= r1;
      ws.acc[j][3] *= r1;
    }
    ws.m = m_new;
  }
  // P' = 2^(s - m) n_v, quantised per (tile, head) to int8 hi/lo with scale 127 / max P'
  float pv[8], pmax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float p = (ws.m == -CUDART_INF_F) ? 0.f : fast_exp2(s[i] - ws.m);
    ws.l += p;
    pv[i] = p * nv[i];
    pmax = fmaxf(pmax, pv[i]);
  }
  pmax = fmaxf(pmax, __shfl_xor_sync(0xffffffffu, pmax, 1));
  pmax = fmaxf(pmax, __shfl_xor_sync(0xffffffffu, pmax, 2));
  const float gam = pmax > 0.f ? __fdividef(127.f, pmax) : 0.f;  // x = pv gam stays <= 127 (1-ulp quotient)
  const float ig = pmax > 0.f ? pmax * (1.0f / 127.0f) : 0.f;
  const int hl = P4 ? 8 * (t & 1) : 8 * t;
  const float igs = (P4 && t >= 2) ? 1.0f / 254.0f : 1.0f;  // P4: lo columns carry P' lo
  const float ig0 = __shfl_sync(0xffffffffu, ig, hl) * igs, ig1 = __shfl_sync(0xffffffffu, ig, hl + 4) * igs;
  uint32_t hb[8], lb[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float x = pv[i] * gam;  // in [0, 127]
    hb[i] = round_low_bits(x);
    const float h = __int_as_float((int)hb[i]) - kMagicF;
    lb[i] = round_low_bits((x - h) * 254.f);
  }
  uint32_t bh0 = pack4(hb[0], hb[1], hb[2], hb[3]), bh1 = pack4(hb[4], hb[5], hb[6], hb[7]);
  const uint32_t bl0 = pack4(lb[0], lb[1], lb[2], lb[3]), bl1 = pack4(lb[4], lb[5], lb[6], lb[7]);
  if (P4) {  // columns g >= 4: P' lo of head g - 4, from lane - 16
    const uint32_t x0 = __shfl_xor_sync(0xffffffffu, bl0, 16), x1 = __shfl_xor_sync(0xffffffffu, bl1, 16);
    if (g >= 4) { bh0 = x0; bh1 = x1; }
  }
  // ---- values: lane chunks (g, t, h = 0, 1) of each V block = 2 VB words at 8 VB * lane
  uint32_t sv[4][4];  // [block*2 + h][word]
#pragma unroll
  for (int blk = 0; blk < 2; ++blk) {
    const uint2* vw = reinterpret_cast<const uint2*>(st + SM::SL_V + v_blk_bytes(VB) * blk + 2 * chunk_bytes(VB) * lane);
    uint32_t w[2 * VB];
#pragma unroll
    for (int i = 0; i < VB; ++i) {
      const uint2 x = vw[i];
      w[2 * i] = x.x;
      w[2 * i + 1] = x.y;
    }
    chunk_selectors<VB>(w, sv[2 * blk]);
    chunk_selectors<VB>(w + VB, sv[2 * blk + 1]);
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int sh = 16 * (j & 1), w = j >> 1;
    const uint32_t c0 = sv[0][w] >> sh, c1 = sv[1][w] >> sh, c2 = sv[2][w] >> sh, c3 = sv[3][w] >> sh;
    const uint32_t h0 = lut4<VB>(VH, c0), h1 = lut4<VB>(VH, c1), h2 = lut4<VB>(VH, c2), h3 = lut4<VB>(VH, c3);
    int d1[4], d2[4];
    imma16832(d1, h0, h1, h2, h3, bh0, bh1, kMagicI, kMagicI, kMagicI, kMagicI);
    if (P4) {
      imma16832(d2, lut4<VB>(VL, c0), lut4<VB>(VL, c1), lut4<VB>(VL, c2), lut4<VB>(VL, c3), bh0, bh1,
                kMagicI, kMagicI, kMagicI, kMagicI);
    } else {
      imma16832(d2, h0, h1, h2, h3, bl0, bl1, kMagicI, kMagicI, kMagicI, kMagicI);
      imma16832(d2, lut4<VB>(VL, c0), lut4<VB>(VL, c1), lut4<VB>(VL, c2), lut4<VB>(VL, c3), bh0, bh1,
                d2[0], d2[1], d2[2], d2[3]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float tv = fmaf(magic_to_float(d2[e]), 1.0f / 254.0f, magic_to_float(d1[e]));
      ws.acc[j][e] = fmaf(tv, (e & 1) ? ig1 : ig0, ws.acc[j][e]);
    }
  }
}

// ------------------------------------------------------------------ query rotation
// Warp h rotates query head h of group (b, kvh), quantises it to int8 hi/lo with scale
// gamma = 127 / max|q'| and writes it in mma A-fragment order: lane l holds coordinates
// 4l..4l+3 = k-slots of chunk cc = (l/2) mod 4, fragment row 4h + l/8.
// P4: head h < 4 fills the fragment rows of lanes g = h (hi, with lo2 as row g + 8) and
// g = h + 4 (lo, row g + 8 zero); see process_tile.
template <bool P4>
__device__ __forceinline__ void rotate_query_row(const void* q, int q_f32, size_t row0, bool live, int rot, float alpha_k,
                                                 int h, const float* prm, uint32_t* qfrag, float* kappa) {
  const int lane = threadIdx.x & 31;
  float x[4] = {0.f, 0.f, 0.f, 0.f};
  if (live) {
    const size_t row = row0 + 4 * lane;
    if (q_f32) {
      const float4 f = __ldcg(reinterpret_cast<const float4*>((const float*)q + row));
      x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
    } else {
      const uint2 u = __ldcg(reinterpret_cast<const uint2*>((const __half*)q + row));
      const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
      const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
      x[0] = f0.x; x[1] = f0.y; x[2] = f1.x; x[3] = f1.y;
    }
    float Mp[4][4];
    variant_block_matrix(rot, prm + lane * params_per_block(rot), Mp);
    warp_rotate_forward(x, Mp, rot == ROT_ISO);
  }
  float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float gam = amax > 0.f ? 127.f / amax : 1.f;
  // q' gamma = hi + lo/254 + lo2/254^2, each an int8 (residuals stay within +-0.5 of a unit)
  uint32_t hi[4], lo[4], lo2[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float y = x[i] * gam;
    hi[i] = round_low_bits(y);
    const float r1 = (y - (__int_as_float((int)hi[i]) - kMagicF)) * 254.f;
    lo[i] = round_low_bits(r1);
    const float r2 = (r1 - (__int_as_float((int)lo[i]) - kMagicF)) * 254.f;
    lo2[i] = round_low_bits(r2);
  }
  const int tq = lane >> 3, cc = (lane >> 1) & 3, e = lane & 1;
  uint32_t* row = qfrag + (4 * h + tq) * QF_WORDS;
  if (P4) {
    uint32_t* row_lo = qfrag + (4 * (h + 4) + tq) * QF_WORDS;
    row[4 * cc + 2 * e] = pack4(hi[0], hi[1], hi[2], hi[3]);
    row[4 * cc + 2 * e + 1] = pack4(lo2[0], lo2[1], lo2[2], lo2[3]);
    row_lo[4 * cc + 2 * e] = pack4(lo[0], lo[1], lo[2], lo[3]);
    row_lo[4 * cc + 2 * e + 1] = 0u;
  } else {
    row[4 * cc + 2 * e] = pack4(hi[0], hi[1], hi[2], hi[3]);
    row[4 * cc + 2 * e + 1] = pack4(lo[0], lo[1], lo[2], lo[3]);
    row[16 + 2 * cc + e] = pack4(lo2[0], lo2[1], lo2[2], lo2[3]);
  }
  if (lane == 0) kappa[h] = live ? kLog2e / (128.f * gam * alpha_k) : 0.f;
}

template <bool P4>
__device__ __forceinline__ void rotate_query(const DecArgs& a, int b, int kvh, int h, const float* prm,
                                             uint32_t* qfrag, float* kappa) {
  rotate_query_row<P4>(a.q, a.q_f32, ((size_t)b * a.n_q_heads + (size_t)kvh * a.g_real + h) * D, h < a.g_real, a.v.rot,
                       a.kc.k.alpha8, h, prm, qfrag, kappa);
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Final merge of one group's partials for the query heads this CTA was given (h = k, k + n,
// ... with k its index among the group's n CTAs), after every partial is in.  Heads are taken
// two at a time, four warps each, one coordinate per lane; when only one of the two exists,
// both warp groups work on it, each over half of the partials, and meet in shared memory.
// O = sum_c 2^(m_c - M) O_c and L likewise, then R^T per head.
// Partial slot of the k-th partial of group gid: the group's CTAs first, then its extra partials.
__device__ __forceinline__ size_t part_slot(const DecArgs& a, int gid, int c_first, int n_parts, int k) {
  return k < n_parts ? (size_t)(c_first + k + gid) : (size_t)a.extra_base + (size_t)gid * a.n_extra + (k - n_parts);
}

__device__ __forceinline__ void merge_group(const DecArgs& a, const Seg& seg, int gid, int c_first, int n_parts, int k,
                                            float* buf, const float* prm) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, grp = warp >> 2;  // groups 0, 1 work
  const int coord = 32 * (warp & 3) + lane;
  float* sacc = buf + 2 * D;                 // [128] group 1's value sums (split case)
  float* sml = buf + 3 * D;                  // [2] group 1's (M, L)
  for (int h0 = k; h0 < a.g_real; h0 += 2 * n_parts) {
    const bool split = h0 + n_parts >= a.g_real;
    const int h = split ? h0 : h0 + grp * n_parts;
    const int half = (n_parts + 1) >> 1;
    const int n_all = n_parts + a.n_extra;
    const int half_all = (n_all + 1) >> 1;
    const int p_lo = split ? grp * half_all : 0, p_hi = split ? (grp ? n_all : half_all) : n_all;
    (void)half;
    float acc = 0.f, M = -CUDART_INF_F, L = 0.f;
    for (int c0 = p_lo; c0 < p_hi && grp < 2; c0 += 32) {
      const int nb = min(32, p_hi - c0);
      float ov[32];
#pragma unroll
      for (int u = 0; u < 32; ++u)
        ov[u] = __ldcg(a.ws.part_o + (part_slot(a, gid, c_first, n_parts, c0 + min(u, nb - 1)) * HMAX + h) * D + coord);
      const float2 ml = lane < nb ? __ldcg(a.ws.part_ml + part_slot(a, gid, c_first, n_parts, c0 + lane) * HMAX + h)
                                  : make_float2(-CUDART_INF_F, 0.f);
      float Mb = ml.x;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) Mb = fmaxf(Mb, __shfl_xor_sync(0xffffffffu, Mb, o));
      Mb = fmaxf(Mb, M);
      if (Mb == -CUDART_INF_F) continue;
      const float fo = (M == -CUDART_INF_F) ? 0.f : fast_exp2(M - Mb);
      const float w = (ml.x == -CUDART_INF_F) ? 0.f : fast_exp2(ml.x - Mb);
      float lw = ml.y * w;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) lw += __shfl_xor_sync(0xffffffffu, lw, o);
      acc *= fo;
#pragma unroll
      for (int u = 0; u < 32; ++u) acc = fmaf(ov[u], __shfl_sync(0xffffffffu, w, u), acc);  // w = 0 past nb
      L = L * fo + lw;
      M = Mb;
    }
    if (split) {
      if (grp == 1) {
        sacc[coord] = acc;
        if (warp == 4 && lane == 0) { sml[0] = M; sml[1] = L; }
      }
      __syncthreads();
      if (grp == 0) {
        const float M1 = sml[0], L1 = sml[1];
        const float Mn = fmaxf(M, M1);
        const float f0 = (M == -CUDART_INF_F) ? 0.f : fast_exp2(M - Mn);
        const float f1 = (M1 == -CUDART_INF_F) ? 0.f : fast_exp2(M1 - Mn);
        acc = acc * f0 + sacc[coord] * f1;
        L = L * f0 + L1 * f1;
      }
    }
    // normalise, gather the head in shared memory, rotate back with one warp
    const bool live = grp < 2 && h < a.g_real && !(split && grp == 1);
    const int slot = split ? 0 : grp;
    if (live) buf[slot * D + coord] = L > 0.f ? acc * (0.08838834764831845f / (a.kc.v.alpha8 * L)) : 0.f;
    __syncthreads();
    if ((warp & 3) == 0 && live) {
      float r[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) r[i] = buf[slot * D + 4 * lane + i];
      float Mp[4][4];
      variant_block_matrix(a.v.rot, prm + lane * params_per_block(a.v.rot), Mp);
      warp_rotate_inverse(r, Mp, a.v.rot == ROT_ISO);
      reinterpret_cast<float4*>(a.out + ((size_t)seg.b * a.n_q_heads + (size_t)seg.kvh * a.g_real + h) * D)[lane] =
          make_float4(r[0], r[1], r[2], r[3]);
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------ the kernel
template <bool FUSED, bool P4, int KB, int VB, int NS = dec_nslot(KB, VB)>
__global__ void __launch_bounds__(DEC_THREADS, 2) decode_kernel(DecArgs a) {
  using DecSmem = iq::DecSmem<KB, VB, NS>;
  constexpr int NSLOT = DecSmem::NSLOT, SLOT_BYTES = DecSmem::SLOT_BYTES;
  pdl_launch_dependents();
  if (!FUSED) pdl_wait();  // a plain call may read anything the previous kernel wrote
  extern __shared__ __align__(128) uint8_t smem[];
  float(*so)[HMAX][SO_STRIDE] = reinterpret_cast<float(*)[HMAX][SO_STRIDE]>(smem + DecSmem::so);
  float(*sm)[HMAX] = reinterpret_cast<float(*)[HMAX]>(smem + DecSmem::sm);
  float(*sl)[HMAX] = reinterpret_cast<float(*)[HMAX]>(smem + DecSmem::sl);
  uint32_t* qfrag = reinterpret_cast<uint32_t*>(smem + DecSmem::qfrag);
  float* kappa = reinterpret_cast<float*>(smem + DecSmem::kappa);
  int* pre = reinterpret_cast<int*>(smem + DecSmem::plan);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Hkv = a.v.n_kv_heads, B = a.batch;
  uint8_t* ring = smem + DecSmem::ring + warp * NSLOT * SLOT_BYTES;
  uint32_t* valid = reinterpret_cast<uint32_t*>(smem + DecSmem::valid) + warp * NSLOT;
  uint64_t* wbar = reinterpret_cast<uint64_t*>(smem + DecSmem::bars) + warp * NSLOT;
  uint64_t* appbar = reinterpret_cast<uint64_t*>(smem + DecSmem::appbar);
  if (lane == 0) {
    for (int s = 0; s < NSLOT; ++s) mbar_init(&wbar[s], 1);
    if (warp == 0) mbar_init(appbar, 2);  // the K and the V half of an append
    mbar_fence_init();
  }
  build_plan(a, pre);  // ends with __syncthreads (barrier inits visible)

  const long long T = (long long)Hkv * pre[B];
  const int n_cta = (int)min((long long)gridDim.x, T);
  const int cta = blockIdx.x;
  const long long c0 = cta < n_cta ? cta_begin(cta, T, n_cta) : 0;
  const long long c1 = cta < n_cta ? cta_begin(cta + 1, T, n_cta) : 0;

  // ---- prefetch: the warp's first tiles (a tile holding this call's new token waits)
  // the segment whose new token is being appended (its first global tile), and the parity of
  // that append's phase of appbar (one phase per segment holding a group's last tile)
  long long app_gstart = -1;
  uint32_t app_parity = 0;
  Cursor* curs = reinterpret_cast<Cursor*>(smem + DecSmem::cursors) + warp;
  Cursor fc;
  int pg = -1;  // lane 0: block-table entry of the cursor's tile
  fc.done = c0 >= c1;
  if (!fc.done) {
    fc.s = segment_at(a, pre, B, Hkv, c0, c1);
    fc.i = fc.s.lo + warp;
    cursor_normalise(fc, a, pre, B, Hkv, c1, warp);
    // lanes 1.. request the block-table entries of the warp's next tiles now, so that the
    // dependent lookups of the first copies below find them in L1
    if (!fc.done && a.v.block_table && lane > 0 && lane < NSLOT) {
      const int t = TT * (fc.s.first + fc.i + lane * DEC_WARPS);
      if (fc.i + lane * DEC_WARPS < fc.s.hi && t < fc.s.ctx && t / a.v.page_size < a.v.max_pages)
        asm volatile("prefetch.global.L1 [%0];" ::"l"(a.v.block_table + (size_t)fc.s.b * a.v.max_pages + t / a.v.page_size));
    }
    pg = cursor_page(fc, a.v);
  }
  if (lane == 0) *curs = fc;
  __syncwarp();
  bool aborted = false;
  int k_fetch = 0, k_done = 0, k_wait = 0;  // tiles issued, tiles passed, slots waited for
  auto top_up = [&]() {
    if (aborted || k_fetch >= k_done + NSLOT) return;
    Cursor fc = *curs;
    if (fc.done) return;
    while (!fc.done && k_fetch < k_done + NSLOT) {
      const int ctx = fc.s.ctx;
      // a tile holding this call's new token is loaded only after this warp has appended it
      if (is_new_token_tile<FUSED>(fc.s, fc.i) &&
          (fc.s.gstart != app_gstart || !__shfl_sync(0xffffffffu, mbar_test_wait(appbar, app_parity), 0)))
        break;
      const int sl_i = k_fetch % NSLOT;
      if (lane == 0)
        issue_tile(a.v, fc.s.b, fc.s.kvh, fc.s.first + fc.i, ctx, fc.s.plo, pg, ring + sl_i * SLOT_BYTES, &valid[sl_i],
                   &wbar[sl_i],
                   SLOT_BYTES);
      ++k_fetch;
      fc.i += DEC_WARPS;
      cursor_normalise(fc, a, pre, B, Hkv, c1, warp);
      pg = cursor_page(fc, a.v);
    }
    __syncwarp();
    if (lane == 0) *curs = fc;
    __syncwarp();
  };
  top_up();
  // rotation parameters of the first segment's kv head into shared memory (they are not
  // written by the kernel this one may overlap)
  float* sprm = reinterpret_cast<float*>(smem + DecSmem::sparams);
  int sprm_kvh = -1;
  if (c0 < c1) {
    sprm_kvh = segment_at(a, pre, B, Hkv, c0, c1).kvh;
    if (threadIdx.x < params_per_head(a.v.rot) / 4)
      reinterpret_cast<float4*>(sprm)[threadIdx.x] =
          reinterpret_cast<const float4*>(a.params_layer + (size_t)sprm_kvh * params_per_head(a.v.rot))[threadIdx.x];
  }
  if (FUSED) {
    // warm L2 with the first segment's queries (a prefetch is only a hint: the rows are read
    // after the wait, so a value written meanwhile by the preceding kernel is the one used)
    if (c0 < c1 && threadIdx.x < a.g_real * 2) {
      const Seg s0 = segment_at(a, pre, B, Hkv, c0, c1);
      const size_t row = ((size_t)s0.b * a.n_q_heads + (size_t)s0.kvh * a.g_real + (threadIdx.x >> 1)) * D;
      const char* p = a.q_f32 ? (const char*)((const float*)a.q + row) : (const char*)((const __half*)a.q + row);
      asm volatile("prefetch.global.L2 [%0];" ::"l"(p + 128 * (threadIdx.x & 1) * (a.q_f32 ? 2 : 1)));
    }
    // and the new token (K and V rows, two lines each) of the groups whose last tile this CTA
    // holds: the segments of the run that end at their group's end (the first four)
    if (warp == 1) {
      long long x = c0;
      for (int n = 0; x < c1 && n < 4; ++n) {
        const Seg s = segment_at(a, pre, B, Hkv, x, c1);
        if (s.hi == s.ntiles && lane < 4) {
          const __half* src = ((lane & 2) ? a.v_new : a.k_new) + ((size_t)s.b * Hkv + s.kvh) * D;
          asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char*>(src) + 128 * (lane & 1)));
        }
        x = s.gstart + s.hi;
      }
    }
    // After an fp16 prefix's kernel (a.n_extra > 0) the wait moves to the final merge, the first
    // read of what that kernel writes (its partials): it starts only once it has waited for the
    // kernel before it, so q and the new token (read through L2) are already final.  The tile
    // work of this kernel then runs while the prefix's kernel is still running.
    if (a.n_extra == 0) pdl_wait();
  }

  // ---- outputs of groups with no tiles (empty context): zeros
  const int n_groups = B * Hkv;
  for (int gi = cta; gi < n_groups; gi += gridDim.x) {
    const int b = gi / Hkv, kvh = gi % Hkv;
    if (pre[b + 1] != pre[b]) continue;
    for (int idx = threadIdx.x; idx < a.g_real * (D / 4); idx += DEC_THREADS) {
      const int h = idx / (D / 4), c4 = idx % (D / 4);
      float4* dst = reinterpret_cast<float4*>(a.out + ((size_t)b * a.n_q_heads + (size_t)kvh * a.g_real + h) * D) + c4;
      *dst = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }

  // ---- segments of this CTA's run
  long long x = c0;
  while (x < c1) {
    const Seg seg = segment_at(a, pre, B, Hkv, x, c1);
    const int gid = seg.b * Hkv + seg.kvh;
    __syncthreads();  // previous segment's readers of qfrag / merge buffer are done
    if (seg.kvh != sprm_kvh) {
      sprm_kvh = seg.kvh;
      if (threadIdx.x < params_per_head(a.v.rot) / 4)
        reinterpret_cast<float4*>(sprm)[threadIdx.x] =
            reinterpret_cast<const float4*>(a.params_layer + (size_t)sprm_kvh * params_per_head(a.v.rot))[threadIdx.x];
      __syncthreads();
    }
    if (warp < (P4 ? 4 : HMAX))
      rotate_query<P4>(a, seg.b, seg.kvh, warp, sprm, qfrag, kappa);
    else if (P4 && warp < HMAX && lane == 0)
      kappa[warp] = 0.f;  // rows of lo terms: their lanes' scores are not used
    __syncthreads();
    // The new token is appended before the tile loops, K by the last warp and V by the one before
    // it: the round robin gives those warps the fewest tiles of the segment.  The warp whose tile
    // holds the token (normally its last tile) copies it only once both have arrived on appbar.
    if (FUSED && seg.hi == seg.ntiles) {
      if (warp >= DEC_WARPS - 2) {
        append_new_token<KB, VB>(a, seg.b, seg.kvh, seg.ctx, sprm, warp == DEC_WARPS - 1 ? 0 : 1);
        __syncwarp();
        fence_proxy_async_global();  // the appended records before the bulk reads of them
        if (lane == 0) mbar_arrive(appbar);
      }
      app_gstart = seg.gstart;
    }
    const float kap = kappa[lane >> 2];
    WarpState st;
    st.m = -CUDART_INF_F;
    st.l = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) st.acc[j][e] = 0.f;

    for (int i = seg.lo + warp; i < seg.hi; i += DEC_WARPS) {
      top_up();  // issues this tile if it is not in flight yet, and refills the ring
      if (FUSED && k_fetch == k_done && !aborted) {
        // not issued: the tile holds the new token, whose append is still running
        if (__all_sync(0xffffffffu, mbar_wait(appbar, app_parity, a.v.status))) {
          fence_proxy_async_global();
          top_up();
        } else {
          aborted = true;
        }
      }
      const int sl_i = k_done % NSLOT;
      if (!aborted) {
        const bool landed = __all_sync(0xffffffffu, mbar_wait(&wbar[sl_i], (k_done / NSLOT) & 1, a.v.status));
        if (landed) ++k_wait; else aborted = true;
      }
      if (!aborted)
        process_tile<P4, KB, VB>(ring + sl_i * SLOT_BYTES, valid[sl_i], qfrag + lane * QF_WORDS, kap,
                                 a.kc, st);
      ++k_done;
      __syncwarp();
    }

    // ---- merge the warps (shared memory, two rounds: warps w+4, w+8, ... into w, then
    // slots 0..3), then one partial per (CTA, group)
    if (P4) {  // add the lo columns (lanes t >= 2) into the hi columns of the same heads
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) st.acc[j][e] += __shfl_xor_sync(0xffffffffu, st.acc[j][e], 2);
    }
    float lq = st.l;
    lq += __shfl_xor_sync(0xffffffffu, lq, 1);
    lq += __shfl_xor_sync(0xffffffffu, lq, 2);
    if ((lane & 3) == 0) {
      sm[warp][lane >> 2] = st.m;
      sl[warp][lane >> 2] = lq;
    }
    {
      const int g = lane >> 2, t = lane & 3;
      if (warp >= 4) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          so[warp - 4][2 * t][16 * j + g] = st.acc[j][0];
          so[warp - 4][2 * t + 1][16 * j + g] = st.acc[j][1];
          so[warp - 4][2 * t][16 * j + g + 8] = st.acc[j][2];
          so[warp - 4][2 * t + 1][16 * j + g + 8] = st.acc[j][3];
        }
      }
      __syncthreads();
      if (warp < 4) {
        constexpr int NO = DEC_WARPS / 4 - 1;  // other warps merged into this one
        float f_self[2], f_oth[NO][2], Mh[2], Lh[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int hh = 2 * t + e;
          const float m0 = sm[warp][hh];
          float M = m0;
#pragma unroll
          for (int k = 0; k < NO; ++k) M = fmaxf(M, sm[warp + 4 * (k + 1)][hh]);
          f_self[e] = (m0 == -CUDART_INF_F) ? 0.f : fast_exp2(m0 - M);
          float L = sl[warp][hh] * f_self[e];
#pragma unroll
          for (int k = 0; k < NO; ++k) {
            const float mk = sm[warp + 4 * (k + 1)][hh];
            f_oth[k][e] = (mk == -CUDART_INF_F) ? 0.f : fast_exp2(mk - M);
            L = fmaf(sl[warp + 4 * (k + 1)][hh], f_oth[k][e], L);
          }
          Mh[e] = M;
          Lh[e] = L;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int hh = 2 * t + (e & 1), c = 16 * j + g + 8 * (e >> 1);
            float o = st.acc[j][e] * f_self[e & 1];
#pragma unroll
            for (int k = 0; k < NO; ++k) o = fmaf(so[warp + 4 * k][hh][c], f_oth[k][e & 1], o);
            so[warp][hh][c] = o;
          }
        }
        __syncwarp();
        if (g == 0) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            sm[warp][2 * t + e] = Mh[e];
            sl[warp][2 * t + e] = Lh[e];
          }
        }
      }
    }
    __syncthreads();
    const int c_first = cta_of(seg.gstart, T, n_cta);
    const int c_last = cta_of(seg.gstart + seg.ntiles - 1, T, n_cta);
    const int h = warp;
    if (h < a.g_real) {
      float M = -CUDART_INF_F;
#pragma unroll
      for (int w = 0; w < 4; ++w) M = fmaxf(M, sm[w][h]);
      float L = 0.f;
      float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float mw = sm[w][h];
        const float f = (mw == -CUDART_INF_F) ? 0.f : fast_exp2(mw - M);
        L = fmaf(sl[w][h], f, L);
        const float4 o = *reinterpret_cast<const float4*>(&so[w][h][4 * lane]);
        O.x = fmaf(o.x, f, O.x); O.y = fmaf(o.y, f, O.y); O.z = fmaf(o.z, f, O.z); O.w = fmaf(o.w, f, O.w);
      }
      const size_t slot = (size_t)cta + gid;
      reinterpret_cast<float4*>(a.ws.part_o + (slot * HMAX + h) * D)[lane] = O;
      if (lane == 0) a.ws.part_ml[slot * HMAX + h] = make_float2(M, L);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      // the barrier orders the CTA's partial stores before this release-ordered arrival (a
      // reduction: no value comes back, so nothing waits for the counter itself)
      asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&a.ws.counters[gid]) : "memory");
    }
    if (FUSED && seg.hi == seg.ntiles) app_parity ^= 1;  // that append's phase is over
    x = seg.gstart + seg.hi;
  }

  // ---- final merges: for every group of the run, the heads given to this CTA, once all of
  // the group's partials are in (every CTA has written all of its partials before waiting)
  if (FUSED && a.n_extra > 0) pdl_wait();  // the fp16 prefix's partials
  x = c0;
  while (x < c1) {
    const Seg seg = segment_at(a, pre, B, Hkv, x, c1);
    const int gid = seg.b * Hkv + seg.kvh;
    const int c_first = cta_of(seg.gstart, T, n_cta);
    const int n_parts = cta_of(seg.gstart + seg.ntiles - 1, T, n_cta) - c_first + 1;
    const int k = cta - c_first;
    uint32_t* done = a.ws.counters + n_groups;
    const int n_mergers = min(a.g_real, n_parts);
    if (k < a.g_real) {
      __syncthreads();
      // this kv head's rotation parameters, loaded while the partials come in
      if (threadIdx.x < params_per_head(a.v.rot) / 4)
        reinterpret_cast<float4*>(sprm)[threadIdx.x] =
            reinterpret_cast<const float4*>(a.params_layer + (size_t)seg.kvh * params_per_head(a.v.rot))[threadIdx.x];
      if (threadIdx.x == 0) {
        const uint64_t t0 = global_timer_ns();
        uint32_t seen;
        while ((int)(seen = ld_acquire(&a.ws.counters[gid])) < n_parts) {
          if (global_timer_ns() - t0 > 1000000000ull) {
            if (a.v.status) atomicOr(a.v.status, IQ_DEVERR_TIMEOUT);
            break;
          }
        }
        if ((int)seen > n_parts && a.v.status) atomicOr(a.v.status, IQ_DEVERR_WORKSPACE);  // counters not zeroed
      }
      // the group's mergers count themselves once they have seen every partial; the last
      // one clears both counters for the next call (nothing reads them again in this one).
      // The count is taken before the merge so that its round trip overlaps the merge.
      uint32_t seen_by = 0;
      if (threadIdx.x == 0) seen_by = atomicAdd(&done[gid], 1u);
      __syncthreads();
      merge_group(a, seg, gid, c_first, n_parts, k, reinterpret_cast<float*>(smem + DecSmem::so), sprm);
      if (threadIdx.x == 0 && (int)seen_by == n_mergers - 1) {
        a.ws.counters[gid] = 0;
        done[gid] = 0;
      }
    }
    x = seg.gstart + seg.hi;
  }

  // ---- leave no bulk copy in flight (only after a timed-out wait can one be pending)
  while (k_wait < k_fetch) {
    const int sl_i = k_wait % NSLOT;
    mbar_wait(&wbar[sl_i], (k_wait / NSLOT) & 1, nullptr);
    ++k_wait;
  }
}

// One decode launch for code widths (KB, VB); k_new / v_new select the fused step; def (or NULL)
// describes an fp16 prefix whose partials a preceding kernel has written.
template <int KB, int VB>
int launch_decode_kv(const LayerView& v, const void* q, int q_f32, int batch, int n_q_heads, const int32_t* ctx_len,
                     int max_ctx, const float* params_layer, float* out, void* workspace, const KernelConsts& kc,
                     void* stream, const void* k_new, const void* v_new, const DeferredInfo* def) {
  if (batch == 0 || n_q_heads == 0) return 0;
  DecArgs a;
  a.v = v;
  a.q = q;
  a.q_f32 = q_f32;
  a.n_q_heads = n_q_heads;
  a.g_real = n_q_heads / v.n_kv_heads;
  a.batch = batch;
  a.max_ctx = max_ctx;
  a.ctx_len = ctx_len;
  a.params_layer = params_layer;
  a.out = out;
  a.ws = carve_workspace(workspace, batch, v.n_kv_heads, def ? batch * v.n_kv_heads * def->n_extra : 0);
  a.pre_len = def ? def->len : nullptr;
  a.n_extra = def ? def->n_extra : 0;
  a.extra_base = def ? workspace_base_slots(batch, v.n_kv_heads) : 0;
  a.k_new = (const __half*)k_new;
  a.v_new = (const __half*)v_new;
  a.kc = kc;
  static std::once_flag attr_once;
  std::call_once(attr_once, [] {
    const int maxb = (int)DecSmem<KB, VB>::bytes(DECODE_MAX_BATCH);
    void (*ks[6])(DecArgs) = {decode_kernel<false, false, KB, VB>, decode_kernel<false, true, KB, VB>,
                              decode_kernel<true, false, KB, VB>,  decode_kernel<true, true, KB, VB>,
                              decode_kernel<true, false, KB, VB, 2>, decode_kernel<true, true, KB, VB, 2>};
    for (auto k : ks) {
      cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, maxb);
      cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    }
  });
  const bool fused = k_new != nullptr;
  // After an fp16 prefix's kernel: two ring slots per warp, so that a CTA fits on an SM beside
  // two of that kernel's CTAs and the two kernels overlap (the packed tail is short)
  auto kern = def ? (a.g_real <= 4 ? decode_kernel<true, true, KB, VB, 2> : decode_kernel<true, false, KB, VB, 2>)
              : fused ? (a.g_real <= 4 ? decode_kernel<true, true, KB, VB> : decode_kernel<true, false, KB, VB>)
                      : (a.g_real <= 4 ? decode_kernel<false, true, KB, VB> : decode_kernel<false, false, KB, VB>);
  const size_t smem = def ? DecSmem<KB, VB, 2>::bytes(batch) : DecSmem<KB, VB>::bytes(batch);
  const int ctas = decode_ctas(batch, v.n_kv_heads, max_ctx, resident_per_sm((const void*)kern, smem, DEC_THREADS));
  if (ctas == 0) return (int)cudaErrorInvalidConfiguration;
  return (int)launch_pdl(kern, dim3(ctas), dim3(DEC_THREADS), smem, (cudaStream_t)stream, a);
}

}  // namespace iq
