// Deferred quantisation: decode attention over a cache whose first tokens are still fp16.
//
// "RotorQuant" (sd114.wiki), section "2. 延迟量化策略", and "压缩与速度的博弈" (zhichai.net), section
// "延迟量化（Deferred Quantization）": during prompt processing the K/V cache stays fp16 (no
// rotation, no quantisation); tokens generated during decoding are quantised when they are
// inserted.  So a decode step attends over an fp16 prefix (positions 0 .. len-1 of each sequence,
// unrotated, as the model produced them) and the packed tail (positions len .. ctx-1, the new
// token appended and quantised by the same step).
//
// Two kernels per call.  prefix_kernel computes the attention of every query head of a kv head
// over a split of the fp16 prefix exactly (fp16 inputs, fp32 products and sums) on the tensor
// cores.  Each warp streams its own 32-token K and V tiles into shared memory with tensor-map
// bulk copies (two 64-coordinate boxes per tile and operand, 128-byte swizzle, so that ldmatrix
// reads are conflict-free; two tiles in flight) and takes S = Q K^T (m16n8k16 fp16, fp32
// accumulators; a q given in fp32 contributes a second, lo, binary16 term in rows 8-15), the
// online softmax of every head in the fragments, and O += P V with P as binary16 hi and lo rows.
// The warps' states are merged, the value sums are rotated forward (R) and scaled to the packed
// kernel's units, and written as extra split partials.  The fused decode step (decode_kernel)
// then appends the new token, attends over the packed tiles from the prefix's tile onward
// (positions below len masked) and merges its own partials with the extra ones before the single
// inverse rotation.  This kernel loads its first fp16 tiles while the kernel before it runs;
// the decode kernel does its tile work while this one runs.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <algorithm>
#include <mutex>

#include "iq_decode_impl.cuh"

namespace iq {

constexpr int PX_WARPS = 4;
constexpr int PX_THREADS = PX_WARPS * 32;
constexpr int PX_NB = 2;                   // tiles in flight per warp
constexpr int PX_BOX = TT * 128;           // one box: 32 rows x 64 coordinates (128 bytes, swizzled)
constexpr int PX_STAGE = 4 * PX_BOX;       // K coordinates 0-63, 64-127, then V likewise
constexpr int PX_SMEM = PX_WARPS * PX_NB * PX_STAGE + 1024;  // + alignment of the boxes to 1024 bytes

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

__device__ __forceinline__ void hmma16816(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                          uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// One box of a 2-D tensor map (coordinates x: elements, y: rows) into shared memory; completes on bar.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
// Byte offset of 16-byte chunk c of row r in a box written with the 128-byte swizzle.
__device__ __forceinline__ int swz(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }
__device__ __forceinline__ uint32_t pack_h2(float x, float y) {
  const __half2 h = __floats2half2_rn(x, y);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// One CTA per (sequence, kv head, split of the prefix); warp w takes tiles t_lo + w, t_lo + w + 4,
// ... of the split.  Fragment rows: g < 8 = head g (hi terms of q and of P), g + 8 = head g's lo
// terms.
__global__ void __launch_bounds__(PX_THREADS) prefix_kernel(PrefixArgs a, const __grid_constant__ CUtensorMap tmk,
                                                           const __grid_constant__ CUtensorMap tmv) {
  __shared__ __align__(16) __half sq[16][D + 8];  // query rows (hi, then lo) as binary16, padded
  __shared__ float sml[PX_WARPS][HMAX][2];
  __shared__ float sprm[256];
  __shared__ __align__(8) uint64_t bars[PX_WARPS][PX_NB];
  extern __shared__ __align__(128) uint8_t px_smem_raw[];  // [warp][stage][K lo, K hi, V lo, V hi boxes]
  uint8_t* const px_smem = px_smem_raw + ((1024 - (smem_u32(px_smem_raw) & 1023)) & 1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int G = a.g_real;
  const int gid = blockIdx.x / a.splits, split = blockIdx.x % a.splits;
  const int b = gid / a.n_kv_heads, kvh = gid % a.n_kv_heads;
  // prefix length, clamped as the decode kernel clamps it (0 <= len < ctx)
  int c = a.ctx_len[b];
  c = c < 0 ? 0 : (c > a.max_ctx ? a.max_ctx : c);
  int p = a.len[b];
  p = p < 0 ? 0 : ((c > 0 && p >= c) ? max(c - 1, 0) : p);
  const bool clamped = p > a.max_len;
  if (clamped) p = a.max_len;
  const int ntiles = (p + TT - 1) / TT;
  const int t_lo = (int)((long long)split * ntiles / a.splits), t_hi = (int)((long long)(split + 1) * ntiles / a.splits);
  const int n_mine = t_hi - t_lo > warp ? (t_hi - t_lo - warp + PX_WARPS - 1) / PX_WARPS : 0;  // this warp's tiles
  const size_t seq_base = ((size_t)b * a.n_kv_heads + kvh) * a.max_len;
  auto stage = [&](int st) { return px_smem + (size_t)(warp * PX_NB + st) * PX_STAGE; };

  if (lane == 0) {
    for (int i = 0; i < PX_NB; ++i) mbar_init(&bars[warp][i], 1);
    mbar_fence_init();
  }
  __syncwarp();
  // the warp's j-th tile into stage j % PX_NB: four boxes of 32 rows (rows past the prefix are
  // whatever the arrays hold there, or zeros past their end; they are cleared before use)
  auto issue = [&](int j) {
    const int tile = t_lo + warp + PX_WARPS * j, st = j % PX_NB;
    if (lane == 0) {
      mbar_arrive_expect_tx(&bars[warp][st], PX_STAGE);
      const int y = (int)(seq_base + (size_t)TT * tile);
      uint8_t* d = stage(st);
      tma_load_2d(d, &tmk, 0, y, &bars[warp][st]);
      tma_load_2d(d + PX_BOX, &tmk, 64, y, &bars[warp][st]);
      tma_load_2d(d + 2 * PX_BOX, &tmv, 0, y, &bars[warp][st]);
      tma_load_2d(d + 3 * PX_BOX, &tmv, 64, y, &bars[warp][st]);
    }
  };
  // The fp16 prefix (and len, ctx_len) is read before waiting for the preceding kernel; q and
  // every write come after.  The wait also comes before letting the decode kernel start, since
  // that kernel reads q and the new token (through L2) before its own wait.
  for (int j = 0; j < PX_NB && j < n_mine; ++j) issue(j);
  pdl_wait();
  pdl_launch_dependents();
  if (clamped && a.status && split == 0 && kvh == 0 && threadIdx.x == 0) atomicOr(a.status, IQ_DEVERR_CTX);

  // queries of the group as binary16 rows: hi in rows 0..7, the residual of an fp32 q in 8..15
  for (int i = threadIdx.x; i < HMAX * D; i += PX_THREADS) {
    const int hh = i / D, x = i % D;
    float val = 0.f;
    if (hh < G) {
      const size_t row = ((size_t)b * a.n_q_heads + (size_t)kvh * G + hh) * D + x;
      val = a.q_f32 ? ((const float*)a.q)[row] : __half2float(((const __half*)a.q)[row]);
    }
    const __half hi = __float2half_rn(val);
    sq[hh][x] = hi;
    sq[8 + hh][x] = __float2half_rn(val - __half2float(hi));
  }
  if (threadIdx.x < params_per_head(a.rot) / 4)
    reinterpret_cast<float4*>(sprm)[threadIdx.x] =
        reinterpret_cast<const float4*>(a.params_layer + (size_t)kvh * params_per_head(a.rot))[threadIdx.x];
  __syncthreads();
  uint32_t qa[D / 16][4];  // A fragments of Q for the eight k-steps of 16 coordinates
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    qa[ks][0] = *reinterpret_cast<const uint32_t*>(&sq[g][16 * ks + 2 * t]);
    qa[ks][1] = *reinterpret_cast<const uint32_t*>(&sq[g + 8][16 * ks + 2 * t]);
    qa[ks][2] = *reinterpret_cast<const uint32_t*>(&sq[g][16 * ks + 2 * t + 8]);
    qa[ks][3] = *reinterpret_cast<const uint32_t*>(&sq[g + 8][16 * ks + 2 * t + 8]);
  }
  const float qs = kLog2e * 0.08838834764831845f;  // scores in log2 units: log2(e) / sqrt(128)
  float m = -CUDART_INF_F, l = 0.f;  // head g: running max, this lane's share of the sum
  float o[D / 8][4];                 // O rows g (P hi) and g + 8 (P lo), coordinates 8 nt + 2 t (+1)
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
  bool ok = true;
  int j = 0;
  for (; j < n_mine; ++j) {
    const int tile = t_lo + warp + PX_WARPS * j, st = j % PX_NB;
    ok = __all_sync(0xffffffffu, mbar_wait(&bars[warp][st], (j / PX_NB) & 1, a.status));
    if (!ok) break;
    const int n_valid = min(TT, p - TT * tile);
    uint8_t* const kt = stage(st);
    uint8_t* const vt = kt + 2 * PX_BOX;
    if (n_valid < TT) {  // rows past the prefix: zeros (their P is 0, and 0 times a NaN is not)
      for (int i = lane; i < (TT - n_valid) * 32; i += 32) {
        const int row = n_valid + i / 32, part = i % 32;  // 4 boxes x 8 chunks
        *reinterpret_cast<uint4*>(kt + (part >> 3) * PX_BOX + row * 128 + 16 * (part & 7)) = make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
    }
    // scores: tokens 8 nt + 2 t (+1) of head g (rows g and g + 8 summed)
    float sc[TT / 8][4];
#pragma unroll
    for (int nt = 0; nt < TT / 8; ++nt) {
      sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
      for (int kp = 0; kp < D / 32; ++kp) {  // two k-steps per ldmatrix.x4: matrices = coordinates 32 kp + 8 i
        uint32_t b0, b1, b2, b3;
        const int cg = 4 * kp + (lane >> 3), tok = 8 * nt + (lane & 7);  // coordinate chunk, token
        ldsm_x4(smem_u32(kt + (cg >> 3) * PX_BOX + swz(tok, cg & 7)), b0, b1, b2, b3);
        hmma16816(sc[nt], qa[2 * kp][0], qa[2 * kp][1], qa[2 * kp][2], qa[2 * kp][3], b0, b1);
        hmma16816(sc[nt], qa[2 * kp + 1][0], qa[2 * kp + 1][1], qa[2 * kp + 1][2], qa[2 * kp + 1][3], b2, b3);
      }
    }
    float s[TT / 4], mx = -CUDART_INF_F;
#pragma unroll
    for (int nt = 0; nt < TT / 8; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int tok = 8 * nt + 2 * t + e;
        const float v = (sc[nt][e] + sc[nt][2 + e]) * qs;
        s[2 * nt + e] = tok < n_valid ? v : -CUDART_INF_F;
        mx = fmaxf(mx, s[2 * nt + e]);
      }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m, mx);
    if (__any_sync(0xffffffffu, m_new > m)) {
      const float r = (m == -CUDART_INF_F) ? 0.f : exp2f(m - m_new);
      l *= r;
#pragma unroll
      for (int nt = 0; nt < D / 8; ++nt) {
        o[nt][0] *= r; o[nt][1] *= r; o[nt][2] *= r; o[nt][3] *= r;
      }
      m = m_new;
    }
    // P as A fragments (k = tokens): rows g = binary16 hi, g + 8 = lo of head g
    uint32_t pa[TT / 16][4];
#pragma unroll
    for (int kk = 0; kk < TT / 16; ++kk)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {  // tokens 16 kk + 2 t (+1), then 16 kk + 8 + 2 t (+1)
        const int nt = 2 * kk + hf;
        const float p0 = (s[2 * nt] == -CUDART_INF_F) ? 0.f : exp2f(s[2 * nt] - m);
        const float p1 = (s[2 * nt + 1] == -CUDART_INF_F) ? 0.f : exp2f(s[2 * nt + 1] - m);
        l += p0 + p1;
        const uint32_t h = pack_h2(p0, p1);
        const float2 hf2 = __half22float2(*reinterpret_cast<const __half2*>(&h));
        pa[kk][2 * hf] = h;
        pa[kk][2 * hf + 1] = pack_h2(p0 - hf2.x, p1 - hf2.y);
      }
    // values: O += P V, coordinates as eight-wide n-tiles; V fragments by transposed ldmatrix
#pragma unroll
    for (int kk = 0; kk < TT / 16; ++kk)
#pragma unroll
      for (int np = 0; np < D / 16; ++np) {  // n-tiles 2 np, 2 np + 1
        uint32_t b0, b1, b2, b3;
        const int cg = 2 * np + (lane >> 4), tok = 16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1);
        ldsm_x4_t(smem_u32(vt + (cg >> 3) * PX_BOX + swz(tok, cg & 7)), b0, b1, b2, b3);
        hmma16816(o[2 * np], pa[kk][0], pa[kk][1], pa[kk][2], pa[kk][3], b0, b1);
        hmma16816(o[2 * np + 1], pa[kk][0], pa[kk][1], pa[kk][2], pa[kk][3], b2, b3);
      }
    __syncwarp();  // every lane is done with this stage
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // its reads before the next copies into it
    if (j + PX_NB < n_mine) issue(j + PX_NB);
  }
  // leave no bulk copy in flight (only after a timed-out wait can one be pending)
  if (!ok && lane == 0)
    for (int jj = j; jj < min(n_mine, j + PX_NB); ++jj) mbar_wait(&bars[warp][jj % PX_NB], (jj / PX_NB) & 1, nullptr);

  // ---- merge the warps per head (shared memory over the tile stages), then R and the partial
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);
  __syncthreads();
  float* so = reinterpret_cast<float*>(px_smem);  // [warp][head][128]
  if (t == 0) {
    sml[warp][g][0] = ok ? m : -CUDART_INF_F;
    sml[warp][g][1] = ok ? l : 0.f;
  }
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt) {  // head g: rows g (hi) + g + 8 (lo)
    so[(warp * HMAX + g) * D + 8 * nt + 2 * t] = o[nt][0] + o[nt][2];
    so[(warp * HMAX + g) * D + 8 * nt + 2 * t + 1] = o[nt][1] + o[nt][3];
  }
  __syncthreads();
  float Mp[4][4];
  variant_block_matrix(a.rot, sprm + lane * params_per_block(a.rot), Mp);
  const float unit = a.alpha_v * 11.313708498984761f;  // alpha_v * sqrt(128)
  for (int h = warp; h < G; h += PX_WARPS) {
    float M = -CUDART_INF_F;
    for (int w = 0; w < PX_WARPS; ++w) M = fmaxf(M, sml[w][h][0]);
    float L = 0.f, ov[4] = {0.f, 0.f, 0.f, 0.f};
    for (int w = 0; w < PX_WARPS; ++w) {
      const float mw = sml[w][h][0];
      if (mw == -CUDART_INF_F) continue;
      const float wt = exp2f(mw - M);
      L = fmaf(sml[w][h][1], wt, L);
      const float4 x = *reinterpret_cast<const float4*>(&so[(w * HMAX + h) * D + 4 * lane]);
      ov[0] = fmaf(x.x, wt, ov[0]); ov[1] = fmaf(x.y, wt, ov[1]); ov[2] = fmaf(x.z, wt, ov[2]); ov[3] = fmaf(x.w, wt, ov[3]);
    }
    // into the packed kernel's basis and units: R o, times alpha_v sqrt(128)
    warp_rotate_forward(ov, Mp, a.rot == ROT_ISO);
    const size_t slot = (size_t)a.extra_base + (size_t)gid * a.splits + split;
    reinterpret_cast<float4*>(a.part_o + (slot * HMAX + h) * D)[lane] =
        make_float4(ov[0] * unit, ov[1] * unit, ov[2] * unit, ov[3] * unit);
    if (lane == 0) a.part_ml[slot * HMAX + h] = make_float2(M, L);
  }
}

int prefix_splits(int batch, int n_kv_heads, int max_len, int n_sm) {
  const int groups = std::max(1, batch * n_kv_heads);
  int s = std::max(1, n_sm / groups);                                // at most one CTA per SM
  s = std::min(s, std::max(1, (max_len + TT - 1) / TT / PX_WARPS));  // every warp with a tile
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
  // 2-D views of the fp16 arrays: rows of 128 coordinates, boxes of 32 rows x 64 coordinates
  using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
  static EncodeFn encode = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaFuncSetAttribute(prefix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, PX_SMEM);
    // the whole unified memory as shared memory: an SM keeps the split it was given while it has
    // CTAs, and the decode CTA that follows must fit beside this one
    cudaFuncSetAttribute(prefix_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      encode = reinterpret_cast<EncodeFn>(fn);
  });
  if (!encode) return (int)cudaErrorNotSupported;
  const cuuint64_t rows = (cuuint64_t)batch * v.n_kv_heads * max_len;
  if (rows == 0 || rows > 0x7FFFFFFFull) return (int)cudaErrorInvalidValue;
  const cuuint64_t dims[2] = {(cuuint64_t)D, rows};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)TT}, estr[2] = {1, 1};
  CUtensorMap tmk, tmv;
  if (encode(&tmk, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(k16), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
      encode(&tmv, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(v16), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return (int)cudaErrorInvalidValue;
  return (int)launch_pdl(prefix_kernel, dim3(batch * v.n_kv_heads * splits), dim3(PX_THREADS), PX_SMEM,
                         (cudaStream_t)stream, a, tmk, tmv);
}

}  // namespace iq
