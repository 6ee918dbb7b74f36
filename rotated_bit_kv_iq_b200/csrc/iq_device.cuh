// Device helpers for libiq kernels (sm_100a).
#pragma once
#include <cuda_fp16.h>
#include <cstdint>

#include "iq_internal.h"

#include <cuda_runtime.h>
#include <utility>

namespace iq {
// Launch with programmatic stream serialization (the kernel may start while the previous
// kernel in the stream finishes; it synchronises with griddepcontrol.wait).
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
}  // namespace iq

namespace iq {

// ------------------------------------------------------------------ rotation blocks
// Block k of S maps y (a quaternion (w,x,y,z) = coordinates 4k..4k+3) to qL * y * conj(qR).
// Left multiplication by a and right multiplication by b as 4x4 matrices (Hamilton
// product), then M = L(qL) R(conj(qR)).  Both quaternions are rescaled to unit length.
__device__ __forceinline__ void block_matrix(const float* qL_in, const float* qR_in, float M[4][4]) {
  float a[4], b[4];
  float na = 0.f, nb = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a[i] = qL_in[i];
    b[i] = qR_in[i];
    na = fmaf(a[i], a[i], na);
    nb = fmaf(b[i], b[i], nb);
  }
  na = 1.f / sqrtf(na);
  nb = 1.f / sqrtf(nb);
  a[0] *= na; a[1] *= na; a[2] *= na; a[3] *= na;
  b[0] *= nb; b[1] = -b[1] * nb; b[2] = -b[2] * nb; b[3] = -b[3] * nb;  // conj(qR)
  const float L[4][4] = {{a[0], -a[1], -a[2], -a[3]},
                         {a[1], a[0], -a[3], a[2]},
                         {a[2], a[3], a[0], -a[1]},
                         {a[3], -a[2], a[1], a[0]}};
  const float R[4][4] = {{b[0], -b[1], -b[2], -b[3]},
                         {b[1], b[0], b[3], -b[2]},
                         {b[2], -b[3], b[0], b[1]},
                         {b[3], b[2], -b[1], b[0]}};
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) M[r][c] = L[r][0] * R[0][c] + L[r][1] * R[1][c] + L[r][2] * R[2][c] + L[r][3] * R[3][c];
}

// Block matrix with the two lowest WHT stages and the 1/sqrt(128) scale folded in:
// M' = M * H4 / sqrt(128), H4[i][j] = (-1)^popcount(i&j).  Applying the WHT stages on
// coordinate bits 2..6 and then M' per block gives S * H * x / sqrt(128) = R x.
__device__ __forceinline__ void fused_block_matrix(const float* q, float Mp[4][4]) {
  float M[4][4];
  block_matrix(q, q + 4, M);
  const float s = 0.08838834764831845f;  // 1/sqrt(128)
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const float m0 = M[r][0], m1 = M[r][1], m2 = M[r][2], m3 = M[r][3];
    Mp[r][0] = (m0 + m1 + m2 + m3) * s;
    Mp[r][1] = (m0 - m1 + m2 - m3) * s;
    Mp[r][2] = (m0 + m1 - m2 - m3) * s;
    Mp[r][3] = (m0 - m1 - m2 + m3) * s;
  }
}

// ------------------------------------------------------------------ warp rotation
// One warp rotates one 128-vector: lane l holds coordinates 4l..4l+3.  Forward: WHT
// stages on coordinate bits 2..6 (lane bits 0..4) by shuffles, then M'_l.  Inverse:
// M'_l^T, then the same stages (H is symmetric and its stages commute).
__device__ __forceinline__ void warp_wht_bits2to6(float v[4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int b = 0; b < 5; ++b) {
    const bool upper = (lane >> b) & 1;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, v[i], 1 << b);
      v[i] = upper ? (o - v[i]) : (v[i] + o);
    }
  }
}

__device__ __forceinline__ void warp_rotate_forward(float v[4], const float Mp[4][4]) {
  warp_wht_bits2to6(v);
  float z[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) z[r] = Mp[r][0] * v[0] + Mp[r][1] * v[1] + Mp[r][2] * v[2] + Mp[r][3] * v[3];
#pragma unroll
  for (int r = 0; r < 4; ++r) v[r] = z[r];
}

__device__ __forceinline__ void warp_rotate_inverse(float v[4], const float Mp[4][4]) {
  float z[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) z[c] = Mp[0][c] * v[0] + Mp[1][c] * v[1] + Mp[2][c] * v[2] + Mp[3][c] * v[3];
#pragma unroll
  for (int c = 0; c < 4; ++c) v[c] = z[c];
  warp_wht_bits2to6(v);
}

// ------------------------------------------------------------------ packed codes
// 32-code chunk: W_w bits [4j,4j+3) = slot 8w+j, bit 4j+3 = bit w of slot 24+j.
// Selector words for byte-permute lookups: sel[w] (w<3) holds slots 8w..8w+7 as clean
// nibbles, sel[3] holds slots 24..31.
__device__ __forceinline__ void chunk_selectors(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t sel[4]) {
  sel[0] = w0 & 0x77777777u;
  sel[1] = w1 & 0x77777777u;
  sel[2] = w2 & 0x77777777u;
  sel[3] = ((w0 >> 3) & 0x11111111u) | ((w1 >> 2) & 0x22222222u) | ((w2 >> 1) & 0x44444444u);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Packed fp32 pairs (add/sub/mul/fma .f32x2: two IEEE fp32 operations per instruction, each
// rounded exactly as its scalar form).
__device__ __forceinline__ uint64_t f2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2s(uint64_t r, float& a, float& b) { asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r)); }
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// ------------------------------------------------------------------ tensor core (mma.sync, int8)
// D = A B + C with A 16x32 (row), B 32x8 (col), s8 inputs, s32 accumulators.
// Fragments (lane = 4 g + t): a0 = A[g][4t..4t+3], a1 = A[g+8][4t..], a2 = A[g][16+4t..],
// a3 = A[g+8][16+4t..]; b0 = B[4t..4t+3][g], b1 = B[16+4t..][g]; d0,d1 = D[g][2t,2t+1],
// d2,d3 = D[g+8][2t,2t+1] (byte i of a register = element i of its run of four).
__device__ __forceinline__ void imma16832(int d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                          uint32_t b1, int c0, int c1, int c2, int c3) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(c0), "r"(c1), "r"(c2), "r"(c3));
}

// Accumulators start at the bit pattern of 1.5 * 2^23: while |sum| < 2^22 the s32 result,
// read as a float, is exactly 1.5 * 2^23 + sum, so one float subtraction converts it.
constexpr int kMagicI = 0x4B400000;
constexpr float kMagicF = 12582912.0f;
__device__ __forceinline__ float magic_to_float(int x) { return __int_as_float(x) - kMagicF; }

// Round-to-nearest integer of |x| < 2^22 placed in the low bits of the result word
// (two's complement): the low byte is the int8 value.
__device__ __forceinline__ uint32_t round_low_bits(float x) { return (uint32_t)__float_as_int(x + kMagicF); }

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float half_bits_to_float(uint16_t h) { return __half2float(__ushort_as_half(h)); }

// Tile record holding `slot` of (page, kv head), and the pieces of one slot inside it.
__device__ __forceinline__ uint8_t* tile_record(const LayerView& v, int page, int head, int slot) {
  return v.pool + (((size_t)page * v.n_kv_heads + head) * (v.page_size / TILE_TOKENS) + slot / TILE_TOKENS) * TILE_BYTES;
}
__device__ __forceinline__ uint8_t* k_record(const LayerView& v, int page, int head, int slot) {
  return tile_record(v, page, head, slot) + TR_K + (slot % TILE_TOKENS) * K_REC;
}
__device__ __forceinline__ uint8_t* v_block(const LayerView& v, int page, int head, int slot) {
  return tile_record(v, page, head, slot) + TR_V + ((slot % TILE_TOKENS) / V_BLK_TOKENS) * V_BLK;
}
__device__ __forceinline__ uint16_t* norm_slot(const LayerView& v, int page, int head, int slot, int side) {
  return reinterpret_cast<uint16_t*>(tile_record(v, page, head, slot) + (side ? TR_VN : TR_KN)) + slot % TILE_TOKENS;
}

// Resolve the page of token `pos` of sequence `b`; returns -1 (and flags) when invalid.
__device__ __forceinline__ int resolve_page(const LayerView& v, int b, int pos) {
  int page;
  if (v.block_table) {
    const int idx = pos / v.page_size;
    if (pos < 0 || idx >= v.max_pages) {
      if (v.status) atomicOr(v.status, IQ_DEVERR_POSITION);
      return -1;
    }
    page = v.block_table[(size_t)b * v.max_pages + idx];
  } else {
    if (pos < 0 || pos >= v.page_size) {
      if (v.status) atomicOr(v.status, IQ_DEVERR_POSITION);
      return -1;
    }
    page = b;
  }
  if (page < 0 || page >= v.n_pages) {
    if (v.status) atomicOr(v.status, IQ_DEVERR_PAGE);
    return -1;
  }
  return page;
}

}  // namespace iq

namespace iq {

// ------------------------------------------------------------------ mbarrier / bulk copy
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Wait for the phase of the given parity to complete, for at most ~1 s; on timeout flag
// IQ_DEVERR_TIMEOUT and return false (the caller stops using the guarded data).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > 1000000000ull) {
      if (status) atomicOr(status, IQ_DEVERR_TIMEOUT);
      return false;
    }
  }
  return true;
}
// One bulk copy global -> this CTA's own shared memory; completes on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void named_barrier_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

}  // namespace iq

namespace iq {

// ------------------------------------------------------------------ programmatic dependent launch
// Every kernel lets the next kernel in the stream launch at once; it waits for the previous
// kernel (griddepcontrol.wait) before reading data that kernel may have written or writing
// anything.  Both are no-ops for kernels launched without the attribute.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Orders this thread's view of generic-proxy global writes before later async-proxy
// (bulk copy) reads.
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// ------------------------------------------------------------------ quantiser
// code = #{ j : u > b_j } with u = sqrt(128) z / n, written with the three positive
// thresholds t_j = b_j n / sqrt(128): magnitude class m = #{ |z| > t_j }, code = 4+m for
// z > 0 and 3-m otherwise.  (Exact ties |z| = t_j are within rounding of a boundary.)
__device__ __forceinline__ uint32_t quantise(float z, float t1, float t2, float t3) {
  const float a = fabsf(z);
  const uint32_t m = (uint32_t)(a > t1) + (uint32_t)(a > t2) + (uint32_t)(a > t3);
  return z > 0.f ? 4u + m : 3u - m;
}

// ------------------------------------------------------------------ one-warp vector encoder
// One warp encodes one fp16 vector (128 values at `src`) into the K (side 0) or V (side 1)
// record of kv head `head` at (page, slot); lane l owns coordinates 4l..4l+3 (one SO(4)
// block).  WHT stages on coordinate bits 2..6 run as shuffles; the lane's fused block matrix
// is passed in.  K words are assembled with two shuffles; a V block gets only this token's
// bits (see below).
__device__ __forceinline__ void warp_encode_vector(const LayerView& v, const __half* __restrict__ src, int head,
                                                   int side, int page, int slot, const float Mp[4][4],
                                                   const KernelConsts& kc) {
  const int lane = threadIdx.x & 31;
  const uint2 raw = *reinterpret_cast<const uint2*>(src + 4 * lane);
  const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
  const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
  float x[4] = {f0.x, f0.y, f1.x, f1.y};
  float ss = x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float n = sqrtf(ss);
  warp_rotate_forward(x, Mp);
  const float sc = n * 0.08838834764831845f;
  const float t1 = kc.bound_pos[0] * sc, t2 = kc.bound_pos[1] * sc, t3 = kc.bound_pos[2] * sc;
  const uint32_t c0 = quantise(x[0], t1, t2, t3), c1 = quantise(x[1], t1, t2, t3);
  const uint32_t c2 = quantise(x[2], t1, t2, t3), c3 = quantise(x[3], t1, t2, t3);
  if (side == 0) {
    // K chunk c = lanes 8c..8c+7; word w = lanes 8c+2w (low half) and 8c+2w+1 (high half);
    // spare slots 24..31 = lanes 8c+6, 8c+7.
    const uint32_t v16 = c0 | (c1 << 4) | (c2 << 8) | (c3 << 12);
    const uint32_t pair = v16 | (__shfl_xor_sync(0xffffffffu, v16, 1) << 16);
    const uint32_t spare = __shfl_sync(0xffffffffu, pair, (lane & ~7) | 6);
    const int w = (lane & 7) >> 1;
    if ((lane & 1) == 0 && w < 3) {
      const uint32_t word = pair | (((spare >> w) & 0x11111111u) << 3);
      uint32_t* rec = reinterpret_cast<uint32_t*>(k_record(v, page, head, slot));
      rec[3 * (lane >> 3) + w] = word;
    }
  } else {
    // V block: this token (u = slot mod 16) owns nibbles j and j+4 of the three words of the
    // chunks (g, tq, h) with tq = (u mod 8) / 2, j = 2 (u / 8) + (u mod 2).  Word w of chunk
    // (g, tq, h) takes codes of coordinates 32w + g + 8h (nibble j) and 32w + 16 + g + 8h
    // (nibble j+4), and bit w of the codes of coordinates 96 + g + 8h and 112 + g + 8h as
    // the spare bits.  Lane l writes words k = l and l + 32 (k < 48) of the token's
    // (g, h, w) list; the other tokens' bits are kept (atomic and/or: tokens of one block may
    // be appended by several warps of one launch).
    const uint32_t mine = c0 | (c1 << 8) | (c2 << 16) | (c3 << 24);
    const int u = slot & 15, tq = (u & 7) >> 1, j = 2 * (u >> 3) + (u & 1);
    uint8_t* blk = v_block(v, page, head, slot);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int k = lane + 32 * r;
      const int kk = k < 48 ? k : 0;
      const int gh = kk / 3, w = kk % 3;
      const int g = gh >> 1, h = gh & 1;
      const int x0 = 32 * w + g + 8 * h, x1 = x0 + 16, x2 = 96 + g + 8 * h, x3 = x2 + 16;
      const uint32_t y0 = (__shfl_sync(0xffffffffu, mine, x0 >> 2) >> (8 * (x0 & 3))) & 7u;
      const uint32_t y1 = (__shfl_sync(0xffffffffu, mine, x1 >> 2) >> (8 * (x1 & 3))) & 7u;
      const uint32_t y2 = (__shfl_sync(0xffffffffu, mine, x2 >> 2) >> (8 * (x2 & 3))) & 7u;
      const uint32_t y3 = (__shfl_sync(0xffffffffu, mine, x3 >> 2) >> (8 * (x3 & 3))) & 7u;
      if (k < 48) {
        const uint32_t n0 = y0 | (((y2 >> w) & 1u) << 3), n1 = y1 | (((y3 >> w) & 1u) << 3);
        const uint32_t bits = (n0 << (4 * j)) | (n1 << (16 + 4 * j));
        const uint32_t mask = (0xFu << (4 * j)) | (0xFu << (16 + 4 * j));
        unsigned int* word = reinterpret_cast<unsigned int*>(blk + 12 * (2 * (4 * g + tq) + h) + 4 * w);
        atomicAnd(word, ~mask);
        atomicOr(word, bits);
      }
    }
  }
  if (lane == 0) *norm_slot(v, page, head, slot, side) = __half_as_ushort(__float2half_rn(fminf(n, 65504.f)));
}

}  // namespace iq
