// Device helpers for libiq kernels (sm_100a).
#pragma once
#include <cuda_fp16.h>
#include <cstdint>

#include "iq_internal.h"

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

// Look up the 4 codes in the low 16 bits of `sel`: returns low and high bytes of the
// binary16 levels in byte order of the nibbles.
__device__ __forceinline__ void lut4(uint32_t sel, const uint32_t lo[2], const uint32_t hi[2], uint32_t& l4,
                                     uint32_t& h4) {
  l4 = prmt(lo[0], lo[1], sel);
  h4 = prmt(hi[0], hi[1], sel);
}
// fp16x2 of (nibble0, nibble1) / (nibble2, nibble3): pairs along a K record.
__device__ __forceinline__ uint32_t pair01(uint32_t l4, uint32_t h4) { return prmt(l4, h4, 0x5140u); }
__device__ __forceinline__ uint32_t pair23(uint32_t l4, uint32_t h4) { return prmt(l4, h4, 0x7362u); }
// fp16x2 of (nibble0, nibble2) / (nibble1, nibble3): pairs across the two tokens of a V record.
__device__ __forceinline__ uint32_t pair02(uint32_t l4, uint32_t h4) { return prmt(l4, h4, 0x6240u); }
__device__ __forceinline__ uint32_t pair13(uint32_t l4, uint32_t h4) { return prmt(l4, h4, 0x7351u); }

// ------------------------------------------------------------------ tensor core (mma.sync)
__device__ __forceinline__ void mma16816(float c[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float half_bits_to_float(uint16_t h) { return __half2float(__ushort_as_half(h)); }

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
