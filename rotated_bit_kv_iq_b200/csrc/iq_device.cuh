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

// The 4x4 matrix that the rotation variant `rot` applies to coordinates 4k..4k+3 after the WHT
// stages on bits 2..6 (ROT_ISO only), from the block's parameters p:
//   ROT_ISO    (qL, qR) at p[0..7]: the fused matrix above;
//   ROT_QUAT   q at p[0..3]: left multiplication y -> q * y (Hamilton product), q rescaled to unit;
//   ROT_PLANAR (c0, s0, c1, s1) at p[0..3]: Givens rotations of the pairs (4k, 4k+1) and
//              (4k+2, 4k+3), (y0, y1) -> (c y0 - s y1, s y0 + c y1), each (c, s) rescaled to unit.
__device__ __forceinline__ void variant_block_matrix(int rot, const float* p, float Mp[4][4]) {
  if (rot == ROT_ISO) {
    fused_block_matrix(p, Mp);
  } else if (rot == ROT_QUAT) {
    float a0 = p[0], a1 = p[1], a2 = p[2], a3 = p[3];
    const float na = 1.f / sqrtf(fmaf(a0, a0, fmaf(a1, a1, fmaf(a2, a2, a3 * a3))));
    a0 *= na; a1 *= na; a2 *= na; a3 *= na;
    Mp[0][0] = a0; Mp[0][1] = -a1; Mp[0][2] = -a2; Mp[0][3] = -a3;
    Mp[1][0] = a1; Mp[1][1] = a0;  Mp[1][2] = -a3; Mp[1][3] = a2;
    Mp[2][0] = a2; Mp[2][1] = a3;  Mp[2][2] = a0;  Mp[2][3] = -a1;
    Mp[3][0] = a3; Mp[3][1] = -a2; Mp[3][2] = a1;  Mp[3][3] = a0;
  } else {
    const float n0 = 1.f / sqrtf(fmaf(p[0], p[0], p[1] * p[1])), n1 = 1.f / sqrtf(fmaf(p[2], p[2], p[3] * p[3]));
    const float c0 = p[0] * n0, s0 = p[1] * n0, c1 = p[2] * n1, s1 = p[3] * n1;
    Mp[0][0] = c0; Mp[0][1] = -s0; Mp[0][2] = 0.f; Mp[0][3] = 0.f;
    Mp[1][0] = s0; Mp[1][1] = c0;  Mp[1][2] = 0.f; Mp[1][3] = 0.f;
    Mp[2][0] = 0.f; Mp[2][1] = 0.f; Mp[2][2] = c1; Mp[2][3] = -s1;
    Mp[3][0] = 0.f; Mp[3][1] = 0.f; Mp[3][2] = s1; Mp[3][3] = c1;
  }
}

// Parameters of block k of kv head `head` in a layer's parameter array.
__device__ __forceinline__ const float* block_params(const float* params_layer, int rot, int head, int k) {
  return params_layer + (size_t)head * params_per_head(rot) + k * params_per_block(rot);
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

__device__ __forceinline__ void warp_rotate_forward(float v[4], const float Mp[4][4], bool wht) {
  if (wht) warp_wht_bits2to6(v);
  float z[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) z[r] = Mp[r][0] * v[0] + Mp[r][1] * v[1] + Mp[r][2] * v[2] + Mp[r][3] * v[3];
#pragma unroll
  for (int r = 0; r < 4; ++r) v[r] = z[r];
}

__device__ __forceinline__ void warp_rotate_inverse(float v[4], const float Mp[4][4], bool wht) {
  float z[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) z[c] = Mp[0][c] * v[0] + Mp[1][c] * v[1] + Mp[2][c] * v[2] + Mp[3][c] * v[3];
#pragma unroll
  for (int c = 0; c < 4; ++c) v[c] = z[c];
  if (wht) warp_wht_bits2to6(v);
}

// ------------------------------------------------------------------ packed codes
// A chunk holds 32 codes (slots 0..31) in BITS little-endian words; its four selector words
// sel[w] (w = 0..3) hold slot 8w + j as nibble j, bits above the code clear:
//   BITS 3: W_w bits [4j,4j+3) = slot 8w+j, bit 4j+3 = bit w of slot 24+j (w < 3);
//   BITS 4: W_w = sel[w];
//   BITS 2: W_w bits [4j,4j+2) = slot 16w+j, bits [4j+2,4j+4) = slot 16w+8+j (w < 2).
template <int BITS>
__device__ __forceinline__ void chunk_selectors(const uint32_t* w, uint32_t sel[4]) {
  if constexpr (BITS == 3) {
    sel[0] = w[0] & 0x77777777u;
    sel[1] = w[1] & 0x77777777u;
    sel[2] = w[2] & 0x77777777u;
    sel[3] = ((w[0] >> 3) & 0x11111111u) | ((w[1] >> 2) & 0x22222222u) | ((w[2] >> 1) & 0x44444444u);
  } else if constexpr (BITS == 4) {
    sel[0] = w[0];
    sel[1] = w[1];
    sel[2] = w[2];
    sel[3] = w[3];
  } else {
    sel[0] = w[0] & 0x33333333u;
    sel[1] = (w[0] >> 2) & 0x33333333u;
    sel[2] = w[1] & 0x33333333u;
    sel[3] = (w[1] >> 2) & 0x33333333u;
  }
}

// Selector word w alone, reading only the storage words it depends on.
template <int BITS>
__device__ __forceinline__ uint32_t chunk_selector(const uint32_t* w, int sel) {
  if constexpr (BITS == 3) {
    if (sel < 3) return w[sel] & 0x77777777u;
    return ((w[0] >> 3) & 0x11111111u) | ((w[1] >> 2) & 0x22222222u) | ((w[2] >> 1) & 0x44444444u);
  } else if constexpr (BITS == 4) {
    return w[sel];
  } else {
    return (w[sel >> 1] >> (2 * (sel & 1))) & 0x33333333u;
  }
}

// Storage word k (k < BITS) of a chunk from its four selector words (the inverse of the
// above).  Every token's codes sit in whole nibbles of the selector words, and this map keeps
// nibble positions: a nibble of the selector words lands in the same nibble of storage words.
template <int BITS>
__device__ __forceinline__ uint32_t pack_word(int k, uint32_t s0, uint32_t s1, uint32_t s2, uint32_t s3) {
  if constexpr (BITS == 4) return k == 0 ? s0 : k == 1 ? s1 : k == 2 ? s2 : s3;
  if constexpr (BITS == 3) {
    const uint32_t s = k == 0 ? s0 : k == 1 ? s1 : s2;
    return s | (((s3 >> k) & 0x11111111u) << 3);
  }
  return k == 0 ? (s0 | (s1 << 2)) : (s2 | (s3 << 2));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Table lookup of four codes (nibbles 0..3 of s, bits above the code clear) into their int8
// centroid terms: byte i of the result = entry (nibble i) of the 2^BITS-entry table t (byte k of
// the little-endian words t[0..] = entry k).  2 and 3 bits: one byte permute; 4 bits: a permute
// in each half of the table and a byte select on the code's top bit.
template <int BITS>
__device__ __forceinline__ uint32_t lut4(const uint32_t* t, uint32_t s) {
  if constexpr (BITS == 2) return prmt(t[0], t[0], s);
  if constexpr (BITS == 3) return prmt(t[0], t[1], s);
  const uint32_t s7 = s & 0x7777u;
  const uint32_t m = prmt(0x0000FF00u, 0u, (s >> 3) & 0x1111u);  // byte i = 0xFF when code i >= 8
  const uint32_t a = prmt(t[0], t[1], s7), b = prmt(t[2], t[3], s7);
  return (a & ~m) | (b & m);
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
  return v.pool + (((size_t)page * v.n_kv_heads + head) * (v.page_size / TILE_TOKENS) + slot / TILE_TOKENS) *
                      (size_t)tile_bytes(v.kb, v.vb);
}
__device__ __forceinline__ uint8_t* k_record(const LayerView& v, int page, int head, int slot) {
  return tile_record(v, page, head, slot) + (slot % TILE_TOKENS) * k_rec_bytes(v.kb);
}
__device__ __forceinline__ uint8_t* v_block(const LayerView& v, int page, int head, int slot) {
  return tile_record(v, page, head, slot) + tr_v(v.kb) + ((slot % TILE_TOKENS) / V_BLK_TOKENS) * v_blk_bytes(v.vb);
}
__device__ __forceinline__ uint16_t* norm_slot(const LayerView& v, int page, int head, int slot, int side) {
  return reinterpret_cast<uint16_t*>(tile_record(v, page, head, slot) + (side ? tr_vn(v.kb, v.vb) : tr_kn(v.kb, v.vb))) +
         slot % TILE_TOKENS;
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
// Non-blocking test of the same (this thread's view).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
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
// code = #{ j : u > b_j } with u = sqrt(128) z / n, written with the positive thresholds
// t_j = b_j n / sqrt(128) (2^(BITS-1) - 1 of them; the middle boundary is 0): magnitude class
// m = #{ |z| > t_j }, code = 2^(BITS-1) + m for z > 0 and 2^(BITS-1) - 1 - m otherwise.
// (Exact ties |z| = t_j are within rounding of a boundary.)
template <int BITS>
__device__ __forceinline__ uint32_t quantise(float z, const float* t) {
  const float a = fabsf(z);
  uint32_t m = 0;
#pragma unroll
  for (int j = 0; j < (1 << (BITS - 1)) - 1; ++j) m += (uint32_t)(a > t[j]);
  constexpr uint32_t half = 1u << (BITS - 1);
  return z > 0.f ? half + m : half - 1u - m;
}

// Thresholds of one side scaled to a vector of norm n: t_j = b_j n / sqrt(128).
template <int BITS>
__device__ __forceinline__ void scaled_thresholds(const SideConsts& sc, float n, float* t) {
  const float s = n * 0.08838834764831845f;
#pragma unroll
  for (int j = 0; j < (1 << (BITS - 1)) - 1; ++j) t[j] = sc.bound_pos[j] * s;
}

// ------------------------------------------------------------------ one-warp vector encoder
// One warp encodes one fp16 vector (128 values at `src`) into the K (side 0, width KB) or V
// (side 1, width VB) record of kv head `head` at (page, slot); lane l owns coordinates
// 4l..4l+3 (one rotation block).  The WHT stages (ROT_ISO) run as shuffles; the lane's block
// matrix is passed in.  A V block gets only this token's bits (see below).
// raw: this lane's four fp16 coordinates 4 lane .. 4 lane + 3 (see warp_encode_vector).
template <int BITS>
__device__ __forceinline__ void warp_encode_loaded(const LayerView& v, uint2 raw, int head, int side, int page,
                                                   int slot, const float Mp[4][4], const SideConsts& sc) {
  const int lane = threadIdx.x & 31;
  const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
  const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
  float x[4] = {f0.x, f0.y, f1.x, f1.y};
  float ss = x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float n = sqrtf(ss);
  warp_rotate_forward(x, Mp, v.rot == ROT_ISO);
  float t[7];
  scaled_thresholds<BITS>(sc, n, t);
  const uint32_t c0 = quantise<BITS>(x[0], t), c1 = quantise<BITS>(x[1], t);
  const uint32_t c2 = quantise<BITS>(x[2], t), c3 = quantise<BITS>(x[3], t);
  if (side == 0) {
    // K chunk c = lanes 8c..8c+7; lane 8c + 2w + e holds nibbles 4e..4e+3 of selector word w.
    const uint32_t v16 = c0 | (c1 << 4) | (c2 << 8) | (c3 << 12);
    const uint32_t sw = v16 | (__shfl_xor_sync(0xffffffffu, v16, 1) << 16);  // selector word on even lanes
    uint32_t* rec = reinterpret_cast<uint32_t*>(k_record(v, page, head, slot));
    if constexpr (BITS == 3) {
      // storage word w = selector word w (lane 8c + 2w) with the spare bits of selector word 3
      const uint32_t spare = __shfl_sync(0xffffffffu, sw, (lane & ~7) | 6);
      const int w = (lane & 7) >> 1;
      if ((lane & 1) == 0 && w < 3) rec[3 * (lane >> 3) + w] = sw | (((spare >> w) & 0x11111111u) << 3);
    } else {
      const int base = lane & ~7;
      const uint32_t s0 = __shfl_sync(0xffffffffu, sw, base), s1 = __shfl_sync(0xffffffffu, sw, base + 2);
      const uint32_t s2 = __shfl_sync(0xffffffffu, sw, base + 4), s3 = __shfl_sync(0xffffffffu, sw, base + 6);
      const int k = lane & 7;
      if (k < BITS) rec[BITS * (lane >> 3) + k] = pack_word<BITS>(k, s0, s1, s2, s3);
    }
  } else {
    // V block: this token (u = slot mod 16) owns nibbles j and j+4 of the selector words of
    // the 16 chunks (g, tq, h), tq = (u mod 8) / 2, j = 2 (u / 8) + (u mod 2): nibble j of
    // selector word w holds coordinate 32w + g + 8h and nibble j+4 coordinate 32w + 16 + g + 8h.
    // Lane l writes the token's storage words r = l, l + 32 (r < 16 BITS) of its (g, h, word)
    // list; the other tokens' bits are kept (atomic and/or: tokens of one block may be
    // appended by several warps of one launch).
    const uint32_t mine = c0 | (c1 << 8) | (c2 << 16) | (c3 << 24);
    const int u = slot & 15, tq = (u & 7) >> 1, j = 2 * (u >> 3) + (u & 1);
    uint8_t* blk = v_block(v, page, head, slot);
    auto code_at = [&](int x) { return (__shfl_sync(0xffffffffu, mine, x >> 2) >> (8 * (x & 3))) & 0xFu; };
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int kk = lane + 32 * r;
      const int k = kk < 16 * BITS ? kk : 0;
      const int gh = k / BITS, w = k % BITS;
      const int x = (gh >> 1) + 8 * (gh & 1);  // g + 8h
      // the token's nibbles j (n0) and j+4 (n1) of storage word w, from the codes they hold
      uint32_t n0, n1;
      if constexpr (BITS == 4) {
        n0 = code_at(32 * w + x);
        n1 = code_at(32 * w + 16 + x);
      } else if constexpr (BITS == 3) {
        n0 = code_at(32 * w + x) | (((code_at(96 + x) >> w) & 1u) << 3);
        n1 = code_at(32 * w + 16 + x) | (((code_at(112 + x) >> w) & 1u) << 3);
      } else {
        n0 = code_at(64 * w + x) | (code_at(64 * w + 32 + x) << 2);
        n1 = code_at(64 * w + 16 + x) | (code_at(64 * w + 48 + x) << 2);
      }
      if (kk < 16 * BITS) {
        const uint32_t bits = (n0 << (4 * j)) | (n1 << (4 * (j + 4)));
        const uint32_t mask = (0xFu << (4 * j)) | (0xFu << (4 * (j + 4)));
        unsigned int* word =
            reinterpret_cast<unsigned int*>(blk + chunk_bytes(BITS) * (2 * (4 * (gh >> 1) + tq) + (gh & 1)) + 4 * w);
        atomicAnd(word, ~mask);
        atomicOr(word, bits);
      }
    }
  }
  if (lane == 0) *norm_slot(v, page, head, slot, side) = __half_as_ushort(__float2half_rn(fminf(n, 65504.f)));
}
template <int BITS>
__device__ __forceinline__ void warp_encode_vector(const LayerView& v, const __half* __restrict__ src, int head,
                                                   int side, int page, int slot, const float Mp[4][4],
                                                   const SideConsts& sc) {
  const uint2 raw = __ldcg(reinterpret_cast<const uint2*>(src + 4 * (threadIdx.x & 31)));
  warp_encode_loaded<BITS>(v, raw, head, side, page, slot, Mp, sc);
}

}  // namespace iq
