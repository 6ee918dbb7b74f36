// Quantise-and-append kernel: fp16 K/V vectors -> packed 3-bit records + binary16 norms.
//
// Steps per vector follow "RotaryQuant" (rebasdaily.com, section "妙处不只是压缩，而是不再展开")
// and its abstract (arXiv 2608.08081): Walsh-Hadamard mixing, then the block SO(4)
// rotation, then scalar quantisation; the quantiser is the Lloyd-Max codebook of N(0,1/d)
// ("压缩与速度的博弈" zhichai.net, sections "Beta 分布的魔力", "Lloyd-Max 最优量化").
//
// Mapping: one thread encodes one 128-vector entirely in registers (all seven butterfly
// stages are register-local, no shuffles).  A CTA covers 128 consecutive positions of one
// (sequence, kv head, K|V); the head's 32 block matrices live in shared memory and every
// lane of a warp reads the same one at the same time (broadcast).  Instead of normalising
// the vector, the rotated coordinates z = R x are compared with the boundaries scaled by
// ||x||/sqrt(128).  The code width (2, 3 or 4 bits, "压缩与速度的博弈" section "K 和 V 的非对称需求")
// is a template parameter; the rotation variant (WHT + quaternion pairs, one quaternion per
// block, Givens pairs: section "三种变体") is read from the layer view.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "iq_device.cuh"

namespace iq {

constexpr int ENC_THREADS = 128;

// Encodes the vectors of the sides side0 .. side0 + n_sides - 1 (0 = K, 1 = V), all of width BITS
// (so one set of codebook constants, sc, serves every side of the launch);
// WHT: the layer's rotation is ROT_ISO (WHT stages, then the fused quaternion-pair blocks); else
// the variant's blocks alone.  (A compile-time choice: a run-time branch around the unrolled
// stages cost the kernel a quarter more registers.)
template <int BITS, bool WHT>
__global__ void __launch_bounds__(ENC_THREADS)
encode_kernel(LayerView v, const __half* __restrict__ k_src, const __half* __restrict__ v_src, int n_new,
              const int32_t* __restrict__ start_pos, const float* __restrict__ params_layer, SideConsts sc,
              int side0, int n_sides) {
  // block matrices M'_k as column pairs: smat[k][c][0] = (M'[0][c], M'[1][c]),
  // smat[k][c][1] = (M'[2][c], M'[3][c])
  __shared__ uint64_t smat[NBLK][4][2];
  pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.z;
  const int head = blockIdx.y / n_sides;
  const int side = side0 + blockIdx.y % n_sides;  // 0 = K, 1 = V
  const __half* src = side ? v_src : k_src;
  if (src == nullptr) return;

  if (threadIdx.x < NBLK) {
    float Mp[4][4];
    variant_block_matrix(v.rot, block_params(params_layer, v.rot, head, threadIdx.x), Mp);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      smat[threadIdx.x][c][0] = f2(Mp[0][c], Mp[1][c]);
      smat[threadIdx.x][c][1] = f2(Mp[2][c], Mp[3][c]);
    }
  }
  __syncthreads();

  const int start = start_pos[b];
  const int pos = (start & ~15) + blockIdx.x * ENC_THREADS + threadIdx.x;  // V-block-aligned lanes
  const int i_new = pos - start;
  const bool in_range = (i_new >= 0) && (i_new < n_new);
  // All lanes of a warp take part in the V-block exchange below, so inactive lanes run
  // the arithmetic on zeros and skip only the loads and stores.
  int page = -1;
  if (in_range) page = resolve_page(v, b, pos);
  const bool active = in_range && page >= 0;

  uint64_t y[D / 2];  // coordinate pairs (2i, 2i+1)
  if (active) {
    const uint4* p = reinterpret_cast<const uint4*>(src + (((size_t)b * n_new + i_new) * v.n_kv_heads + head) * D);
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      uint4 w = __ldg(p + q);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ws[e]));
        y[4 * q + e] = f2(f.x, f.y);
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < D / 2; ++i) y[i] = 0ull;
  }

  // ||x||^2 in fp32 (even and odd coordinates summed separately, then added)
  uint64_t ss = 0ull;
#pragma unroll
  for (int i = 0; i < D / 2; ++i) ss = fma2(y[i], y[i], ss);
  float ss0, ss1;
  f2s(ss, ss0, ss1);
  const float n = sqrtf(ss0 + ss1);

  if (WHT) {
    // Butterfly stages on coordinate bits 2..6 (bits 0,1 are inside M'), two butterflies per
    // packed instruction.
#pragma unroll
    for (int bit = 2; bit < 7; ++bit) {
      const int h = 1 << (bit - 1);  // in pairs
#pragma unroll
      for (int i = 0; i < D / 2; ++i) {
        if ((i & h) == 0) {
          const uint64_t a = y[i], c = y[i + h];
          y[i] = add2(a, c);
          y[i + h] = sub2(a, c);
        }
      }
    }
  }
  // Block matrices: rows (0,1) and (2,3) as pairs, z = M' v.
#pragma unroll
  for (int k = 0; k < NBLK; ++k) {
    float v0, v1, v2, v3;
    f2s(y[2 * k], v0, v1);
    f2s(y[2 * k + 1], v2, v3);
    const uint64_t b0 = f2(v0, v0), b1 = f2(v1, v1), b2 = f2(v2, v2), b3 = f2(v3, v3);
    uint64_t z01 = mul2(smat[k][3][0], b3), z23 = mul2(smat[k][3][1], b3);
    z01 = fma2(smat[k][2][0], b2, z01);
    z23 = fma2(smat[k][2][1], b2, z23);
    z01 = fma2(smat[k][1][0], b1, z01);
    z23 = fma2(smat[k][1][1], b1, z23);
    y[2 * k] = fma2(smat[k][0][0], b0, z01);
    y[2 * k + 1] = fma2(smat[k][0][1], b0, z23);
  }

  float t[7];
  scaled_thresholds<BITS>(sc, n, t);
  // codes once: cw[r] holds coordinates 8r..8r+7 as nibbles (bits above the code clear)
  uint32_t cw[16];
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    uint32_t w = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float za, zb;
      f2s(y[4 * r + e], za, zb);
      w |= quantise<BITS>(za, t) << (8 * e);
      w |= quantise<BITS>(zb, t) << (8 * e + 4);
    }
    cw[r] = w;
  }

  const int slot = pos % v.page_size;
  if (side == 0) {
    // K record: chunk c has selector words cw[4c..4c+3] (slot 8w + j = coordinate 32c + 8w + j).
    if (active) {
      uint32_t rec[4 * BITS];
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int k = 0; k < BITS; ++k)
          rec[BITS * c + k] = pack_word<BITS>(k, cw[4 * c], cw[4 * c + 1], cw[4 * c + 2], cw[4 * c + 3]);
      uint4* dst = reinterpret_cast<uint4*>(k_record(v, page, head, slot));
#pragma unroll
      for (int i = 0; i < BITS; ++i) dst[i] = make_uint4(rec[4 * i], rec[4 * i + 1], rec[4 * i + 2], rec[4 * i + 3]);
    }
  } else {
    // V block (16 tokens = 16 consecutive lanes).  Chunk (g, tq, h) holds the codes of the
    // quad of tokens u with (u mod 8)/2 = tq (lanes u, u^1, u^8, u^9; token u is quad member
    // m = 2 (u/8) + (u mod 2)): nibble m of selector word w = coordinate 32w + g + 8h, nibble
    // m + 4 = coordinate 32w + 16 + g + 8h.  Member m stores the chunks of g = 2m, 2m+1, whose
    // codes are byte m of every code word cw[r] of the four members: a 4 x 4 byte transpose
    // in the quad (two shuffles and two permutes per word) gives it T[r], byte s = byte m of
    // member s's cw[r].  Packing keeps nibble positions, so the selector words are the bytes'
    // low (g even) or high (g odd) nibbles side by side.
    const unsigned lane = threadIdx.x & 31;
    const int u = lane & 15, tq = (u & 7) >> 1, m = 2 * (u >> 3) + (u & 1);
    uint32_t qmask = active ? ((0xFu << (4 * m)) | (0xFu << (16 + 4 * m))) : 0u;
    qmask |= __shfl_xor_sync(0xffffffffu, qmask, 1);
    qmask |= __shfl_xor_sync(0xffffffffu, qmask, 8);
    // the storing member may lie outside the launch: take the block's page from an active one
    int qpage = active ? page : -1;
    qpage = max(qpage, __shfl_xor_sync(0xffffffffu, qpage, 1));
    qpage = max(qpage, __shfl_xor_sync(0xffffffffu, qpage, 8));
    uint8_t* blk = v_block(v, qpage < 0 ? 0 : qpage, head, slot);
    const uint32_t sel1 = (u & 1) ? 0x3715u : 0x6240u, sel2 = (u >> 3) ? 0x3276u : 0x5410u;
    uint32_t T[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      const uint32_t x = active ? cw[r] : 0u;  // members outside the launch contribute nothing
      const uint32_t w1 = prmt(x, __shfl_xor_sync(0xffffffffu, x, 1), sel1);
      T[r] = prmt(w1, __shfl_xor_sync(0xffffffffu, w1, 8), sel2);
    }
#pragma unroll
    for (int gg = 0; gg < 2; ++gg) {
      uint32_t wd[2 * BITS];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t sw[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const uint32_t xa = (gg ? T[4 * w + h] >> 4 : T[4 * w + h]) & 0x0F0F0F0Fu;
          const uint32_t xb = (gg ? T[4 * w + 2 + h] >> 4 : T[4 * w + 2 + h]) & 0x0F0F0F0Fu;
          sw[w] = prmt(xa | (xa >> 4), xb | (xb >> 4), 0x6420u);
        }
#pragma unroll
        for (int k = 0; k < BITS; ++k) wd[BITS * h + k] = pack_word<BITS>(k, sw[0], sw[1], sw[2], sw[3]);
      }
      if (qmask != 0u) {
        const int g = 2 * m + gg;
        uint32_t* dst = reinterpret_cast<uint32_t*>(blk + 2 * chunk_bytes(BITS) * (4 * g + tq));
        if (qmask == 0xFFFFFFFFu) {
          uint2* d2 = reinterpret_cast<uint2*>(dst);
#pragma unroll
          for (int i = 0; i < BITS; ++i) d2[i] = make_uint2(wd[2 * i], wd[2 * i + 1]);
        } else {
          // tokens of this quad outside the launch keep their bits
#pragma unroll
          for (int i = 0; i < 2 * BITS; ++i) {
            atomicAnd(reinterpret_cast<unsigned int*>(dst + i), ~qmask);
            atomicOr(reinterpret_cast<unsigned int*>(dst + i), wd[i]);
          }
        }
      }
    }
  }

  if (active) *norm_slot(v, page, head, slot, side) = __half_as_ushort(__float2half_rn(fminf(n, 65504.f)));
}

// Small appends (decode steps): one warp per vector (see warp_encode_vector).
constexpr int APP_WARPS = 4;
template <int KB, int VB>
__global__ void __launch_bounds__(APP_WARPS * 32)
append_kernel(LayerView v, const __half* __restrict__ k_src, const __half* __restrict__ v_src, int batch, int n_new,
              const int32_t* __restrict__ start_pos, const float* __restrict__ params_layer, KernelConsts kc) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const long vid = (long)blockIdx.x * APP_WARPS + (threadIdx.x >> 5);
  const int side = (int)(vid & 1);
  const long rest = vid >> 1;
  const int head = (int)(rest % v.n_kv_heads);
  const long rest2 = rest / v.n_kv_heads;
  const int i_new = (int)(rest2 % n_new);
  const int b = (int)(rest2 / n_new);
  if (b >= batch) return;  // warp-uniform
  const __half* src = side ? v_src : k_src;
  if (src == nullptr) return;
  const int pos = start_pos[b] + i_new;
  const int page = resolve_page(v, b, pos);
  if (page < 0) return;
  float Mp[4][4];
  variant_block_matrix(v.rot, block_params(params_layer, v.rot, head, lane), Mp);
  const __half* x = src + (((size_t)b * n_new + i_new) * v.n_kv_heads + head) * D;
  if (side == 0)
    warp_encode_vector<KB>(v, x, head, 0, page, pos % v.page_size, Mp, kc.k);
  else
    warp_encode_vector<VB>(v, x, head, 1, page, pos % v.page_size, Mp, kc.v);
}

template <int BITS>
static int launch_bulk(const LayerView& v, const void* k, const void* vsrc, int batch, int n_new,
                       const int32_t* start_pos, const float* params_layer, const KernelConsts& kc, void* stream,
                       int side0, int n_sides) {
  dim3 grid((n_new + 15 + ENC_THREADS - 1) / ENC_THREADS, v.n_kv_heads * n_sides, batch);
  auto kern = v.rot == ROT_ISO ? encode_kernel<BITS, true> : encode_kernel<BITS, false>;
  return (int)launch_pdl(kern, grid, dim3(ENC_THREADS), 0, (cudaStream_t)stream, v, (const __half*)k,
                         (const __half*)vsrc, n_new, start_pos, params_layer, side0 == 0 ? kc.k : kc.v, side0, n_sides);
}

template <int KB, int VB>
static int launch_encode_kv(const LayerView& v, const void* k, const void* vsrc, int batch, int n_new,
                            const int32_t* start_pos, const float* params_layer, const KernelConsts& kc, void* stream) {
  const long vectors = (long)batch * n_new * v.n_kv_heads * 2;
  if (n_new <= 8) {  // decode-style appends: latency matters, not throughput
    const long blocks = (vectors + APP_WARPS - 1) / APP_WARPS;
    return (int)launch_pdl(append_kernel<KB, VB>, dim3((unsigned)blocks), dim3(APP_WARPS * 32), 0,
                           (cudaStream_t)stream, v, (const __half*)k, (const __half*)vsrc, batch, n_new, start_pos,
                           params_layer, kc);
  }
  if (KB == VB) return launch_bulk<KB>(v, k, vsrc, batch, n_new, start_pos, params_layer, kc, stream, 0, 2);
  int e = k ? launch_bulk<KB>(v, k, nullptr, batch, n_new, start_pos, params_layer, kc, stream, 0, 1) : 0;
  if (e) return e;
  return vsrc ? launch_bulk<VB>(v, nullptr, vsrc, batch, n_new, start_pos, params_layer, kc, stream, 1, 1) : 0;
}

int launch_encode(const LayerView& v, const void* k, const void* vsrc, int batch, int n_new,
                  const int32_t* start_pos, const float* params_layer, const KernelConsts& kc, void* stream) {
  if (batch == 0 || n_new == 0) return 0;
#define IQ_ENC(KB, VB) \
  if (v.kb == KB && v.vb == VB) return launch_encode_kv<KB, VB>(v, k, vsrc, batch, n_new, start_pos, params_layer, kc, stream);
  IQ_ENC(2, 2)
  IQ_ENC(3, 2)
  IQ_ENC(3, 3)
  IQ_ENC(4, 2)
  IQ_ENC(4, 3)
  IQ_ENC(4, 4)
#undef IQ_ENC
  return (int)cudaErrorInvalidValue;
}

}  // namespace iq
