// Quantise-and-append kernel: fp16 K/V vectors -> packed 3-bit records + binary16 norms.
//
// Steps per vector follow "RotaryQuant" (rebasdaily.com, section "妙处不只是压缩，而是不再展开")
// and its abstract (arXiv 2608.08081): Walsh-Hadamard mixing, then the block SO(4)
// rotation, then scalar quantisation; the quantiser is the Lloyd-Max codebook of N(0,1/d)
// ("压缩与速度的博弈" zhichai.net, sections "Beta 分布的魔力", "Lloyd-Max 最优量化").
//
// Mapping: one thread encodes one 128-vector entirely in registers (all seven butterfly
// stages are register-local, no shuffles).  A CTA covers 128 consecutive positions of one
// (sequence, kv head, K|V); the head's 32 fused block matrices live in shared memory and
// every lane of a warp reads the same one at the same time (broadcast).  Instead of
// normalising the vector, the rotated coordinates z = R x are compared with the
// boundaries scaled by ||x||/sqrt(128).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "iq_device.cuh"

namespace iq {

constexpr int ENC_THREADS = 128;

__global__ void __launch_bounds__(ENC_THREADS)
encode_kernel(LayerView v, const __half* __restrict__ k_src, const __half* __restrict__ v_src, int n_new,
              const int32_t* __restrict__ start_pos, const float* __restrict__ params_layer, KernelConsts kc) {
  // fused block matrices M'_k as column pairs: smat[k][c][0] = (M'[0][c], M'[1][c]),
  // smat[k][c][1] = (M'[2][c], M'[3][c])
  __shared__ uint64_t smat[NBLK][4][2];
  pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.z;
  const int head = blockIdx.y >> 1;
  const int side = blockIdx.y & 1;  // 0 = K, 1 = V
  const __half* src = side ? v_src : k_src;
  if (src == nullptr) return;

  if (threadIdx.x < NBLK) {
    float Mp[4][4];
    fused_block_matrix(params_layer + ((size_t)head * NBLK + threadIdx.x) * 8, Mp);
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
  // Fused SO(4) blocks: rows (0,1) and (2,3) as pairs, z = M' v.
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

  const float sc = n * 0.08838834764831845f;  // n / sqrt(128)
  const float t1 = kc.bound_pos[0] * sc, t2 = kc.bound_pos[1] * sc, t3 = kc.bound_pos[2] * sc;
  // codes once: cw[r] holds coordinates 8r..8r+7 as nibbles (bit 3 clear)
  uint32_t cw[16];
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    uint32_t w = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float za, zb;
      f2s(y[4 * r + e], za, zb);
      w |= quantise(za, t1, t2, t3) << (8 * e);
      w |= quantise(zb, t1, t2, t3) << (8 * e + 4);
    }
    cw[r] = w;
  }

  const int slot = pos % v.page_size;
  if (side == 0) {
    // K record: chunk c = cw[4c..4c+3]; word w of the chunk = slots 8w..8w+7 plus bit w of
    // slots 24..31 as the spare bits.
    if (active) {
      uint32_t rec[12];
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int w = 0; w < 3; ++w) rec[3 * c + w] = cw[4 * c + w] | (((cw[4 * c + 3] >> w) & 0x11111111u) << 3);
      uint4* dst = reinterpret_cast<uint4*>(k_record(v, page, head, slot));
      dst[0] = make_uint4(rec[0], rec[1], rec[2], rec[3]);
      dst[1] = make_uint4(rec[4], rec[5], rec[6], rec[7]);
      dst[2] = make_uint4(rec[8], rec[9], rec[10], rec[11]);
    }
  } else {
    // V block (16 tokens = 16 consecutive lanes): token u = lane mod 16 owns nibbles j and
    // j+4 of the words of chunks (g, tq, h), tq = (u mod 8)/2, j = 2 (u/8) + (u mod 2); word w
    // takes coordinates 32w + g + 8h, 32w + 16 + g + 8h and, as spare bits (bit w), 96 + g + 8h
    // and 112 + g + 8h.  The four tokens of a quad (lanes u, u^1, u^8, u^9) OR their words
    // together and member j stores the chunks of g = 2j, 2j+1 (24 contiguous bytes each).
    const unsigned lane = threadIdx.x & 31;
    const int u = lane & 15, tq = (u & 7) >> 1, j = 2 * (u >> 3) + (u & 1);
    uint32_t qmask = active ? ((0xFu << (4 * j)) | (0xFu << (16 + 4 * j))) : 0u;
    qmask |= __shfl_xor_sync(0xffffffffu, qmask, 1);
    qmask |= __shfl_xor_sync(0xffffffffu, qmask, 8);
    // the storing member may lie outside the launch: take the block's page from an active one
    int qpage = active ? page : -1;
    qpage = max(qpage, __shfl_xor_sync(0xffffffffu, qpage, 1));
    qpage = max(qpage, __shfl_xor_sync(0xffffffffu, qpage, 8));
    uint8_t* blk = v_block(v, qpage < 0 ? 0 : qpage, head, slot);
#pragma unroll 1
    for (int g = 0; g < 8; ++g) {  // rolled: keeps the kernel's code small
      uint32_t wd[6];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // codes of coordinates 16m + g + 8h: nibble g of cw[2m + h]
        uint32_t cm[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) cm[m] = (cw[2 * m + h] >> (4 * g)) & 7u;
#pragma unroll
        for (int w = 0; w < 3; ++w) {
          const uint32_t n0 = cm[2 * w] | (((cm[6] >> w) & 1u) << 3), n1 = cm[2 * w + 1] | (((cm[7] >> w) & 1u) << 3);
          uint32_t part = active ? ((n0 << (4 * j)) | (n1 << (16 + 4 * j))) : 0u;
          part |= __shfl_xor_sync(0xffffffffu, part, 1);
          part |= __shfl_xor_sync(0xffffffffu, part, 8);
          wd[3 * h + w] = part;
        }
      }
      if (j == (g >> 1) && qmask != 0u) {
        uint32_t* dst = reinterpret_cast<uint32_t*>(blk + 24 * (4 * g + tq));
        if (qmask == 0xFFFFFFFFu) {
          uint2* d2 = reinterpret_cast<uint2*>(dst);
          d2[0] = make_uint2(wd[0], wd[1]);
          d2[1] = make_uint2(wd[2], wd[3]);
          d2[2] = make_uint2(wd[4], wd[5]);
        } else {
          // tokens of this quad outside the launch keep their bits
#pragma unroll
          for (int i = 0; i < 6; ++i) {
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
  fused_block_matrix(params_layer + ((size_t)head * NBLK + lane) * 8, Mp);
  warp_encode_vector(v, src + (((size_t)b * n_new + i_new) * v.n_kv_heads + head) * D, head, side, page,
                     pos % v.page_size, Mp, kc);
}

int launch_encode(const LayerView& v, const void* k, const void* vsrc, int batch, int n_new,
                  const int32_t* start_pos, const float* params_layer, const KernelConsts& kc, void* stream) {
  if (batch == 0 || n_new == 0) return 0;
  const long vectors = (long)batch * n_new * v.n_kv_heads * 2;
  if (n_new <= 8) {  // decode-style appends: latency matters, not throughput
    const long blocks = (vectors + APP_WARPS - 1) / APP_WARPS;
    return (int)launch_pdl(append_kernel, dim3((unsigned)blocks), dim3(APP_WARPS * 32), 0, (cudaStream_t)stream, v,
                           (const __half*)k, (const __half*)vsrc, batch, n_new, start_pos, params_layer, kc);
  }
  dim3 grid((n_new + 15 + ENC_THREADS - 1) / ENC_THREADS, v.n_kv_heads * 2, batch);
  return (int)launch_pdl(encode_kernel, grid, dim3(ENC_THREADS), 0, (cudaStream_t)stream, v, (const __half*)k,
                         (const __half*)vsrc, n_new, start_pos, params_layer, kc);
}

}  // namespace iq
