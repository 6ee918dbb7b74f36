// Export kernel: packed K/V records -> canonical codes (uint8, coordinate order) and norms.
// One thread per (kv head, token); used to check the packed format against the oracle.
#include <cuda_runtime.h>

#include "iq_device.cuh"

namespace iq {

// The 32 codes of one chunk (slot order) from its storage words.
template <int BITS>
__device__ __forceinline__ void chunk_codes(const uint8_t* chunk, uint8_t y[32]) {
  uint32_t w[BITS], sel[4];
  for (int i = 0; i < BITS; ++i) w[i] = reinterpret_cast<const uint32_t*>(chunk)[i];
  chunk_selectors<BITS>(w, sel);
  for (int s = 0; s < 32; ++s) y[s] = (uint8_t)((sel[s >> 3] >> (4 * (s & 7))) & 0xFu);
}

template <int BITS>
__device__ void export_token(const LayerView& v, int kv, int page, int head, int slot, uint8_t* y) {
  uint8_t c[32];
  if (kv == 0) {
    // K record: chunk c holds coordinates 32c .. 32c+31 in slot order
    const uint8_t* rec = k_record(v, page, head, slot);
    for (int ch = 0; ch < 4; ++ch) {
      chunk_codes<BITS>(rec + chunk_bytes(BITS) * ch, c);
      for (int s = 0; s < 32; ++s) y[32 * ch + s] = c[s];
    }
  } else {
    // V block: chunk (g, tq, h) at 2 (4g + tq) + h; slot 8 (m/2) + 4 (m mod 2) + j holds this
    // token (tq = (u mod 8)/2, j = 2 (u/8) + (u mod 2)) at coordinate 16m + g + 8h.
    const uint8_t* blk = v_block(v, page, head, slot);
    const int u = slot & 15, tq = (u & 7) >> 1, j = 2 * (u >> 3) + (u & 1);
    for (int g = 0; g < 8; ++g)
      for (int h = 0; h < 2; ++h) {
        chunk_codes<BITS>(blk + chunk_bytes(BITS) * (2 * (4 * g + tq) + h), c);
        for (int m = 0; m < 8; ++m) y[16 * m + g + 8 * h] = c[8 * (m >> 1) + 4 * (m & 1) + j];
      }
  }
}

__global__ void export_kernel(LayerView v, int kv, int seq, int t0, int n, uint8_t* __restrict__ codes,
                              uint16_t* __restrict__ norms) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int head = blockIdx.y;
  if (i >= n) return;
  const int pos = t0 + i;
  const int page = resolve_page(v, seq, pos);
  uint8_t* out = codes + ((size_t)head * n + i) * D;
  if (page < 0) {
    for (int c = 0; c < D; ++c) out[c] = 0xFF;
    if (norms) norms[(size_t)head * n + i] = 0xFFFF;
    return;
  }
  const int slot = pos % v.page_size;
  uint8_t y[D];
  const int bits = kv == 0 ? v.kb : v.vb;
  if (bits == 2) export_token<2>(v, kv, page, head, slot, y);
  else if (bits == 3) export_token<3>(v, kv, page, head, slot, y);
  else export_token<4>(v, kv, page, head, slot, y);
  for (int c = 0; c < D; ++c) out[c] = y[c];
  if (norms) norms[(size_t)head * n + i] = *norm_slot(v, page, head, slot, kv);
}

int launch_export(const LayerView& v, int kv, int seq, int t0, int n, uint8_t* codes, uint16_t* norms, void* stream) {
  if (n == 0) return 0;
  dim3 grid((n + 127) / 128, v.n_kv_heads);
  export_kernel<<<grid, 128, 0, (cudaStream_t)stream>>>(v, kv, seq, t0, n, codes, norms);
  return (int)cudaGetLastError();
}

}  // namespace iq
