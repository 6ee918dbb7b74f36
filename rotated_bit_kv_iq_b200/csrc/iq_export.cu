// Export kernel: packed K/V records -> canonical codes (uint8, coordinate order) and norms.
// One thread per (kv head, token); used to check the packed format against the oracle.
#include <cuda_runtime.h>

#include "iq_device.cuh"

namespace iq {

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
  if (kv == 0) {
    const uint32_t* rec = reinterpret_cast<const uint32_t*>(k_record(v, page, head, slot));
    for (int c = 0; c < 4; ++c) {
      const uint32_t w[3] = {rec[3 * c], rec[3 * c + 1], rec[3 * c + 2]};
      for (int s = 0; s < 32; ++s) {
        uint32_t code;
        if (s < 24) code = (w[s >> 3] >> (4 * (s & 7))) & 7u;
        else code = ((w[0] >> (4 * (s - 24) + 3)) & 1u) | (((w[1] >> (4 * (s - 24) + 3)) & 1u) << 1) |
                    (((w[2] >> (4 * (s - 24) + 3)) & 1u) << 2);
        y[32 * c + s] = (uint8_t)code;
      }
    }
  } else {
    // V block: chunk (g, tq, h) at 12 (2 (4g + tq) + h); slot 8 (m/2) + 4 (m mod 2) + j holds
    // this token (tq = (u mod 8)/2, j = 2 (u/8) + (u mod 2)) at coordinate 16m + g + 8h.
    const uint8_t* blk = v_block(v, page, head, slot);
    const int u = slot & 15, tq = (u & 7) >> 1, j = 2 * (u >> 3) + (u & 1);
    for (int g = 0; g < 8; ++g) {
      for (int h = 0; h < 2; ++h) {
        const uint32_t* w = reinterpret_cast<const uint32_t*>(blk + 12 * (2 * (4 * g + tq) + h));
        for (int m = 0; m < 8; ++m) {
          const int s = 8 * (m >> 1) + 4 * (m & 1) + j;
          uint32_t code;
          if (s < 24) code = (w[s >> 3] >> (4 * (s & 7))) & 7u;
          else code = ((w[0] >> (4 * (s - 24) + 3)) & 1u) | (((w[1] >> (4 * (s - 24) + 3)) & 1u) << 1) |
                      (((w[2] >> (4 * (s - 24) + 3)) & 1u) << 2);
          y[16 * m + g + 8 * h] = (uint8_t)code;
        }
      }
    }
  }
  for (int c = 0; c < D; ++c) out[c] = y[c];
  if (norms) norms[(size_t)head * n + i] = *norm_slot(v, page, head, slot, kv);
}

int launch_export(const LayerView& v, int kv, int seq, int t0, int n, uint8_t* codes, uint16_t* norms,
                  const KernelConsts&, void* stream) {
  if (n == 0) return 0;
  dim3 grid((n + 127) / 128, v.n_kv_heads);
  export_kernel<<<grid, 128, 0, (cudaStream_t)stream>>>(v, kv, seq, t0, n, codes, norms);
  return (int)cudaGetLastError();
}

}  // namespace iq
