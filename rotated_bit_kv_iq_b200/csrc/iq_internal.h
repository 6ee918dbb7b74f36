// Internal declarations shared by the host and device translation units of libiq.
#pragma once
#include <cstddef>
#include <cstdint>

#include "../../include/iq.h"

namespace iq {

constexpr int D = 128;          // head dimension
constexpr int NBLK = 32;        // SO(4) blocks per head
constexpr int K_REC = 48;       // bytes of a K record (one token)
constexpr int V_BLK_TOKENS = 16;  // tokens per V block
constexpr int V_BLK = 768;      // bytes of a V block (16 tokens x 128 codes x 3 bits)
// Tile record: 32 consecutive slots of one (page, kv head), 3200 bytes:
//   [0, 1536) 32 K records | [1536, 3072) 2 V blocks | [3072, 3136) 32 K norms | [3136, 3200) 32 V norms
constexpr int TILE_TOKENS = 32;
constexpr int TR_K = 0;
constexpr int TR_V = TR_K + TILE_TOKENS * K_REC;
constexpr int TR_KN = TR_V + 2 * V_BLK;
constexpr int TR_VN = TR_KN + TILE_TOKENS * 2;
constexpr int TILE_BYTES = TR_VN + TILE_TOKENS * 2;
static_assert(TILE_BYTES == 3200, "tile record size");

// Lloyd-Max quantiser of N(0,1): 8 ascending levels, 7 midpoint boundaries (double).
struct Codebook {
  double level[8];
  double bound[7];
};
Codebook compute_codebook();

// Seeded rotation parameters, [L][Hkv][32][2][4] float32, written to `out` (host).
void init_rotation_params(uint64_t seed, int n_layers, int n_kv_heads, float* out);

// Constants handed to kernels by value.  The eight centroids reach the tensor cores as
// int8 pairs: alpha8 * c_k = hi_k + lo_k / 254 (hi_k, lo_k in [-127, 127]).
struct KernelConsts {
  float bound_pos[3];    // positive N(0,1) boundaries b4, b5, b6 (b3 = 0)
  uint32_t lut_hi[2];    // bytes hi_k, k = 0..3 in the first word, 4..7 in the second
  uint32_t lut_lo[2];    // bytes lo_k
  float alpha8;          // the int8 scale
};
const KernelConsts& kernel_consts();

// Device geometry of one layer's pools, resolved on the host.
struct LayerView {
  uint8_t* pool;         // layer base of the tile-record pool
  const int32_t* block_table;  // NULL -> sequence b uses page b
  int32_t max_pages;     // pages per sequence in the block table (1 when table is NULL)
  int32_t page_size;
  int32_t n_pages;
  int32_t n_kv_heads;
  uint32_t* status;
};

// Kernel launchers (defined in the .cu files); return the launch error.
int launch_encode(const LayerView& v, const void* k, const void* vsrc, int batch, int n_new,
                  const int32_t* start_pos, const float* params_layer, const KernelConsts& kc,
                  void* stream);
int launch_decode(const LayerView& v, const void* q, int q_f32, int batch, int n_q_heads,
                  const int32_t* ctx_len, int max_ctx, const float* params_layer, float* out,
                  void* workspace, const KernelConsts& kc, void* stream);
int launch_decode_step(const LayerView& v, const void* q, int q_f32, const void* k_new, const void* v_new, int batch,
                       int n_q_heads, const int32_t* ctx_len, int max_ctx, const float* params_layer, float* out,
                       void* workspace, const KernelConsts& kc, void* stream);
int launch_export(const LayerView& v, int kv, int seq, int t0, int n, uint8_t* codes,
                  uint16_t* norms, const KernelConsts& kc, void* stream);

// Decode grid (host): CTAs of one decode launch on the current device, given how many CTAs of
// the kernel an SM holds at once.
int decode_ctas(int batch, int n_kv_heads, int max_ctx, int resident_per_sm);
size_t decode_workspace_bytes(int batch, int n_q_heads, int n_kv_heads, int max_ctx);
size_t decode_counter_bytes(int batch, int n_kv_heads);  // leading bytes that must be zero between calls
constexpr int DECODE_MAX_BATCH = 2048;  // sequences per decode call (per-CTA plan in shared memory)

}  // namespace iq
