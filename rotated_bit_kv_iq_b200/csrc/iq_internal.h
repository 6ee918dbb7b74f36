// Internal declarations shared by the host and device translation units of libiq.
#pragma once
#include <cstddef>
#include <cstdint>

#include "../../include/iq.h"

#ifdef __CUDACC__
#define IQ_HD __host__ __device__
#else
#define IQ_HD
#endif

namespace iq {

constexpr int D = 128;            // head dimension
constexpr int NBLK = 32;          // 4-coordinate rotation blocks per head
constexpr int V_BLK_TOKENS = 16;  // tokens per V block
constexpr int TILE_TOKENS = 32;   // slots per tile record

// Record geometry for a code width of `bits` (2, 3 or 4) per coordinate.  A chunk holds 32
// codes in `bits` 32-bit words; a K record is four chunks (one token); a V block is 64 chunks
// (16 tokens).  Tile record of 32 consecutive slots of one (page, kv head) with K width kb and
// V width vb:
//   [0, tr_v)        32 K records
//   [tr_v, tr_kn)    2 V blocks
//   [tr_kn, tr_vn)   32 K norms (binary16)
//   [tr_vn, +64)     32 V norms (binary16)
IQ_HD constexpr int chunk_bytes(int bits) { return 4 * bits; }
IQ_HD constexpr int k_rec_bytes(int bits) { return 16 * bits; }
IQ_HD constexpr int v_blk_bytes(int bits) { return 256 * bits; }
IQ_HD constexpr int tr_v(int kb) { return TILE_TOKENS * k_rec_bytes(kb); }
IQ_HD constexpr int tr_kn(int kb, int vb) { return tr_v(kb) + 2 * v_blk_bytes(vb); }
IQ_HD constexpr int tr_vn(int kb, int vb) { return tr_kn(kb, vb) + 2 * TILE_TOKENS; }
IQ_HD constexpr int tile_bytes(int kb, int vb) { return tr_vn(kb, vb) + 2 * TILE_TOKENS; }
static_assert(tile_bytes(3, 3) == 3200, "tile record size of the 3-bit format");

// The (K, V) code widths the kernels are built for (K never narrower than V).
IQ_HD constexpr bool supported_widths(int kb, int vb) {
  return (kb == 2 && vb == 2) || (kb == 3 && (vb == 2 || vb == 3)) || (kb == 4 && vb >= 2 && vb <= 4);
}

// Rotation variants (iq_rotation): WHT + quaternion pairs, one quaternion per block, Givens pairs.
constexpr int ROT_ISO = 0, ROT_QUAT = 1, ROT_PLANAR = 2;
IQ_HD constexpr int params_per_head(int rot) { return rot == ROT_ISO ? 256 : 128; }
IQ_HD constexpr int params_per_block(int rot) { return rot == ROT_ISO ? 8 : 4; }

// Lloyd-Max quantiser of N(0,1) with 2^bits ascending levels and midpoint boundaries (double).
struct Codebook {
  int bits;
  double level[16];
  double bound[15];
};
Codebook compute_codebook(int bits);

// Seeded rotation parameters, [L][Hkv][params_per_head(rot)] float32, written to `out` (host).
void init_rotation_params(uint64_t seed, int rot, int n_layers, int n_kv_heads, float* out);

// Constants of one side's (K or V) codebook handed to kernels by value.  The levels reach the
// tensor cores as int8 pairs: alpha8 * c_k = hi_k + lo_k / 254 (hi_k, lo_k in [-127, 127]);
// byte k of the little-endian words lut_hi / lut_lo is entry k (2^bits entries).
struct SideConsts {
  float bound_pos[7];  // positive N(0,1) boundaries, ascending (the middle boundary is 0)
  uint32_t lut_hi[4];
  uint32_t lut_lo[4];
  float alpha8;
  int bits;
  // the N(0,1) centroids as binary16 pairs c = c_hi + c_lo: low bytes (f16_lb) and high bytes
  // (f16_hb) of term t (0 = hi, 1 = lo) of entry k at byte k % 4 of word k / 4
  uint32_t f16_lb[2][4];
  uint32_t f16_hb[2][4];
};
struct KernelConsts {
  SideConsts k, v;
};
const KernelConsts& kernel_consts(int kb, int vb);

// Device geometry of one layer's pools, resolved on the host.
struct LayerView {
  uint8_t* pool;               // layer base of the tile-record pool
  const int32_t* block_table;  // NULL -> sequence b uses page b
  int32_t max_pages;           // pages per sequence in the block table (1 when table is NULL)
  int32_t page_size;
  int32_t n_pages;
  int32_t n_kv_heads;
  uint32_t* status;
  int32_t kb, vb;              // K and V code widths
  int32_t rot;                 // rotation variant
};

// An fp16 prefix of the cache (deferred quantisation), resolved on the host: positions
// 0 .. len[b]-1 of sequence b live in fp16 [batch][Hkv][max_len][128] K and V arrays; their
// attention arrives as n_extra partials per (sequence, kv head).
struct DeferredInfo {
  const int32_t* len;
  int n_extra;
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
int launch_prefill(const LayerView& v, const void* q, int q_f32, int batch, int n_tok, int n_q_heads,
                   const int32_t* start, int max_ctx, const float* params_layer, float* out, void* workspace,
                   const KernelConsts& kc, void* stream);
size_t prefill_workspace_bytes(int batch, int n_tok, int n_kv_heads, int max_ctx);
int launch_export(const LayerView& v, int kv, int seq, int t0, int n, uint8_t* codes,
                  uint16_t* norms, void* stream);

// Decode grid (host): CTAs of one decode launch on the current device, given how many CTAs of
// the kernel an SM holds at once.
int decode_ctas(int batch, int n_kv_heads, int max_ctx, int resident_per_sm);
size_t decode_workspace_bytes(int batch, int n_q_heads, int n_kv_heads, int max_ctx, int extra_slots = 0);
int prefix_splits(int batch, int n_kv_heads, int max_len, int n_sm);
int sm_count();
// CTAs of kernel fn with the given dynamic shared memory and block size that fit on one SM.
int resident_per_sm(const void* fn, size_t smem, int threads);
int launch_prefix(const LayerView& v, const void* k16, const void* v16, const int32_t* len, int max_len,
                  const int32_t* ctx_len, int max_ctx, const void* q, int q_f32, int batch, int n_q_heads,
                  const float* params_layer, const KernelConsts& kc, void* workspace, int splits, int extra_base,
                  void* stream);
int launch_decode_deferred(const LayerView& v, const void* q, int q_f32, const void* k_new, const void* v_new,
                           int batch, int n_q_heads, const int32_t* ctx_len, int max_ctx, const float* params_layer,
                           float* out, void* workspace, const KernelConsts& kc, void* stream, const void* k16,
                           const void* v16, const int32_t* len, int max_len);
size_t decode_counter_bytes(int batch, int n_kv_heads);  // leading bytes that must be zero between calls
constexpr int DECODE_MAX_BATCH = 2048;  // sequences per decode call (per-CTA plan in shared memory)

}  // namespace iq
