/*
 * iq.h -- C ABI of the IsoQuant packed KV cache library (libiq.so, sm_100a).
 *
 * What the library computes (sources are web pages, cited by title and section):
 *   - "RotaryQuant" write-up, rebasdaily.com 2026-08-14, section
 *     "妙处不只是压缩，而是不再展开": KV vectors are mixed by a Walsh-Hadamard
 *     transform and block-diagonal SO(4) rotations, scalar-quantised to 3 bits, and
 *     attention runs directly on the packed tensors (scores, softmax, value
 *     accumulation, one inverse rotation) without rebuilding full-precision K/V.
 *   - RotaryQuant abstract, arXiv 2608.08081 (arxivdaily entry): WHT followed by
 *     block-diagonal SO(4), 256 parameters per head, 3-bit scalar quantisation.
 *   - "压缩与速度的博弈——TurboQuant 和 RotorQuant 的真相" (zhichai.net), sections
 *     "Beta 分布的魔力" (rotated unit-vector coordinates ~ N(0, 1/d)) and
 *     "Lloyd-Max 最优量化" (the optimal scalar quantiser, applied by lookup).
 *   - "RotorQuant：LLM KV 缓存压缩的“几何革命”" (sd114.wiki), section
 *     "3. V 缓存的逆旋转修复": values must be rotated back with the inverse rotation;
 *     section "1. 绕过蝴蝶网络" and "压缩与速度的博弈" section "三种变体": the block rotations
 *     without the WHT (one quaternion per group of 4, or a Givens rotation per pair);
 *     "压缩与速度的博弈" section "K 和 V 的非对称需求": more bits for K than for V.
 *
 * Conventions for every entry point:
 *   - Pointers named *_dev / all tensors are DEVICE memory owned by the caller; the
 *     library never allocates, frees or retains them.  Host pointers are marked.
 *   - Calls are asynchronous on the given CUDA stream (NULL = legacy default stream);
 *     argument errors are detected on the host and returned before any launch.
 *   - Launch failures return IQ_ERR_CUDA (the CUDA error is left for the caller to
 *     read with cudaGetLastError / cudaPeekAtLastError).
 *   - Data-dependent errors found on the device (a position outside a sequence's
 *     pages, a block-table entry outside the pool, a context length outside
 *     [0, max_ctx]) never cause an out-of-range access: the offending token or
 *     sequence is skipped and an IQ_DEVERR_* bit is OR-ed into cache->status_dev
 *     when that pointer is non-NULL.
 *   - No C++ exception crosses this interface.
 *   - head_dim is 128; every device pointer must be 16-byte aligned (workspace 256).
 *
 * Code widths: K codes of kb bits and V codes of vb bits per coordinate, (kb, vb) one of
 *   (2,2), (3,2), (3,3), (4,2), (4,3), (4,4) (K never narrower than V); 3 bits by default.
 * Cache layout: one pool, [L][n_pages][Hkv][page_size/32] tile records of
 *   TB = 512 kb + 512 vb + 128 bytes (3200 for 3/3); the tile record of 32 consecutive slots
 *   s0..s0+31 (s0 a multiple of 32) holds
 *       bytes [0, 512 kb)                 the 32 K records, slot order (16 kb bytes each)
 *       bytes [512 kb, 512 (kb + vb))     the two V blocks of slots s0..s0+15 and s0+16..s0+31
 *       next 64 bytes                     the 32 K norms (binary16), then the 32 V norms
 *   (16 (kb + vb) + 4 bytes per token and kv head; 100 for 3/3; one tile record is one bulk copy
 *   for the decoder).
 *   Token t of sequence b lives on page
 *       block_table_dev[b * max_pages_per_seq + t / page_size]   (paged), or
 *       b                                                         (block_table_dev == NULL)
 *   at slot t % page_size.  page_size is a positive multiple of 32.
 *
 * Record formats (this library's own; the pages fix none):
 *   code k in 0..2^bits-1 = index of the ascending Lloyd-Max centroid of N(0,1):
 *       k = #{ j : u > b_j },  u = sqrt(128) * (R x / ||x||)
 *   32-code chunk = 4*bits bytes = little-endian uint32 words W0..W(bits-1); for j in 0..7:
 *       3 bits: bits [4j,4j+3) of Ww = code of slot 8w+j; bit 4j+3 of Ww = bit w of slot 24+j
 *       4 bits: bits [4j,4j+4) of Ww = code of slot 8w+j
 *       2 bits: bits [4j,4j+2) of Ww = code of slot 16w+j; bits [4j+2,4j+4) = slot 16w+8+j
 *   K record (per token): chunk c = 0..3, slot s -> coordinate 32c+s.
 *   V block (positions 16b..16b+15 of one sequence and kv head): 64 chunks, chunk
 *       (g, tq, h) (g 0..7, tq 0..3, h 0..1) at byte 4*bits*(2*(4g+tq)+h); its slot
 *       8*(m/2) + 4*(m%2) + j (m 0..7, j 0..3) holds token 8*(j/2) + 2*tq + (j%2) of the block
 *       at coordinate 16m + g + 8h.  Token u owns nibbles j, j+4 of the words of the 16 chunks
 *       with tq = (u%8)/2, j = 2*(u/8) + u%2, and nothing else (in every width).
 *   Norm: ||x||_2 of the fp16 input, rounded to binary16 (nearest even), saturating
 *       at 65504.
 *
 * Rotation R (iq_cache.rotation), parameters float32 [L][Hkv][P] (P per head):
 *   IQ_ROT_ISO (P = 256): [32][2][4] = per 4-coordinate block k the unit quaternions (qL, qR),
 *       each (w,x,y,z); R x = S(H x / sqrt(128)), H Sylvester-ordered, block k of S maps
 *       y[4k..4k+3] (read as a quaternion) to qL * y * conj(qR).
 *   IQ_ROT_QUAT (P = 128): [32][4] = one unit quaternion q per block; block k maps
 *       x[4k..4k+3] to q * x (no WHT).
 *   IQ_ROT_PLANAR (P = 128): [64][2] = (c, s) per coordinate pair i; (x[2i], x[2i+1]) ->
 *       (c x0 - s x1, s x0 + c x1) (no WHT).
 *   Every stored quaternion and (c, s) pair is rescaled to unit length at use.
 */
#ifndef IQ_H
#define IQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* iq_stream_t; /* same type as cudaStream_t */

typedef enum {
  IQ_OK = 0,
  IQ_ERR_INVALID_ARG = 1, /* NULL pointer, negative size, inconsistent shapes */
  IQ_ERR_UNSUPPORTED = 2, /* head_dim != 128, GQA group size above 8, bad dtype, code widths or
                             rotation variant not supported */
  IQ_ERR_CAPACITY = 3,    /* a host-known size exceeds the cache's capacity */
  IQ_ERR_WORKSPACE = 4,   /* workspace NULL or smaller than iq_decode_workspace_size */
  IQ_ERR_ALIGNMENT = 5,   /* a device pointer is not 16-byte aligned (workspace: 256) */
  IQ_ERR_CUDA = 6         /* a kernel launch or CUDA runtime call failed */
} iq_status;

typedef enum { IQ_F16 = 0, IQ_F32 = 1 } iq_dtype;

typedef enum { IQ_ROT_ISO = 0, IQ_ROT_QUAT = 1, IQ_ROT_PLANAR = 2 } iq_rotation;

/* Bits OR-ed into *status_dev by kernels that meet bad data (see conventions). */
#define IQ_DEVERR_POSITION 1u /* token position outside its sequence's pages */
#define IQ_DEVERR_PAGE 2u     /* block-table entry outside [0, n_pages) */
#define IQ_DEVERR_CTX 4u      /* context length outside [0, max_ctx] */
#define IQ_DEVERR_TIMEOUT 8u  /* a bounded wait inside a kernel gave up (outputs undefined) */
#define IQ_DEVERR_WORKSPACE 16u /* decode workspace counters were not zero (outputs undefined) */

typedef struct {
  void* pool;                      /* device, tile records (see layout above), 16-byte aligned */
  int32_t n_layers;                /* L >= 1 */
  int32_t n_kv_heads;              /* Hkv >= 1 */
  int32_t head_dim;                /* must be 128 */
  int32_t page_size;               /* tokens per page, multiple of 32 */
  int32_t n_pages;                 /* pages in the pool */
  const int32_t* block_table_dev;  /* [batch][max_pages_per_seq] or NULL */
  int32_t max_pages_per_seq;       /* ignored when block_table_dev is NULL */
  uint32_t* status_dev;            /* device word for IQ_DEVERR_* bits, or NULL */
  int32_t k_bits;                  /* K code width: 2, 3 or 4 (0 = 3) */
  int32_t v_bits;                  /* V code width: 2, 3 or 4 (0 = 3); (k_bits, v_bits) as listed above */
  int32_t rotation;                /* iq_rotation */
} iq_cache;

/* Library version string (static storage). */
const char* iq_version(void);

/* Human-readable text of a status code (static storage; never NULL). */
const char* iq_status_string(iq_status s);

/* Bytes of the cache pool for the given geometry and code widths (0 = 3 bits; 100 bytes per
 * token slot and kv head for 3/3).  Host-only; returns IQ_ERR_INVALID_ARG on bad sizes (page_size
 * not a positive multiple of 32), IQ_ERR_UNSUPPORTED for a width pair not listed above. */
iq_status iq_cache_bytes(int32_t n_layers, int32_t n_kv_heads, int32_t page_size, int32_t n_pages, int32_t k_bits,
                         int32_t v_bits, size_t* pool_bytes_host);

/* Rotation parameters from a seed (host-only; writes n_layers*n_kv_heads*256 floats to
 * params_host).  Defined by: RotaryQuant abstract (arXiv 2608.08081), 256 parameters per head
 * for the block-diagonal SO(4) stage; "RotaryQuant" (rebasdaily.com), section
 * "妙处不只是压缩，而是不再展开", the WHT + SO(4) structure they parametrise.  Each quaternion is drawn uniformly from the unit 3-sphere by Marsaglia's
 * method from a splitmix64 counter stream keyed by (seed, layer, head, block, side); the
 * pages publish no parameter values, they fix only their number (256 per head).
 * Errors: IQ_ERR_INVALID_ARG for NULL params_host or non-positive sizes. */
iq_status iq_init_rotation(uint64_t seed, int32_t n_layers, int32_t n_kv_heads, float* params_host);

/* Parameters per head of a rotation variant (256, 128, 128), 0 for an unknown value. */
int32_t iq_rotation_params_per_head(int32_t rotation);

/* Rotation parameters of any variant (host-only; writes n_layers*n_kv_heads*P floats).
 * IQ_ROT_ISO gives the same values as iq_init_rotation; IQ_ROT_QUAT draws one quaternion per
 * block from the unit 3-sphere, IQ_ROT_PLANAR one (c, s) pair per coordinate pair from the unit
 * circle (a disc point by rejection, normalised), each from its own splitmix64 stream.
 * Defined by: "压缩与速度的博弈" (zhichai.net), section "三种变体" (128 parameters for the
 * quaternion and the Givens variants); "RotorQuant" (sd114.wiki), section "1. 绕过蝴蝶网络".
 * Errors: IQ_ERR_INVALID_ARG for NULL params_host or non-positive sizes, IQ_ERR_UNSUPPORTED for
 * an unknown variant. */
iq_status iq_init_rotation_variant(uint64_t seed, int32_t rotation, int32_t n_layers, int32_t n_kv_heads,
                                   float* params_host);

/* Quantise-and-append: encode n_new new tokens of every sequence into layer `layer`.
 * Defined by: "RotaryQuant" (rebasdaily.com), section "妙处不只是压缩，而是不再展开" (rotate,
 * then scalar-quantise each coordinate to 3 bits and pack); "压缩与速度的博弈" (zhichai.net),
 * sections "Beta 分布的魔力" (rotated unit-vector coordinates ~ N(0, 1/d)) and "Lloyd-Max 最优量化"
 * (the quantiser).
 *   k_dev, v_dev : fp16 [batch][n_new][Hkv][128]; either may be NULL (that side skipped).
 *   start_pos_dev: int32 [batch], position of each sequence's first new token.
 *   params_dev   : float32 [L][Hkv][P] of the cache's rotation variant.
 * Per vector: norm (fp32 accumulate) -> rotation (WHT + SO(4) blocks, or the variant's blocks)
 * -> threshold search against the 2^bits - 1 Lloyd-Max boundaries -> packed record + binary16
 * norm written at its slot.
 * Writes only the bits of the tokens it encodes (the other tokens of a V block keep theirs;
 * tokens of one block may come from different calls, but calls that overlap on the GPU must
 * not append to the same block).  Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, CUDA; IQ_DEVERR_POSITION /
 * IQ_DEVERR_PAGE on the device. */
iq_status iq_encode_append(const iq_cache* cache, int32_t layer, const void* k_dev, const void* v_dev,
                           int32_t batch, int32_t n_new, const int32_t* start_pos_dev,
                           const float* params_dev, iq_stream_t stream);

/* Workspace bytes iq_decode_attention / iq_decode_step need for these sizes on the current
 * device: per-(sequence, kv head) arrival counters followed by the split partials.  The
 * counters must be zero when a call starts: zero-fill a new workspace once (e.g.
 * cudaMemsetAsync); every call leaves them zero again, so the buffer can be reused by later
 * calls on the same stream.  A call cut short by a device error (IQ_DEVERR_TIMEOUT) may leave
 * them set: zero-fill again after one. */
size_t iq_decode_workspace_size(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int32_t max_ctx);

/* Decode attention over the packed cache of layer `layer`.
 * Defined by: "RotaryQuant" (rebasdaily.com), section "妙处不只是压缩，而是不再展开" and its
 * abstract (attention directly on the packed tensors: rotated query, scores, softmax, value sum,
 * one inverse rotation); "RotorQuant" (sd114.wiki), section "3. V 缓存的逆旋转修复" (the value sum
 * goes back through the inverse rotation); "压缩与速度的博弈" (zhichai.net), section
 * "为什么压缩 KV 缓存这么难？" (softmax(Q K^T / sqrt(d)) V).
 *   q_dev        : [batch][n_q_heads][128], fp16 (IQ_F16) or fp32 (IQ_F32).
 *   ctx_len_dev  : int32 [batch], tokens 0..ctx_len-1 of each sequence are attended;
 *                  0 gives a zero output row; values outside [0, max_ctx] are clamped
 *                  into range and flagged with IQ_DEVERR_CTX.
 *   max_ctx      : host upper bound on ctx_len (sizes the split-K grid); must not exceed
 *                  the per-sequence capacity (page_size, or page_size*max_pages_per_seq).
 *   params_dev   : float32 [L][Hkv][P], the parameters used when encoding.
 *   out_dev      : float32 [batch][n_q_heads][128].
 *   workspace_dev: at least iq_decode_workspace_size(...) bytes, 256-byte aligned,
 *                  zero-filled before its first use (see iq_decode_workspace_size); calls
 *                  that overlap on the GPU must not share one.
 *   batch        : at most 2048 (IQ_ERR_UNSUPPORTED above).
 * q head h reads kv head h / (n_q_heads / n_kv_heads); that group size must be 1 .. 8 (every call
 * below has the same limit).
 * out[b][h] = sum_t softmax_t(<q, K_t>/sqrt(128)) V_t with K_t, V_t the dequantised
 * vectors n * R^T c[codes] / sqrt(128), computed without forming them: q is rotated once,
 * scores and the value sum are formed in the rotated basis from codes and norms,
 * split-K partials are merged, and one inverse rotation is applied per output row.
 * Ordering: launched with programmatic dependent launch, but the kernel waits for the
 * preceding kernel on the stream before it reads or writes anything. */
iq_status iq_decode_attention(const iq_cache* cache, int32_t layer, const void* q_dev, iq_dtype q_dtype,
                              int32_t batch, int32_t n_q_heads, const int32_t* ctx_len_dev, int32_t max_ctx,
                              const float* params_dev, float* out_dev, void* workspace_dev,
                              size_t workspace_bytes, iq_stream_t stream);

/* Decode step: append one new token to every sequence and attend over it, in one kernel.
 * Defined by: the two calls above; "RotorQuant" (sd114.wiki), section "2. 延迟量化策略" (a token
 * generated during decoding is quantised when it is inserted into the cache).
 *   k_new_dev, v_new_dev: fp16 [batch][Hkv][128], the new token's K and V; it is encoded (as by
 *                  iq_encode_append) into position ctx_len[b]-1 of sequence b.
 *   Other arguments and the result as for iq_decode_attention over positions [0, ctx_len[b]);
 *   ctx_len[b] >= 1 counts the new token.  Same result as iq_encode_append(start_pos =
 *   ctx_len-1, n_new = 1) followed by iq_decode_attention, without the separate launch.
 * Ordering: the kernel may start while the kernel issued just before it on the stream is
 * still running (programmatic dependent launch).  Before waiting for that kernel it reads
 * only ctx_len_dev, the block table, params (the rotation of one kv head) and the cached
 * records of positions < ctx_len-1 (it starts their bulk loads); q, k_new and v_new are
 * read, and the cache, workspace and out are written, only after the wait.  So the
 * immediately preceding kernel must not write ctx_len, the block table, params or older
 * cache positions (host copies and earlier kernels may). */
iq_status iq_decode_step(const iq_cache* cache, int32_t layer, const void* q_dev, iq_dtype q_dtype,
                         const void* k_new_dev, const void* v_new_dev, int32_t batch, int32_t n_q_heads,
                         const int32_t* ctx_len_dev, int32_t max_ctx, const float* params_dev, float* out_dev,
                         void* workspace_dev, size_t workspace_bytes, iq_stream_t stream);

/* Deferred quantisation ("RotorQuant" (sd114.wiki), section "2. 延迟量化策略"; "压缩与速度的博弈"
 * (zhichai.net), section "延迟量化（Deferred Quantization）"): the prompt's K/V stay fp16 as the model
 * produced them (no rotation, no quantisation) and tokens generated during decoding are quantised
 * when they are inserted.  An fp16 prefix of one layer: */
typedef struct {
  const void* k_dev;       /* device fp16 [batch][n_kv_heads][max_len][128], unrotated K of positions 0.. */
  const void* v_dev;       /* device fp16 [batch][n_kv_heads][max_len][128], unrotated V */
  const int32_t* len_dev;  /* device int32 [batch]: positions 0 .. len-1 of sequence b are here */
  int32_t max_len;         /* capacity of the arrays per sequence and kv head (tokens) */
} iq_fp16_prefix;

/* Workspace bytes iq_decode_step_deferred needs (the decode workspace plus the fp16 prefix's
 * split partials); zero-filled before its first use, like the decode workspace. */
size_t iq_decode_deferred_workspace_size(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads, int32_t max_ctx,
                                         int32_t max_len);

/* Decode step over a cache whose first len[b] positions are the fp16 prefix: the new token (k_new,
 * v_new, position ctx_len[b]-1) is quantised and appended to the packed cache like
 * iq_decode_step, and every query head attends over positions 0 .. ctx_len[b]-1: the prefix's from
 * the fp16 arrays (exact fp16 products, fp32 sums), positions len[b] .. ctx_len[b]-1 from the
 * packed cache.  Requires 0 <= len[b] < ctx_len[b] and len[b] <= max_len (values outside are
 * clamped and flagged with IQ_DEVERR_CTX); the packed cache is read from the tile holding
 * position len[b] on (earlier positions of that tile are ignored).  Other arguments, results and
 * errors as for iq_decode_step, with the workspace of iq_decode_deferred_workspace_size.  Two
 * kernels: the prefix's attention (split partials, rotated forward into the packed basis), then
 * the fused step, which merges both before its single inverse rotation.  Ordering: the first
 * kernel may start while the kernel issued just before the call is still running; before
 * waiting for it, it reads only len_dev and ctx_len_dev and starts the bulk loads of the fp16
 * arrays' first tiles, so that kernel must not write len, ctx_len or the fp16 arrays (host
 * copies and earlier kernels may).  q is read, and the workspace written, only after the wait.
 * The second kernel starts once the first is past that wait, attends over the packed tail
 * while the first is still running, and waits for it only before merging its partials. */
iq_status iq_decode_step_deferred(const iq_cache* cache, int32_t layer, const iq_fp16_prefix* prefix, const void* q_dev,
                                  iq_dtype q_dtype, const void* k_new_dev, const void* v_new_dev, int32_t batch,
                                  int32_t n_q_heads, const int32_t* ctx_len_dev, int32_t max_ctx,
                                  const float* params_dev, float* out_dev, void* workspace_dev, size_t workspace_bytes,
                                  iq_stream_t stream);

/* Workspace bytes iq_prefill_attention needs for these sizes on the current device (per query
 * block of 8 tokens, kv head and split of the context: the split partials).  Needs no zeroing. */
size_t iq_prefill_workspace_size(int32_t batch, int32_t n_tokens, int32_t n_kv_heads, int32_t max_ctx);

/* Chunked-prefill attention over the packed cache of layer `layer`: n_tokens query tokens per
 * sequence, causal.  Defined by: "RotaryQuant" (rebasdaily.com), section
 * "妙处不只是压缩，而是不再展开" (attention on the packed tensors), applied to a chunk of prompt
 * tokens; "RotorQuant" (sd114.wiki), section "性能基准", and "压缩与速度的博弈" (zhichai.net),
 * section "宣称的数字", report prefill speed over such caches.
 *   q_dev        : [batch][n_tokens][n_q_heads][128], fp16 (IQ_F16) or fp32 (IQ_F32).
 *   start_pos_dev: int32 [batch]; query token i of sequence b is at position start_pos[b] + i and
 *                  attends to positions 0 .. start_pos[b] + i of the cache, which must hold them
 *                  (append the chunk's K/V with iq_encode_append first).  Values outside
 *                  [0, max_ctx - n_tokens] are clamped into range and flagged with IQ_DEVERR_CTX.
 *   max_ctx      : host upper bound on start_pos + n_tokens (sizes the split of the work); must
 *                  not exceed the per-sequence capacity.
 *   out_dev      : float32 [batch][n_tokens][n_q_heads][128].
 *   workspace_dev: at least iq_prefill_workspace_size(...) bytes, 256-byte aligned.
 * Each CTA takes up to 128 query rows (floor(128 / G) tokens x the G query heads of one kv head)
 * and expands every 64-token step of packed K/V it loads once for all of them
 * (binary16 hi/lo operands on the tensor cores, fp32 accumulators); the result equals
 * iq_decode_attention of each query token over its own causal context within the tolerance of
 * that call.  Two kernels (attention splits, then their merge with the inverse rotation); they
 * wait for the preceding kernel on the stream before reading anything. */
iq_status iq_prefill_attention(const iq_cache* cache, int32_t layer, const void* q_dev, iq_dtype q_dtype, int32_t batch,
                               int32_t n_tokens, int32_t n_q_heads, const int32_t* start_pos_dev, int32_t max_ctx,
                               const float* params_dev, float* out_dev, void* workspace_dev, size_t workspace_bytes,
                               iq_stream_t stream);

/* Size of the fixed device scratch used by iq_decode_attention_noalloc (per device). */
#define IQ_NOALLOC_SCRATCH_BYTES (4u << 20)

/* iq_decode_attention without a caller-provided workspace.  (The method has no counterpart:
 * this entry point only changes where the split-K scratch lives.)
 * For callers that may not allocate device memory -- plugins whose host owns every device
 * allocation, and services that must not allocate after start-up.  Inputs, outputs and their
 * meaning are those of iq_decode_attention; the split-K scratch is a fixed array of
 * IQ_NOALLOC_SCRATCH_BYTES inside the library on each device (kept until the process exits).
 * The call allocates nothing.  The first call on a device looks up that array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call before capturing a
 * stream.  Returns IQ_ERR_WORKSPACE when iq_decode_workspace_size(batch, n_q_heads, n_kv_heads,
 * max_ctx) exceeds IQ_NOALLOC_SCRATCH_BYTES.  All calls on a device share the one array: calls
 * that overlap on the GPU (other streams, or a second call before the first has finished on a
 * stream that is not ordered after it) race on it.  Each call clears the array's arrival
 * counters (cudaMemsetAsync on its stream) before the kernel; nothing else has to start zeroed.
 * The looked-up address is kept for the life of the process: after cudaDeviceReset (or anything
 * else that destroys the device's primary context) it is stale, and this entry point must not
 * be called on that device again. */
iq_status iq_decode_attention_noalloc(const iq_cache* cache, int32_t layer, const void* q_dev, iq_dtype q_dtype,
                                      int32_t batch, int32_t n_q_heads, const int32_t* ctx_len_dev,
                                      int32_t max_ctx, const float* params_dev, float* out_dev,
                                      iq_stream_t stream);

/* Read back tokens [t0, t0+n) of sequence `seq` in layer `layer` as canonical codes (a test
 * and inspection utility: the pages define no such call; it undoes only this library's own
 * bit layout):
 *   codes_dev: uint8 [Hkv][n][128] (coordinate order), norms_dev: uint16 [Hkv][n] or NULL.
 *   kv: 0 = K pool, 1 = V pool.  Host-checked against the sequence capacity. */
iq_status iq_export_codes(const iq_cache* cache, int32_t layer, int32_t kv, int32_t seq, int32_t t0,
                          int32_t n, uint8_t* codes_dev, uint16_t* norms_dev, iq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* IQ_H */
